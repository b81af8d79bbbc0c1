"""The debug build (libmxfp4_moe_debug.so, device-side index checks in place of a sanitizer):
small-shape parity against the oracle, a planted out-of-range routing slot turned into
DEVICE_BOUNDS instead of an access, and an intact context afterwards.  It runs in a child
process because a process loads one build of the library."""

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_debug_build_parity_and_bounds_check():
    from mxfp4_quantized_moe_b200 import build
    build.build(debug=True)
    env = dict(os.environ, MXFP4_MOE_LIBRARY="debug")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_child.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
