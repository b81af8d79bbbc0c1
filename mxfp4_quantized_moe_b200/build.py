"""Builds the in-tree shared library ``libmxfp4_moe.so`` with nvcc (sm_100a only).

Usage: ``python -m mxfp4_quantized_moe_b200.build [--verbose-ptxas]``.  Cross-compiles
without a GPU.  The library statically links the CUDA runtime, so it loads on a
machine without a driver (calls then fail with MXFP4_MOE_ERR_CUDA).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmxfp4_moe.so")
SOURCES = ["csrc/api.cu", "csrc/grouped_gemm.cu", "csrc/kernels_small.cu",
           "csrc/forward_static.cu", "csrc/selftest.cu"]
DEPS = SOURCES + ["csrc/common.cuh", "csrc/kernels.h", "csrc/aux_kernels.h"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(HERE, d) for d in DEPS] + [os.path.join(ROOT, "include", "mxfp4_moe.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-o", LIB + ".tmp"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(HERE, s) for s in SOURCES]
    r = subprocess.run(cmd, cwd=HERE, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if ptxas_verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))
