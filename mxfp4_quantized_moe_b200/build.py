"""Builds the in-tree shared libraries with nvcc (sm_100a only).

* ``libmxfp4_moe.so``: the library.
* ``libmxfp4_moe_debug.so``: the same sources with ``-DMXFP4_MOE_DEBUG=1``: kernels check the
  indices they read from the workspace and record MXFP4_MOE_ERR_DEVICE_BOUNDS instead of
  making the access (``mxfp4_moe_build_flags`` reports the build).  Loaded instead of the
  library when ``MXFP4_MOE_LIBRARY=debug``.

Usage: ``python -m mxfp4_quantized_moe_b200.build [--verbose-ptxas]`` builds both.  Cross-compiles
without a GPU.  The libraries statically link the CUDA runtime, so they load on a machine
without a driver (calls then fail with MXFP4_MOE_ERR_CUDA).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmxfp4_moe.so")
LIB_DEBUG = os.path.join(HERE, "libmxfp4_moe_debug.so")
SOURCES = ["csrc/api.cu", "csrc/grouped_gemm.cu", "csrc/kernels_small.cu",
           "csrc/forward_static.cu", "csrc/selftest.cu", "csrc/residual_router.cu"]
DEPS = SOURCES + ["csrc/common.cuh", "csrc/kernels.h", "csrc/aux_kernels.h"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(HERE, d) for d in DEPS] + [os.path.join(ROOT, "include", "mxfp4_moe.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-Xcompiler", "-fvisibility=hidden",
           "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp"]
    if debug:
        cmd += ["-DMXFP4_MOE_DEBUG=1"]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(HERE, s) for s in SOURCES]
    r = subprocess.run(cmd, cwd=HERE, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if ptxas_verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


def build_all(force: bool = False, ptxas_verbose: bool = False) -> list[str]:
    return [build(force, ptxas_verbose), build(force, False, debug=True)]


if __name__ == "__main__":
    print("\n".join(build_all(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)))
