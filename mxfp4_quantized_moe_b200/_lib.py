"""ctypes binding of ``libmxfp4_moe.so`` (the C ABI declared in include/mxfp4_moe.h).

Argument marshalling only: every step of the expert block runs in the library's CUDA
kernels.  Importing this module loads the in-tree library and fails loudly if it is
missing; there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# MXFP4_MOE_LIBRARY=debug loads the debug build (device-side index checks), else the library
_VARIANT = os.environ.get("MXFP4_MOE_LIBRARY", "")
if _VARIANT not in ("", "release", "debug"):
    raise RuntimeError(f"MXFP4_MOE_LIBRARY={_VARIANT!r}: expected 'debug' or 'release'")
LIB_PATH = os.path.join(HERE, "libmxfp4_moe_debug.so" if _VARIANT == "debug" else "libmxfp4_moe.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_WORKSPACE_TOO_SMALL = -2
ERR_UNSUPPORTED_DEVICE = -3
ERR_CUDA = -4
ERR_DEVICE_TIMEOUT = -5
ERR_DEVICE_BOUNDS = -6

# every symbol the header declares, with (restype, argtypes)
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("glu_alpha", ctypes.c_float),
                ("glu_limit", ctypes.c_float), ("gate_up_format", ctypes.c_int32)]


GATE_UP_BF16 = 0
GATE_UP_BLOCK_SCALED = 1


class Weights(ctypes.Structure):
    _fields_ = [("gu_blocks", _vp), ("gu_scales", _vp), ("gu_bias", _vp),
                ("dn_blocks", _vp), ("dn_scales", _vp), ("dn_bias", _vp)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_double)]


SIGNATURES = {
    "mxfp4_moe_workspace_size": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(_sz)]),
    "mxfp4_moe_transposed_weights_size": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(_sz)]),
    "mxfp4_moe_transpose_weights": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Weights),
                                                   _vp, _sz, _vp]),
    "mxfp4_moe_forward": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Weights), _vp, _vp,
                                         _vp, _vp, _vp, _vp, _sz, _vp]),
    "mxfp4_moe_forward_static": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Weights),
                                                _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_moe_forward_static_check": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_int32)]),
    "mxfp4_moe_backward_input": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Weights),
                                                _vp, _sz, _vp, _vp, _sz, _vp, _vp, _vp, _vp]),
    "mxfp4_moe_grouped_matmul": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                ctypes.c_int32, _vp, _vp, _vp, _vp, ctypes.c_int32,
                                                _vp, _vp, _vp]),
    "mxfp4_moe_dequantize": (ctypes.c_int, [_vp, _vp, ctypes.c_int64, ctypes.c_int64, _vp, _vp]),
    "mxfp4_moe_residual_router": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                 _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_moe_grad_chain": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            _vp, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_moe_check": (ctypes.c_int, [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]),
    "mxfp4_moe_selftest_wait_timeout": (ctypes.c_int, [_vp, ctypes.c_size_t, _vp]),
    "mxfp4_moe_interleave_gate_up": (ctypes.c_int, [ctypes.POINTER(Dims), _vp, _vp, _vp, _vp, _vp,
                                                    _vp, _vp]),
    "mxfp4_moe_profile_begin": (ctypes.c_int, []),
    "mxfp4_moe_profile_end": (ctypes.c_int, [ctypes.POINTER(KernelTime), ctypes.c_int32,
                                             ctypes.POINTER(ctypes.c_int32)]),
    "mxfp4_moe_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "mxfp4_moe_build_flags": (ctypes.c_int, []),
}


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mxfp4_quantized_moe_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def strerror(code: int) -> str:
    return lib.mxfp4_moe_strerror(int(code)).decode()


def check(rc: int, what: str) -> None:
    if rc != OK:
        raise MoeError(rc, what)
