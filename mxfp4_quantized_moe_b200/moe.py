"""Torch-facing wrappers over the C ABI (device memory and streams come from torch).

Each function checks shapes and dtypes, hands raw device pointers and the current CUDA
stream to the library, and returns torch tensors.  All computation happens in the
library's kernels.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import Dims, Weights, check, lib


@dataclass
class MoeShape:
    T: int
    H: int
    I: int
    E: int
    k: int
    glu_alpha: float = 1.702
    glu_limit: float = 7.0
    # forward gate_up operands: 0 = bf16 (weights dequantized on the fly), 1 = block-scaled
    # (E2M1 weights as stored against E4M3 hi / lo token parts with UE8M0 block scales)
    gate_up_format: int = 0

    def dims(self) -> Dims:
        return Dims(self.T, self.H, self.I, self.E, self.k, self.glu_alpha, self.glu_limit,
                    self.gate_up_format)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _weights(w: dict) -> Weights:
    for key, dt in (("gu_blocks", torch.uint8), ("gu_scales", torch.uint8),
                    ("gu_bias", torch.bfloat16), ("dn_blocks", torch.uint8),
                    ("dn_scales", torch.uint8), ("dn_bias", torch.bfloat16)):
        if w[key].dtype != dt:
            raise TypeError(f"{key} must be {dt}")
    return Weights(_ptr(w["gu_blocks"]), _ptr(w["gu_scales"]), _ptr(w["gu_bias"]),
                   _ptr(w["dn_blocks"]), _ptr(w["dn_scales"]), _ptr(w["dn_bias"]))


def workspace_bytes(shape: MoeShape) -> int:
    n = ctypes.c_size_t()
    check(lib.mxfp4_moe_workspace_size(ctypes.byref(shape.dims()), ctypes.byref(n)),
          "mxfp4_moe_workspace_size")
    return n.value


def transposed_weights_bytes(shape: MoeShape) -> int:
    n = ctypes.c_size_t()
    check(lib.mxfp4_moe_transposed_weights_size(ctypes.byref(shape.dims()), ctypes.byref(n)),
          "mxfp4_moe_transposed_weights_size")
    return n.value


def alloc_workspace(shape: MoeShape, device="cuda") -> torch.Tensor:
    return torch.zeros(workspace_bytes(shape), dtype=torch.uint8, device=device)


def transpose_weights(shape: MoeShape, w: dict, out: torch.Tensor | None = None, stream=None):
    n = transposed_weights_bytes(shape)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=w["gu_blocks"].device)
    check(lib.mxfp4_moe_transpose_weights(ctypes.byref(shape.dims()), ctypes.byref(_weights(w)),
                                          _ptr(out), out.numel(), _stream(stream)),
          "mxfp4_moe_transpose_weights")
    return out


def forward(shape: MoeShape, w: dict, x: torch.Tensor, logits: torch.Tensor, ws: torch.Tensor,
            y: torch.Tensor | None = None, topk_idx: torch.Tensor | None = None,
            topk_w: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    T, H = shape.T, shape.H
    if x.shape != (T, H) or x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16 [T, H]")
    if logits.shape != (T, shape.E) or logits.dtype != torch.float32:
        raise ValueError("logits must be fp32 [T, E]")
    if y is None:
        y = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    check(lib.mxfp4_moe_forward(ctypes.byref(shape.dims()), ctypes.byref(_weights(w)), _ptr(x),
                                _ptr(logits), _ptr(y), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                ws.numel(), _stream(stream)), "mxfp4_moe_forward")
    return y


def backward_input(shape: MoeShape, w: dict, wt: torch.Tensor, dy: torch.Tensor,
                   ws: torch.Tensor, dx: torch.Tensor | None = None,
                   d_topk_w: torch.Tensor | None = None, d_logits: torch.Tensor | None = None,
                   want_d_logits: bool = True, stream=None):
    T, H = shape.T, shape.H
    if dy.shape != (T, H) or dy.dtype != torch.bfloat16:
        raise ValueError("dy must be bf16 [T, H]")
    dev = dy.device
    if dx is None:
        dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    if d_topk_w is None:
        d_topk_w = torch.empty(T, shape.k, dtype=torch.float32, device=dev)
    if d_logits is None and want_d_logits:
        d_logits = torch.empty(T, shape.E, dtype=torch.float32, device=dev)
    check(lib.mxfp4_moe_backward_input(ctypes.byref(shape.dims()), ctypes.byref(_weights(w)),
                                       _ptr(wt), wt.numel(), _ptr(dy), _ptr(ws), ws.numel(),
                                       _ptr(dx), _ptr(d_topk_w), _ptr(d_logits),
                                       _stream(stream)), "mxfp4_moe_backward_input")
    return dx, d_topk_w, d_logits


def dequantize(blocks: torch.Tensor, scales: torch.Tensor, stream=None,
               out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [rows, K] from packed uint8 [rows, K/2] and UE8M0 scales [rows, K/32]."""
    rows = blocks.numel() // blocks.shape[-1]
    K = blocks.shape[-1] * 2
    if scales.numel() != rows * (K // 32):
        raise ValueError("scales do not match blocks")
    if out is None:
        out = torch.empty(*blocks.shape[:-1], K, dtype=torch.bfloat16, device=blocks.device)
    elif out.numel() != rows * K or out.dtype != torch.bfloat16:
        raise ValueError("out must be bf16 with rows * K elements")
    check(lib.mxfp4_moe_dequantize(_ptr(blocks), _ptr(scales), rows, K, _ptr(out),
                                   _stream(stream)), "mxfp4_moe_dequantize")
    return out


def grouped_matmul(off: torch.Tensor, x: torch.Tensor, blocks: torch.Tensor,
                   scales: torch.Tensor, N: int, transposed: bool = False,
                   err: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[r] = x[r] W_e^T for the rows r of expert e (off: int32 [E+1] on the device)."""
    E = off.numel() - 1
    A, K = x.shape
    if x.dtype != torch.bfloat16 or off.dtype != torch.int32:
        raise TypeError("x must be bf16 and off int32")
    out = torch.empty(A, N, dtype=torch.bfloat16, device=x.device)
    check(lib.mxfp4_moe_grouped_matmul(E, N, K, A, _ptr(off), _ptr(x), _ptr(blocks),
                                       _ptr(scales), 1 if transposed else 0, _ptr(out),
                                       _ptr(err), _stream(stream)), "mxfp4_moe_grouped_matmul")
    return out


def device_check(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    """Synchronize and read (then clear) the device error word: (code, where)."""
    where = ctypes.c_int32(0)
    rc = lib.mxfp4_moe_check(_ptr(ws), _stream(stream), ctypes.byref(where))
    return rc, where.value


def interleave_gate_up(shape: MoeShape, blocks: torch.Tensor, scales: torch.Tensor,
                       bias: torch.Tensor, stream=None):
    """Stacked gate_up (rows [gates; ups]) -> interleaved (gate j at 2j, up j at 2j+1);
    returns new (blocks, scales, bias) tensors."""
    ob, os_, obias = torch.empty_like(blocks), torch.empty_like(scales), torch.empty_like(bias)
    check(lib.mxfp4_moe_interleave_gate_up(ctypes.byref(shape.dims()), _ptr(blocks), _ptr(scales),
                                           _ptr(bias), _ptr(ob), _ptr(os_), _ptr(obias),
                                           _stream(stream)), "mxfp4_moe_interleave_gate_up")
    return ob, os_, obias


def residual_router(x: torch.Tensor, y: torch.Tensor | None, w_r: torch.Tensor | None,
                    b_r: torch.Tensor | None = None, x_out: torch.Tensor | None = None,
                    logits: torch.Tensor | None = None, stream=None):
    """The residual stream between stacked blocks in one kernel: x_out = bf16(x + y) when y is
    given, and logits = (x_out or x) W_r + b_r in fp32 when w_r is given.  Returns
    (x_out or None, logits or None)."""
    T, H = x.shape
    if x.dtype != torch.bfloat16 or (y is not None and (y.shape != x.shape or y.dtype != x.dtype)):
        raise ValueError("x and y must be bf16 [T, H]")
    E = w_r.shape[1] if w_r is not None else 1
    if w_r is not None:
        if w_r.shape != (H, E) or w_r.dtype != torch.bfloat16:
            raise ValueError("w_r must be bf16 [H, E]")
        if b_r is not None and (b_r.shape != (E,) or b_r.dtype != torch.bfloat16):
            raise ValueError("b_r must be bf16 [E]")
        if logits is None:
            logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
    else:
        logits = None
    if y is not None and x_out is None:
        x_out = torch.empty_like(x)
    if y is None:
        x_out = None
    check(lib.mxfp4_moe_residual_router(T, H, E, _ptr(x), _ptr(y), _ptr(w_r), _ptr(b_r),
                                        _ptr(x_out), _ptr(logits), _stream(stream)),
          "mxfp4_moe_residual_router")
    return x_out, logits


def grad_chain(g: torch.Tensor, dx: torch.Tensor, d_logits: torch.Tensor, w_r: torch.Tensor,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16(g + dx + d_logits W_r^T) in fp32, one kernel (out may be g itself)."""
    T, H = g.shape
    E = w_r.shape[1]
    if g.dtype != torch.bfloat16 or dx.shape != g.shape or dx.dtype != g.dtype:
        raise ValueError("g and dx must be bf16 [T, H]")
    if d_logits.shape != (T, E) or d_logits.dtype != torch.float32:
        raise ValueError("d_logits must be fp32 [T, E]")
    if w_r.shape != (H, E) or w_r.dtype != torch.bfloat16:
        raise ValueError("w_r must be bf16 [H, E]")
    if out is None:
        out = torch.empty_like(g)
    check(lib.mxfp4_moe_grad_chain(T, H, E, _ptr(g), _ptr(dx), _ptr(d_logits), _ptr(w_r),
                                   _ptr(out), _stream(stream)), "mxfp4_moe_grad_chain")
    return out


def selftest_wait_timeout(ws: torch.Tensor, stream=None) -> None:
    """Enqueue the failure-detection self-test on `ws` (first 16 bytes zero); read the outcome
    with device_check(ws): (MXFP4_MOE_ERR_DEVICE_TIMEOUT, 0xF00) after about one second."""
    check(lib.mxfp4_moe_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(),
                                               _stream(stream)), "mxfp4_moe_selftest_wait_timeout")


def weights_to(inp: dict, device) -> dict:
    keys = ("gu_blocks", "gu_scales", "gu_bias", "dn_blocks", "dn_scales", "dn_bias")
    return {k: inp[k].to(device).contiguous() for k in keys}


def profile_begin() -> None:
    check(lib.mxfp4_moe_profile_begin(), "mxfp4_moe_profile_begin")


def profile_end() -> dict:
    """{kernel name: (launches, total device ms)} since profile_begin()."""
    buf = (_lib.KernelTime * 64)()
    n = ctypes.c_int32(0)
    check(lib.mxfp4_moe_profile_end(buf, 64, ctypes.byref(n)), "mxfp4_moe_profile_end")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n.value)}
