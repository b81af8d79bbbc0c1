"""The forward for callers that cannot allocate (mxfp4_moe_forward_static).

Callers such as an inference-engine plugin that receives only input and output pointers, or a
serving loop that must not pay for cudaMalloc's implicit synchronization, run the forward with
the library's own fixed scratch array instead of a workspace.  These tests call that entry
point through the C ABI and compare it with the ordinary workspace forward on the same inputs,
on two calls in a row (the second call finds the first call's contents in the shared array).

This file is collected last on purpose, so that a run that stops at the first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REL_TOL = 2e-2
COS_TOL = 0.9999


def _close(got, ref, name):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), name
    err = float(np.max(np.abs(got - ref)))
    scale = float(np.max(np.abs(ref)))
    cos = float((got * ref).sum() / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    assert err <= REL_TOL * scale, f"{name}: max|err| {err:.3e} > {REL_TOL} * {scale:.3e}"
    assert cos >= COS_TOL, f"{name}: cosine {cos:.7f}"


def _static_forward(L, shape, w, x, logits, y, ti, tw):
    from mxfp4_quantized_moe_b200 import moe
    rc = L.lib.mxfp4_moe_forward_static(
        ctypes.byref(shape.dims()), ctypes.byref(moe._weights(w)), ctypes.c_void_p(x.data_ptr()),
        ctypes.c_void_p(logits.data_ptr()), ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(ti.data_ptr()), ctypes.c_void_p(tw.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc


@pytest.mark.parametrize("T,H,I,E,k", [(64, 256, 256, 8, 2), (200, 2880, 2880, 32, 4)])
def test_static_scratch_forward_matches_workspace_forward(T, H, I, E, k):
    from mxfp4_quantized_moe_b200 import _lib as L
    from mxfp4_quantized_moe_b200 import inputs, moe
    shape = moe.MoeShape(T, H, I, E, k)
    assert moe.workspace_bytes(shape) <= (64 << 20)  # fits the static scratch
    for call, seed in enumerate((21, 22)):  # two calls in a row, different inputs
        inp = inputs.make_layer(T, H, I, E, k, seed)
        w = moe.weights_to(inp, "cuda")
        x, lg = inp["x"].cuda(), inp["logits"].cuda()
        ws = moe.alloc_workspace(shape)
        ti_ref = torch.empty(T, k, dtype=torch.int32, device="cuda")
        tw_ref = torch.empty(T, k, dtype=torch.float32, device="cuda")
        y_ref = moe.forward(shape, w, x, lg, ws, topk_idx=ti_ref, topk_w=tw_ref)
        y = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        ti = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        tw = torch.zeros(T, k, dtype=torch.float32, device="cuda")
        assert _static_forward(L, shape, w, x, lg, y, ti, tw) == 0
        torch.cuda.synchronize()
        assert torch.equal(ti, ti_ref), f"call {call}: routing differs"
        np.testing.assert_allclose(tw.cpu().numpy(), tw_ref.cpu().numpy(), rtol=2e-6, atol=1e-7)
        _close(y.float().cpu().numpy(), y_ref.float().cpu().numpy(), f"call {call}: y")
        # the static array's error word: no device-side fault recorded
        where = ctypes.c_int32(-1)
        rc = L.lib.mxfp4_moe_forward_static_check(
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(where))
        assert (rc, where.value) == (0, 0), f"call {call}: device error {rc} at {where.value:#x}"


def test_static_scratch_rejects_problems_larger_than_the_array():
    from mxfp4_quantized_moe_b200 import _lib as L
    from mxfp4_quantized_moe_b200 import moe
    shape = moe.MoeShape(4096, 2880, 2880, 32, 4)  # needs ~480 MB of workspace
    assert moe.workspace_bytes(shape) > (64 << 20)
    d = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(d.data_ptr())
    w = L.Weights(p, p, p, p, p, p)
    rc = L.lib.mxfp4_moe_forward_static(ctypes.byref(shape.dims()), ctypes.byref(w), p, p, p,
                                        None, None, None)
    assert rc == L.ERR_WORKSPACE_TOO_SMALL
