"""The residual stack of blocks on the GPU against the fp64 oracle.

Each block's output and input gradients are compared with the oracle block run on that
block's own inputs as the GPU saw them (x_l, logits_l and the upstream gradient g_{l+1}),
through the stack harness's forward and its recompute-per-block backward:

* a small stack (4 blocks, T=64, H=I=256, E=8, k=2) on every token;
* the full stack (24 gpt-oss-20b blocks, T=32768) on 16 sampled tokens, since each token's
  path through the stack is independent of the other tokens.

Between the blocks, the library's two caller-side kernels are checked on the same tokens:
x_{l+1} = bf16(x_l + y_l) bit for bit, the logits of every block against x_l W_r + b_r in
fp64, and each upstream gradient g_l against g_{l+1} + dX_l + d_logits_l W_r^T in fp64.

The stack output is not compared end to end with an fp64 chain: the caller rounds the
residual stream to bf16 after every block, and a difference at that rounding flips top-k
and clamp decisions downstream (an fp64 emulation of the bf16 stream alone drifts to cosine
0.9995 on x_L and 0.97 on dL/dx_0 after 4 small blocks).  The chaining itself (residual,
router path, recompute order) is checked against the fp64 oracle stack on the CPU.
"""

import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs, stack

import oracle_pool
from test_gpu_parity import _ws_offsets, assert_close, assert_d_logits_close
from test_gpu_residual import _check_logits

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().double().cpu().numpy()


def _run_blockwise(wl, seed, sel, workers=1):
    """Runs the stack on the GPU, records the blocks' inputs and results for tokens `sel`,
    then checks every block against the oracle."""
    from mxfp4_quantized_moe_b200 import moe
    shape, blocks, x, dy = stack.build_stack(wl, seed=seed)
    selc = torch.as_tensor(sel, dtype=torch.long, device=x.device)
    fw, bw = {}, {}

    def tap_f(l, d):
        fw[l] = {k: d[k][selc].cpu() for k in ("x", "logits", "y")}

    o = _ws_offsets(wl.T, wl.E, wl.k)
    nA = wl.T * wl.k

    def tap_b(l, d):
        bw[l] = {k: d[k][selc].cpu() for k in ("g", "dx", "d_logits", "d_w")}
        # the routing the block's backward used (its recomputed forward's, in the workspace)
        ws = st.ws
        bw[l]["idx"] = ws[o["idx"]:o["idx"] + 4 * nA].view(torch.int32).view(wl.T, wl.k)[selc].cpu()
        bw[l]["w"] = ws[o["w"]:o["w"] + 4 * nA].view(torch.float32).view(wl.T, wl.k)[selc].cpu()

    st = stack.MoeStack(shape, blocks)
    out, saved = st.forward(x, tap=tap_f)
    g0 = st.backward(dy, saved, tap=tap_b)
    torch.cuda.synchronize()
    w_r = [b.w_r.cpu() for b in blocks]
    b_r = [b.b_r.cpu() for b in blocks]
    g0_sel = g0[selc].cpu()
    rc, where = moe.device_check(st.ws)
    assert rc == 0, f"device error {rc} at {where:#x}"
    assert torch.isfinite(out.float()).all() and torch.isfinite(g0.float()).all()
    del st, blocks, saved, out, g0
    torch.cuda.empty_cache()

    jobs = [(wl, seed, l, _np(fw[l]["x"]), fw[l]["logits"].double().numpy(), _np(bw[l]["g"]))
            for l in range(wl.layers)]
    if workers > 1:
        # blocks are independent given their recorded inputs: fp64 oracle blocks in parallel
        # worker processes (spawned: no CUDA state is inherited)
        ctx = multiprocessing.get_context("spawn")
        with ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
            refs = list(ex.map(oracle_pool.block, jobs))
    else:
        refs = [oracle_pool.block(j) for j in jobs]
    # the caller-side kernels between the blocks
    for l in range(wl.layers):
        if l == 0:
            _check_logits(fw[0]["logits"], fw[0]["x"], w_r[0], b_r[0])
        if l + 1 < wl.layers:
            ref_x = (fw[l]["x"].float() + fw[l]["y"].float()).to(torch.bfloat16)
            assert torch.equal(fw[l + 1]["x"], ref_x), f"x[{l + 1}] is not bf16(x + y)"
            _check_logits(fw[l + 1]["logits"], fw[l + 1]["x"], w_r[l + 1], b_r[l + 1])
        # g_l, the upstream gradient of block l - 1 (of the stack input for l = 0)
        g_l = bw[l - 1]["g"] if l > 0 else g0_sel
        parts = [bw[l]["g"].double().numpy(), bw[l]["dx"].double().numpy(),
                 bw[l]["d_logits"].double().numpy() @ w_r[l].double().numpy().T]
        ref = sum(parts)
        scale = sum(np.abs(p) for p in parts[:2]) + \
            np.abs(bw[l]["d_logits"].double().numpy()) @ np.abs(w_r[l].double().numpy()).T
        err = np.abs(g_l.double().numpy() - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-5 * scale + 1e-30), f"g[{l}]"
    for l, (out, dX, d_w, d_logits, w, y_abs) in enumerate(refs):
        assert_close(_np(fw[l]["y"]), out, f"y[{l}]")
        assert_close(_np(bw[l]["dx"]), dX, f"dx[{l}]")
        gdw = _np(bw[l]["d_w"])
        assert_close(gdw, d_w, f"d_w[{l}]", np.float32)
        gdl = _np(bw[l]["d_logits"])
        # d_logits against the oracle, with the per-token floor of the bf16 rounding of y
        assert_d_logits_close(gdl, d_logits, w, d_w, f"d_logits[{l}]", y_abs=y_abs)
        # the softmax Jacobian itself, applied in fp64 to the GPU's own routing (its top-k
        # and weights, which a near tie in the logits can set apart from the oracle's) and d_w
        gi = bw[l]["idx"].numpy().astype(np.int64)
        gw = bw[l]["w"].double().numpy()
        sel = gw * (gdw - (gw * gdw).sum(axis=1, keepdims=True))
        jac = np.zeros_like(gdl)
        np.put_along_axis(jac, gi, sel, axis=1)
        assert_d_logits_close(gdl, jac, gw, gdw, f"d_logits[{l}] from the GPU's d_w")


def test_small_stack_blockwise_all_tokens():
    wl = inputs.Workload("stack4-T64-H256-E8-k2", 64, 256, 256, 8, 2, layers=4)
    _run_blockwise(wl, 3, np.arange(wl.T))


def test_stack24_full_size_blockwise_sampled_tokens():
    """16 seeded tokens through all 24 blocks; each block's oracle touches most of its 32
    experts, so the blocks are checked in parallel processes."""
    wl = inputs.WORKLOADS["gpt-oss-20b-moe-stack24-T32768"]
    sel = np.sort(np.random.default_rng(24).choice(wl.T, 16, replace=False))
    _run_blockwise(wl, 0, sel, workers=max(1, min(8, (os.cpu_count() or 2) // 2)))
