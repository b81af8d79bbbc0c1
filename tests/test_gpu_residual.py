"""The residual stream's kernels between stacked blocks, against their definitions in fp64.

mxfp4_moe_residual_router: x_out = bf16(x + y) (fp32 sum rounded once: bit-exact against
torch's bf16 addition, which rounds the fp32 sum the same way) and logits = xs W_r + b_r with
fp32 accumulation (within the fp32 accumulation bound of the exact sum).
mxfp4_moe_grad_chain: g_out = bf16(g + dx + d_logits W_r^T) (one bf16 rounding of the exact
value, plus fp32 accumulation).
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from mxfp4_quantized_moe_b200 import moe as m
    return m


def _draw(T, H, E, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(T, H, generator=g) * scale).to(torch.bfloat16)
    y = (torch.randn(T, H, generator=g) * scale).to(torch.bfloat16)
    w_r = (torch.randn(H, E, generator=g) * 0.02).to(torch.bfloat16)
    b_r = (torch.randn(E, generator=g) * 0.01).to(torch.bfloat16)
    return x, y, w_r, b_r


def _check_logits(got, xs, w_r, b_r):
    xs64, w64 = xs.double().numpy(), w_r.double().numpy()
    ref = xs64 @ w64 + (0.0 if b_r is None else b_r.double().numpy())
    bound = 2e-5 * (np.abs(xs64) @ np.abs(w64)) + 1e-7
    err = np.abs(got.double().cpu().numpy() - ref)
    assert np.all(err <= bound), float((err / bound).max())


SHAPES = [
    (100, 96, 8, 0),      # T not a multiple of the 64-token tile; H = 96: one and a half chunks
    (64, 2880, 32, 1),    # gpt-oss-20b widths
    (1, 32, 1, 2),        # a single token, one expert, half a chunk
    (130, 64, 100, 3),    # E = 100: a second pass over H for experts 64..99
    (77, 128, 256, 4),    # E = 256 (the maximum): four passes
]


@pytest.mark.parametrize("T,H,E,seed", SHAPES)
def test_residual_router(moe, T, H, E, seed):
    x, y, w_r, b_r = _draw(T, H, E, seed, scale=4.0)
    xc, yc, wc, bc = x.cuda(), y.cuda(), w_r.cuda(), b_r.cuda()
    x_out, logits = moe.residual_router(xc, yc, wc, bc)
    torch.cuda.synchronize()
    ref_x = (x.float() + y.float()).to(torch.bfloat16)
    assert torch.equal(x_out.cpu(), ref_x), "x_out is not bf16(x + y)"
    _check_logits(logits, ref_x, w_r, b_r)
    # logits of x itself (the stack's first block and the backward's recompute), no bias
    none_out, lg0 = moe.residual_router(xc, None, wc, None)
    assert none_out is None
    _check_logits(lg0, x, w_r, None)
    # the residual alone
    x2, lg2 = moe.residual_router(xc, yc, None)
    assert lg2 is None and torch.equal(x2.cpu(), ref_x)


@pytest.mark.parametrize("T,H,E,seed", SHAPES)
def test_grad_chain(moe, T, H, E, seed):
    g_, dx, w_r, _ = _draw(T, H, E, seed + 10)
    gen = torch.Generator().manual_seed(seed + 20)
    d_logits = torch.randn(T, E, generator=gen) * 3.0
    d_logits[0, : E // 2] = 0.0  # sparse rows like the router gradient's
    out = moe.grad_chain(g_.cuda(), dx.cuda(), d_logits.cuda(), w_r.cuda())
    torch.cuda.synchronize()
    g64, dx64, dl64, w64 = (t.double().numpy() for t in (g_, dx, d_logits, w_r))
    ref = g64 + dx64 + dl64 @ w64.T
    scale = np.abs(g64) + np.abs(dx64) + np.abs(dl64) @ np.abs(w64).T
    err = np.abs(out.double().cpu().numpy() - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-5 * scale + 1e-30)
    # in place on g
    gc = g_.cuda()
    moe.grad_chain(gc, dx.cuda(), d_logits.cuda(), w_r.cuda(), out=gc)
    torch.cuda.synchronize()
    assert torch.equal(gc.cpu(), out.cpu())
