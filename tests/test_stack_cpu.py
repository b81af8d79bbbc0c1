"""The residual stack of blocks on the CPU (no GPU).

* The oracle's fp64 stack is pinned by central finite differences of its own forward: the
  gradient of <dY, x_L> with respect to x_0 must match `stack_backward`, which exercises the
  residual path, the block's input gradient and the router path d_logits W_r^T together.
  A planted mistake (the router path dropped) must fail that pin.
* The stack harness (router linear, residual add, gradient chaining, recompute order) is
  run on float64 tensors with blocks backed by the oracle and must reproduce the oracle's
  stack to rounding.
"""

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs
from mxfp4_quantized_moe_b200.stack import MoeStack, StackBlock
from oracle import mxfp4_oracle as O

T, H, I, E, K, L = 3, 64, 64, 4, 2, 3


def _stack(seed=21):
    layers, x, dy = [], None, None
    for l in range(L):
        inp = inputs.make_layer(T, H, I, E, K, seed + l, with_dy=(l == 0))
        n = inputs.as_numpy(inp)
        if l == 0:
            x, dy = n["x"], n["dy"]
        layers.append({"W": n["W"], "w_r": inp["w_r"].double().numpy(),
                       "b_r": inp["b_r"].double().numpy()})
    return layers, x, dy


def _loss(x0, layers, dY):
    out, _ = O.stack_forward(x0, layers, K)
    return float((out * dY).sum())


def _check_fd(layers, x, dY):
    out, recs = O.stack_forward(x, layers, K)
    g0, _ = O.stack_backward(dY, recs, layers)
    # preconditions for central differences: no top-k set within reach of the step, no
    # clamp kink (g or |u| at the limit) within reach of the step
    for r in recs:
        srt = -np.sort(-r["logits"], axis=1)
        assert np.all(srt[:, K - 1] - srt[:, K] > 1e-4)
        h = r["fwd"]["h"]
        assert np.all(np.abs(np.abs(h) - 7.0) > 0.05)
    eps = 1e-6
    rng = np.random.default_rng(1)
    for _ in range(16):
        t, c = rng.integers(T), rng.integers(H)
        xp = x.copy(); xp[t, c] += eps
        xm = x.copy(); xm[t, c] -= eps
        fd = (_loss(xp, layers, dY) - _loss(xm, layers, dY)) / (2 * eps)
        assert fd == pytest.approx(g0[t, c], rel=1e-6, abs=1e-6)


def test_oracle_stack_gradient_matches_finite_differences():
    layers, x, dy = _stack()
    _check_fd(layers, x, dy)


def test_stack_pin_catches_a_dropped_router_path(monkeypatch):
    layers, x, dy = _stack()
    orig = O.moe_backward

    def no_router(dY, fwd, W, alpha=1.702, limit=7.0):
        dX, d_w, d_logits = orig(dY, fwd, W, alpha, limit)
        return dX, d_w, np.zeros_like(d_logits)
    monkeypatch.setattr(O, "moe_backward", no_router)
    with pytest.raises(AssertionError):
        _check_fd(layers, x, dy)


def test_harness_chaining_matches_oracle_stack():
    layers, x, dy = _stack()
    fwd_of = {}
    calls = []

    def block_forward(l, xt, logits):
        calls.append(("f", l))
        f = O.moe_forward(xt.numpy(), logits.numpy(), layers[l]["W"], K)
        fwd_of[l] = f  # the block's saved state, refilled by every (re)computed forward
        return torch.from_numpy(f["out"])

    def block_backward(l, g):
        calls.append(("b", l))
        dX, d_w, d_logits = O.moe_backward(g.numpy(), fwd_of[l], layers[l]["W"])
        return torch.from_numpy(dX), torch.from_numpy(d_logits), torch.from_numpy(d_w)

    blocks = [StackBlock(None, None, torch.from_numpy(ly["w_r"]), torch.from_numpy(ly["b_r"]))
              for ly in layers]
    def residual_router(xt, y, w_r, b_r):  # the caller-side steps by definition, in fp64
        x_next = None if y is None else xt + y
        xs = xt if y is None else x_next
        return x_next, (None if w_r is None else xs @ w_r + b_r)

    def grad_chain(g, dx, d_logits, w_r):
        return g + dx + d_logits @ w_r.T

    st = MoeStack(None, blocks, block_forward=block_forward, block_backward=block_backward,
                  residual_router=residual_router, grad_chain=grad_chain)
    xt = torch.from_numpy(x.copy())
    out, saved = st.forward(xt)
    calls_fwd = list(calls)
    g0 = st.backward(torch.from_numpy(dy.copy()), saved)

    ref_out, recs = O.stack_forward(x, layers, K)
    ref_g0, _ = O.stack_backward(dy, recs, layers)
    np.testing.assert_allclose(out.numpy(), ref_out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g0.numpy(), ref_g0, rtol=1e-11, atol=1e-11)
    # the forward keeps only block inputs; the backward recomputes each block just before
    # its backward, from the last block down
    assert calls_fwd == [("f", l) for l in range(L)]
    assert calls[L:] == [c for l in reversed(range(L)) for c in (("f", l), ("b", l))]
    assert len(saved) == L and all(s[0].shape == (T, H) and s[1].shape == (T, E)
                                   for s in saved)
