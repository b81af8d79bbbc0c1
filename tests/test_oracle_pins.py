"""Pins for the fp64 oracle (CPU only).

Each test ties an oracle function to something other than itself: a hand-typed
table from the MX specification, a hand-derived worked example, a library
routine the oracle does not use, a closed form, brute force (the scalar twin),
finite differences, or an invariant.  The last group plants plausible mistakes
in a copy of the oracle and checks that the pins catch them.
"""

import math
import os

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs
from oracle import mxfp4_oracle as O
from oracle import scalar_twin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _tiny(T=4, H=64, I=64, E=4, k=2, seed=3, scale_lo=119, scale_hi=123):
    inp = inputs.make_layer(T, H, I, E, k, seed, scale_lo=scale_lo, scale_hi=scale_hi)
    return inp, inputs.as_numpy(inp)


# ---------------------------------------------------------------- MXFP4 decode -------
def test_e2m1_table_matches_mx_spec():
    rows = _rows("e2m1_codes.txt")
    assert len(rows) == 16
    for code, bits, val in rows:
        code = int(code)
        assert int(bits, 2) == code
        got = float(O.decode_e2m1(code))
        assert got == float(val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))  # -0.0 for code 8


def test_ue8m0_scales_match_mx_spec():
    for byte, val in _rows("ue8m0_scales.txt"):
        got = float(O.decode_ue8m0(int(byte)))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == 2.0 ** int(val.split("^")[1])


def test_dequant_worked_example():
    rows = {r[0]: r[1:] for r in _rows("dequant_worked_example.txt")}
    scales = np.array([[int(s) for s in rows["scales"]]], dtype=np.uint8)
    blocks = np.array([[int(b, 16) for b in rows["bytes"]]], dtype=np.uint8)
    want = np.array([float(v) for v in rows["values"]])
    got = O.dequantize(blocks, scales)[0]
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))


def test_dequant_matches_torch_float4_decode_exhaustive():
    """All 16 codes x all 256 scales against torch's own fp32->bf16 rounding of the
    exact fp32 value (an independent route to the same bf16 bits)."""
    codes = np.arange(16)
    s = np.arange(256)
    cc, ss = np.meshgrid(codes, s, indexing="ij")
    blocks = np.zeros((16 * 256, 16), np.uint8)
    scales = np.zeros((16 * 256, 1), np.uint8)
    blocks[:, 0] = cc.ravel()  # element 0 = low nibble
    scales[:, 0] = ss.ravel()
    val = O.dequantize(blocks, scales)[:, 0]
    bits = O.f64_to_bf16_bits(val)
    # independent: fp32 power-of-two arithmetic in torch, then torch's bf16 cast
    mag = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=torch.float64)
    tv = mag[torch.tensor(cc.ravel() & 7)] * torch.where(torch.tensor(cc.ravel() >= 8), -1.0, 1.0)
    tv = tv * torch.pow(torch.tensor(2.0, dtype=torch.float64), torch.tensor(ss.ravel() - 127.0))
    tb = tv.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    nan = ss.ravel() == 255
    assert np.array_equal(bits[~nan], tb[~nan])
    assert np.all(bits[nan] == 0x7FC0)


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormal range
        np.clip(rng.standard_normal(2000) * 1.5e38, -3.3e38, 3.3e38).astype(np.float32),  # near overflow
        np.array([0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.3895313892515355e38,
                  3.39e38, 2 ** -133, 2 ** -134, 1.5 * 2 ** -134], np.float32),
    ])
    got = O.f64_to_bf16_bits(x.astype(np.float64))
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(got, want)
    back = O.bf16_bits_to_f64(got)
    assert np.array_equal(back, torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).double().numpy())


# ---------------------------------------------------------------- routing -----------
def test_route_ties_go_to_lower_index_and_weights_are_softmax():
    logits = np.array([[1.0, 3.0, 3.0, 0.5], [2.0, 2.0, 2.0, 2.0]], np.float32)
    idx, w = O.route(logits, 2)
    assert idx.tolist() == [[1, 2], [0, 1]]
    assert np.allclose(w, 0.5)
    logits = np.array([[0.0, 1.0, -1.0]], np.float32)
    idx, w = O.route(logits, 2)
    assert idx.tolist() == [[1, 0]]
    assert w[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), abs=1e-15)  # sigmoid(l1 - l0)


def test_route_k1_is_argmax_with_weight_one():
    rng = np.random.default_rng(1)
    lg = rng.standard_normal((50, 7)).astype(np.float32)
    idx, w = O.route(lg, 1)
    assert np.array_equal(idx[:, 0], np.argmax(lg, axis=1))
    assert np.all(w == 1.0)


# ---------------------------------------------------------------- GLU ---------------
def test_glu_known_points_and_gelu_approximation():
    # u = -1 kills the output; g = 0 kills it too
    h = np.array([0.7, -1.0, 0.0, 3.0])
    assert np.all(O.glu(h) == 0.0)
    # g * sigmoid(1.702 g) is the sigmoid approximation of GELU = g * Phi(g); its
    # largest deviation on the real line is about 0.02 (at |g| near 2)
    g = np.linspace(-6, 6, 2001)
    hh = np.stack([g, np.zeros_like(g)], -1).reshape(-1)
    approx = O.glu(hh)
    gelu = np.array([v * 0.5 * (1 + math.erf(v / math.sqrt(2))) for v in g])
    assert np.max(np.abs(approx - gelu)) < 0.021
    # the clamp: g above the limit behaves as g = limit; u outside [-7, 7] saturates
    a = O.glu(np.array([9.0, 2.0, 7.0, 2.0, 1.0, 11.0, 1.0, 7.0, 1.0, -9.0, 1.0, -7.0]))
    assert a[0] == a[1] and a[2] == a[3] and a[4] == a[5]


def test_glu_backward_matches_finite_differences():
    rng = np.random.default_rng(2)
    h = rng.standard_normal(400) * 5
    # keep away from the clamp kinks
    h = np.where(np.abs(np.abs(h) - 7.0) < 1e-3, h + 0.01, h)
    dact = rng.standard_normal(200)
    dh = O.glu_backward(h, dact)
    eps = 1e-6
    for i in range(0, 400, 7):
        hp = h.copy(); hp[i] += eps
        hm = h.copy(); hm[i] -= eps
        j = i // 2  # only act[j] depends on h[i]
        fd = (O.glu(hp)[j] - O.glu(hm)[j]) * dact[j] / (2 * eps)
        assert fd == pytest.approx(dh[i], rel=1e-6, abs=1e-9)


def test_clamp_masks_are_decided_on_bf16_preactivations():
    # 7.01 rounds to bf16 7.0 (spacing 1/32 in [4, 8)): the gate clamp passes the gradient;
    # 7.02 rounds to 7.03125 and blocks it.  Same for u at -7.01 / -7.02.
    h = np.array([7.01, 1.0, 7.02, 1.0, 1.0, -7.01, 1.0, -7.02])
    dact = np.ones(4)
    hb = O.round_bf16(h)
    assert hb.tolist() == [7.0, 1.0, 7.03125, 1.0, 1.0, -7.0, 1.0, -7.03125]
    dh = O.glu_backward(h, dact, h_mask=hb)
    assert dh[0] != 0 and dh[2] == 0 and dh[5] != 0 and dh[7] == 0
    dh64 = O.glu_backward(h, dact)
    assert dh64[0] == 0 and dh64[5] == 0
    # away from the clamp the mask precision is irrelevant
    assert dh[1] == dh64[1] and dh[4] == dh64[4]


# ---------------------------------------------------------------- block -------------
def test_scalar_twin_matches_oracle_brute_force():
    inp, n = _tiny()
    f = O.moe_forward(n["x"], n["logits"], n["W"], 2)
    dX, dw, dl = O.moe_backward(n["dy"], f, n["W"])
    tw = scalar_twin.forward_backward(n["x"].tolist(), n["logits"].tolist(), n["dy"].tolist(),
                                      n["W"], 2)
    assert np.array_equal(f["idx"], np.array(tw["idx"]))
    np.testing.assert_allclose(f["w"], tw["w"], rtol=1e-13, atol=0)
    np.testing.assert_allclose(f["out"], tw["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dX, tw["dX"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, tw["d_w"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dl, tw["d_logits"], rtol=1e-10, atol=1e-12)


def _stacked_forward(x, logits, W, k):
    """Same block with gate_up stored stacked [gate; up] and a split-halves GLU."""
    E, I2, _ = W["gu_blocks"].shape
    I = I2 // 2
    perm = np.concatenate([np.arange(0, I2, 2), np.arange(1, I2, 2)])
    idx, w = O.route(logits, k)
    out = np.zeros_like(x)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        wgu = O.dequantize(W["gu_blocks"][e][perm], W["gu_scales"][e][perm])
        wd = O.dequantize(W["dn_blocks"][e], W["dn_scales"][e])
        h = x[tt] @ wgu.T + W["gu_bias"][e][perm]
        g, u = h[:, :I], h[:, I:]
        gc = np.minimum(g, 7.0)
        uc = np.clip(u, -7.0, 7.0)
        act = (uc + 1) * gc / (1 + np.exp(-1.702 * gc))
        y = act @ wd.T + W["dn_bias"][e]
        np.add.at(out, tt, w[tt, jj][:, None] * y)
    return out


def test_interleaved_equals_stacked_gate_up():
    inp, n = _tiny(T=16, E=4, k=2)
    f = O.moe_forward(n["x"], n["logits"], n["W"], 2)
    np.testing.assert_allclose(f["out"], _stacked_forward(n["x"], n["logits"], n["W"], 2),
                               rtol=1e-12, atol=1e-13)


def test_interleaving_twice_is_not_identity():
    # a converter that interleaves stacked rows, applied twice, is another permutation
    I2 = 16
    inter = np.empty(I2, int)
    inter[0::2] = np.arange(I2 // 2)
    inter[1::2] = np.arange(I2 // 2) + I2 // 2
    assert not np.array_equal(inter[inter], np.arange(I2))


def _dense_mixture(x, logits, W):
    E = logits.shape[1]
    lg = logits.astype(np.float64)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    out = np.zeros_like(x)
    for e in range(E):
        wgu = O.dequantize(W["gu_blocks"][e], W["gu_scales"][e])
        wd = O.dequantize(W["dn_blocks"][e], W["dn_scales"][e])
        y = O.glu(x @ wgu.T + W["gu_bias"][e]) @ wd.T + W["dn_bias"][e]
        out += p[:, e:e + 1] * y
    return out


def test_topk_equal_E_is_dense_softmax_mixture():
    inp, n = _tiny(T=12, E=4, k=4)
    f = O.moe_forward(n["x"], n["logits"], n["W"], 4)
    np.testing.assert_allclose(f["out"], _dense_mixture(n["x"], n["logits"], n["W"]),
                               rtol=1e-11, atol=1e-12)


def test_single_expert_is_plain_glu_mlp():
    inp, n = _tiny(T=5, E=1, k=1)
    W = n["W"]
    f = O.moe_forward(n["x"], n["logits"], W, 1)
    wgu = O.dequantize(W["gu_blocks"][0], W["gu_scales"][0])
    wd = O.dequantize(W["dn_blocks"][0], W["dn_scales"][0])
    g = n["x"] @ wgu[0::2].T + W["gu_bias"][0][0::2]
    u = n["x"] @ wgu[1::2].T + W["gu_bias"][0][1::2]
    g = np.minimum(g, 7); u = np.clip(u, -7, 7)
    want = ((u + 1) * g / (1 + np.exp(-1.702 * g))) @ wd.T + W["dn_bias"][0]
    np.testing.assert_allclose(f["out"], want, rtol=1e-12, atol=1e-13)


def test_zero_weights_give_routed_down_bias():
    inp, n = _tiny(T=6, E=4, k=2)
    W = dict(n["W"])
    W["gu_blocks"] = np.zeros_like(W["gu_blocks"])
    W["dn_blocks"] = np.zeros_like(W["dn_blocks"])
    f = O.moe_forward(n["x"], n["logits"], W, 2)
    want = np.einsum("tj,tjh->th", f["w"], W["dn_bias"][f["idx"]])
    np.testing.assert_allclose(f["out"], want, rtol=1e-13, atol=1e-15)


def test_token_permutation_equivariance_and_backward_linearity():
    inp, n = _tiny(T=10, E=4, k=2)
    f = O.moe_forward(n["x"], n["logits"], n["W"], 2)
    perm = np.random.default_rng(5).permutation(10)
    fp = O.moe_forward(n["x"][perm], n["logits"][perm], n["W"], 2)
    np.testing.assert_allclose(fp["out"], f["out"][perm], rtol=1e-13, atol=1e-14)
    a = O.moe_backward(n["dy"], f, n["W"])
    b = O.moe_backward(2.5 * n["dy"], f, n["W"])
    for u, v in zip(a, b):
        np.testing.assert_allclose(v, 2.5 * u, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(np.sum(f["w"], axis=1), 1.0, rtol=0, atol=1e-15)


def _loss(x, logits, W, dY, k):
    return float(np.sum(O.moe_forward(x, logits, W, k)["out"] * dY))


def test_backward_matches_finite_differences():
    inp, n = _tiny(T=4, H=64, I=64, E=4, k=2, seed=11)
    x, lg, W, dY = n["x"], n["logits"].astype(np.float64), n["W"], n["dy"]
    f = O.moe_forward(x, lg, W, 2)
    dX, dw, dl = O.moe_backward(dY, f, W)
    eps = 1e-6
    rng = np.random.default_rng(0)
    for _ in range(24):
        t, c = rng.integers(4), rng.integers(64)
        xp = x.copy(); xp[t, c] += eps
        xm = x.copy(); xm[t, c] -= eps
        fd = (_loss(xp, lg, W, dY, 2) - _loss(xm, lg, W, dY, 2)) / (2 * eps)
        assert fd == pytest.approx(dX[t, c], rel=1e-6, abs=1e-7)
    # logits: perturb only where the top-k set is stable under the perturbation
    srt = -np.sort(-lg, axis=1)
    for t in range(4):
        if srt[t, 1] - srt[t, 2] <= 10 * eps:
            continue
        for e in range(4):
            lp = lg.copy(); lp[t, e] += eps
            lm = lg.copy(); lm[t, e] -= eps
            fd = (_loss(x, lp, W, dY, 2) - _loss(x, lm, W, dY, 2)) / (2 * eps)
            assert fd == pytest.approx(dl[t, e], rel=1e-6, abs=1e-7)
    # routing weights: the loss is linear in w, so d_w is exact against a re-weighted combine
    y = f["y"]
    for t in range(4):
        for j in range(2):
            assert dw[t, j] == pytest.approx(float(np.dot(dY[t], y[t, j])), rel=1e-12)


# ---------------------------------------------------------------- planted mistakes ---
def _check_all_pins():
    test_dequant_worked_example()
    test_e2m1_table_matches_mx_spec()
    test_scalar_twin_matches_oracle_brute_force()
    test_backward_matches_finite_differences()
    test_interleaved_equals_stacked_gate_up()


@pytest.mark.parametrize("mistake", ["nibble_order", "exp_bias", "transposed_down",
                                     "dropped_bias", "glu_sign", "wrong_dact"])
def test_pins_catch_planted_mistakes(monkeypatch, mistake):
    if mistake == "nibble_order":
        orig = O.dequantize

        def bad(blocks, scales):
            b = np.asarray(blocks, np.uint8)
            return orig(((b & 0x0F) << 4) | (b >> 4), scales)
        monkeypatch.setattr(O, "dequantize", bad)
    elif mistake == "exp_bias":
        monkeypatch.setattr(O, "decode_ue8m0", lambda s: np.ldexp(1.0, np.asarray(s, np.int64) - 128))
    elif mistake == "transposed_down":
        def bad_w(W, e):
            wgu = O.dequantize(W["gu_blocks"][e], W["gu_scales"][e])
            wd = O.dequantize(W["dn_blocks"][e], W["dn_scales"][e])
            return wgu, wd.T.copy() if wd.shape[0] == wd.shape[1] else wd
        monkeypatch.setattr(O, "_expert_weights", bad_w)
    elif mistake == "dropped_bias":
        orig_fwd = O.moe_forward

        def bad_fwd(x, logits, W, k, alpha=1.702, limit=7.0):
            W2 = dict(W); W2["gu_bias"] = np.zeros_like(W["gu_bias"])
            return orig_fwd(x, logits, W2, k, alpha, limit)
        monkeypatch.setattr(O, "moe_forward", bad_fwd)
    elif mistake == "glu_sign":
        monkeypatch.setattr(O, "_sigmoid", lambda z: 1.0 / (1.0 + np.exp(z)))
    elif mistake == "wrong_dact":
        orig_b = O.glu_backward
        monkeypatch.setattr(O, "glu_backward",
                            lambda h, d, a=1.702, l=7.0, **kw: orig_b(h, d, a, l, **kw)[..., ::-1])
    with pytest.raises(AssertionError):
        _check_all_pins()


# ---------------------------------------------------------------- shapes at random ---
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=12, deadline=None)
@given(T=st.integers(1, 5), H=st.sampled_from([32, 64, 96]), I=st.sampled_from([32, 64]),
       E=st.integers(1, 5), kk=st.integers(1, 5), seed=st.integers(0, 10_000))
def test_oracle_matches_scalar_twin_on_random_shapes(T, H, I, E, kk, seed):
    """The vectorised oracle and the scalar twin agree for shapes other than the fixed pins
    (H != I, one expert, k = E, single tokens): catches a transposed or mis-sliced operand that
    happens to be invisible at square shapes."""
    k = min(kk, E)
    inp = inputs.make_layer(T, H, I, E, k, seed)
    n = inputs.as_numpy(inp)
    f = O.moe_forward(n["x"], n["logits"], n["W"], k)
    dX, dw, dl = O.moe_backward(n["dy"], f, n["W"])
    tw = scalar_twin.forward_backward(n["x"].tolist(), n["logits"].tolist(), n["dy"].tolist(),
                                      n["W"], k)
    assert np.array_equal(f["idx"], np.array(tw["idx"]))
    np.testing.assert_allclose(f["out"], tw["out"], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dX, tw["dX"], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dw, tw["d_w"], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dl, tw["d_logits"], rtol=1e-9, atol=1e-11)


# ---------------------------------------------------------------- E4M3 split -----------
def test_round_e4m3_matches_torch_float8_exhaustively():
    """Every bf16 value of magnitude up to 448 rounds to E4M3 exactly as torch's own cast."""
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    v = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float()
    keep = torch.isfinite(v) & (v.abs() <= 448.0)
    v = v[keep]
    ref = v.to(torch.float8_e4m3fn).float().double().numpy()
    got = O.round_e4m3(v.double().numpy())
    assert np.array_equal(got, ref)
    assert np.isnan(O.round_e4m3(np.array([470.0, -1e6]))).all()


def test_mx_split_is_exact_near_the_block_maximum_and_bounded_below_it():
    rng = np.random.default_rng(4)
    x = torch.from_numpy(rng.standard_normal((256, 64)) * np.exp(rng.uniform(-8, 8, (256, 1))))
    x = x.to(torch.bfloat16).double().numpy()  # bf16 activations
    hi, lo, S = O.mx_split(x)
    xb, hb, lb = x.reshape(-1, 32), hi.reshape(-1, 32), lo.reshape(-1, 32)
    y = np.ldexp(xb, -S[:, None])
    amax = np.abs(y).max(axis=1)
    assert np.all((amax > 224.0) & (amax <= 448.0))            # the smallest fitting scale
    resid = np.abs(y - hb - lb)
    near = np.abs(y) >= amax[:, None] * 2.0 ** -9               # within 2^9 of the maximum
    assert np.all(resid[near] == 0.0)
    assert np.all(resid <= 2.0 ** -10)                          # half the subnormal spacing
    assert near.mean() > 0.95
