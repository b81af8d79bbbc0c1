"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bar: dequantized weights and top-k indices bit-exact; y, dX, d(routing weights) and
d(logits) within max|err| <= 2e-2 * max|ref| per tensor with cosine >= 0.9999.
The oracle and the CUDA path consume the same seeded inputs (the same fp32 logits), so
routing must agree exactly.
"""

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs
from oracle import mxfp4_oracle as O

pytestmark = pytest.mark.gpu

REL_TOL = 2e-2
COS_TOL = 0.9999


@pytest.fixture(scope="module")
def moe():
    from mxfp4_quantized_moe_b200 import moe as m
    return m


def assert_close(got, ref, name, out_dtype=None):
    """`out_dtype` is the precision of the GPU output; the fp64 reference is rounded to it
    first (fp32 routing gradients: a reference far below fp32's range is zero there)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if out_dtype is not None:
        ref = ref.astype(out_dtype).astype(np.float64)
    assert got.shape == ref.shape, name
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = float(np.max(np.abs(got - ref)))
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:  # degenerate case (e.g. d_logits with k == 1): must be exactly zero
        assert err == 0.0, f"{name}: expected all zeros, max|got| {err:.3e}"
        return
    cos = float((got * ref).sum() / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    assert err <= REL_TOL * scale, f"{name}: max|err| {err:.3e} > {REL_TOL} * {scale:.3e}"
    assert cos >= COS_TOL, f"{name}: cosine {cos:.7f}"


def assert_d_logits_close(got, ref, w, d_w, name="d_logits", require_resolved=False, y_abs=None):
    """d_logits[t, idx_j] = w_j (d_w_j - sum_i w_i d_w_i) cancels when routing is nearly
    one-hot: the fp32 router backward cannot resolve it below about 2^-23 max|w * d_w| per
    token, while the fp64 oracle does.  So the reference (rounded to fp32, the output's
    precision) is compared with an absolute floor of 2^-20 max|w * d_w| per token (8x the
    fp32 resolution of the k-term sum); above the floor this is the usual per-tensor bar.

    With `y_abs` (sum_h |dY_h| |y_{j,h}| per token and slot) the floor also covers the bf16
    rounding of the expert outputs y that d_w = <dY, y_j> is taken on: each d_w_j is then off
    by up to 2^-9 y_abs_j (plus the fp32 sum), and the Jacobian can pass twice that on, so the
    floor is 2^-7 max_j w_j max_i y_abs_i per token."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64).astype(np.float32).astype(np.float64)
    floor = 2.0 ** -20 * np.max(np.abs(np.asarray(w, np.float64) * np.asarray(d_w, np.float64)),
                                axis=1, keepdims=True)
    margin = 1.0
    if y_abs is not None:
        wmax = np.max(np.asarray(w, np.float64), axis=1, keepdims=True)
        floor = np.maximum(floor, 2.0 ** -7 * wmax * np.max(y_abs, axis=1, keepdims=True))
        margin = 64.0  # the per-tensor bar only for tokens resolved well above their floor
    resolved = np.abs(ref).max(axis=1, keepdims=True) > margin * floor
    if require_resolved:
        assert resolved.all(), f"{name}: a token's reference lies below the fp32 floor"
    # tokens whose d_logits lies below the fp32 floor: absolute bound only
    assert np.all(np.abs(got - ref)[~resolved[:, 0]] <= floor[~resolved[:, 0]]), \
        f"{name}: unresolved tokens off by more than the fp32 floor"
    if resolved.any():
        assert_close(got[resolved[:, 0]], ref[resolved[:, 0]], name)


def run_block(moe, T, H, I, E, k, seed, tokens=None, gate_up_format=0, **kw):
    inp = inputs.make_layer(T, H, I, E, k, seed, **kw)
    shape = moe.MoeShape(T, H, I, E, k, gate_up_format=gate_up_format)
    w = moe.weights_to(inp, "cuda")
    x, lg, dy = inp["x"].cuda(), inp["logits"].cuda(), inp["dy"].cuda()
    ws = moe.alloc_workspace(shape)
    wt = moe.transpose_weights(shape, w)
    ti = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    y = moe.forward(shape, w, x, lg, ws, topk_idx=ti, topk_w=tw)
    dx, dtw, dl = moe.backward_input(shape, w, wt, dy, ws)
    rc, where = moe.device_check(ws)
    assert rc == 0, f"device error {rc} at {where:#x}"
    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    n = inputs.as_numpy(inp, sel)
    n["W"]["_dequant_cache"] = {}  # each touched expert dequantized once for fwd and bwd
    f = O.moe_forward(n["x"], n["logits"], n["W"], k)
    dX, dW, dL = O.moe_backward(n["dy"], f, n["W"])
    got = {
        "idx": ti.cpu().numpy()[sel], "w": tw.cpu().numpy()[sel], "y": y.float().cpu().numpy()[sel],
        "dx": dx.float().cpu().numpy()[sel], "d_w": dtw.cpu().numpy()[sel],
        "d_logits": dl.cpu().numpy()[sel],
    }
    ref = {"idx": f["idx"], "w": f["w"], "y": f["out"], "dx": dX, "d_w": dW, "d_logits": dL}
    return got, ref


def check_all(got, ref):
    assert np.array_equal(got["idx"], ref["idx"]), "top-k indices differ"
    np.testing.assert_allclose(got["w"], ref["w"], rtol=2e-6, atol=1e-7)
    for name in ("y", "dx"):
        assert_close(got[name], ref[name], name)
    assert_close(got["d_w"], ref["d_w"], "d_w", np.float32)
    # single layers route well away from one-hot: every token must clear the floor (k >= 2)
    assert_d_logits_close(got["d_logits"], ref["d_logits"], ref["w"], ref["d_w"],
                          require_resolved=ref["w"].shape[1] >= 2)


# ------------------------------------------------------------------ dequant -----------
def test_dequant_bit_exact_all_codes_and_scales(moe):
    rng = np.random.default_rng(0)
    codes = np.arange(16)
    s = np.arange(256)
    cc, ss = np.meshgrid(codes, s, indexing="ij")
    blocks = rng.integers(0, 256, (16 * 256, 32), dtype=np.uint8)
    blocks[:, 0] = cc.ravel() | (np.roll(cc.ravel(), 5) << 4)
    scales = np.stack([ss.ravel(), rng.integers(0, 256, 16 * 256)], 1).astype(np.uint8)
    out = moe.dequantize(torch.from_numpy(blocks).cuda(), torch.from_numpy(scales).cuda())
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = O.f64_to_bf16_bits(O.dequantize(blocks, scales))
    assert np.array_equal(got, ref)


def test_dequant_gpt_oss_rows_bit_exact(moe):
    inp = inputs.make_layer(4, 2880, 2880, 2, 1, seed=9)
    b, s = inp["gu_blocks"][1], inp["gu_scales"][1]
    out = moe.dequantize(b.cuda(), s.cuda())
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.f64_to_bf16_bits(O.dequantize(b.numpy(), s.numpy())))


def test_transposed_weights_are_a_pure_transpose(moe):
    T, H, I, E, k = 8, 96, 160, 3, 2
    inp = inputs.make_layer(T, H, I, E, k, seed=2)
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    wt = moe.transpose_weights(shape, w).cpu().numpy()

    def unpack(b):
        return np.stack([b & 15, b >> 4], -1).reshape(*b.shape[:-1], b.shape[-1] * 2)

    def region(off, n):
        start = (off + 255) // 256 * 256
        return wt[start:start + n], start + n

    o = 0
    dn_t, o = region(o, E * I * H // 2)
    gu_t, o = region(o, E * H * I)
    dn_s, o = region(o, E * (I // 32) * H)
    gu_s, o = region(o, E * (H // 32) * 2 * I)
    dn = unpack(inp["dn_blocks"].numpy())  # [E][H][I]
    gu = unpack(inp["gu_blocks"].numpy())  # [E][2I][H]
    assert np.array_equal(unpack(dn_t.reshape(E, I, H // 2)), dn.transpose(0, 2, 1))
    assert np.array_equal(unpack(gu_t.reshape(E, H, I)), gu.transpose(0, 2, 1))
    assert np.array_equal(dn_s.reshape(E, I // 32, H), inp["dn_scales"].numpy().transpose(0, 2, 1))
    assert np.array_equal(gu_s.reshape(E, H // 32, 2 * I), inp["gu_scales"].numpy().transpose(0, 2, 1))


# ------------------------------------------------------------------ routing -----------
def test_router_ties_and_topk_exact(moe):
    T, H, I, E, k = 96, 64, 64, 8, 3
    inp = inputs.make_layer(T, H, I, E, k, seed=3)
    lg = inp["logits"].clone()
    lg[0] = 1.0  # all equal: experts 0, 1, 2
    lg[1, 5] = lg[1, 2] = lg[1].max() + 1  # tie at the top: 2 before 5
    lg[2] = torch.arange(E, dtype=torch.float32)  # strictly increasing: 7, 6, 5
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    ws = moe.alloc_workspace(shape)
    ti = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.forward(shape, w, inp["x"].cuda(), lg.cuda(), ws, topk_idx=ti, topk_w=tw)
    idx, wr = O.route(lg.numpy(), k)
    got = ti.cpu().numpy()
    assert got[0].tolist() == [0, 1, 2] and got[1, :2].tolist() == [2, 5]
    assert got[2].tolist() == [7, 6, 5]
    assert np.array_equal(got, idx)
    np.testing.assert_allclose(tw.cpu().numpy(), wr, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("E,k", [(256, 40), (128, 4), (40, 33)])
def test_router_signed_zeros_infinities_and_wide_k(moe, E, k):
    """Top-k against the oracle's stable sort where the ranking is delicate: +0 and -0 tie (the
    lower expert wins), -inf logits rank last, negative logits, every group of 32 experts of a
    lane occupied (E = 256), and more than 32 selections per token (k = 40 and 33)."""
    T, H, I = 64, 64, 64
    inp = inputs.make_layer(T, H, I, E, k, seed=21)
    lg = inp["logits"].clone()
    lg[0] = 0.0
    lg[0, 1::2] = -0.0                                   # +0 / -0 alternate: all tie
    lg[1] = -torch.arange(E, dtype=torch.float32)       # strictly decreasing from 0
    lg[1, 3] = -0.0                                      # -0 ties with expert 0's +0
    lg[2] = float("-inf")
    lg[2, E - 1] = -1e30                                 # one finite logit, then -inf ties
    lg[3, ::3] = float("-inf")
    lg[4] = torch.where(torch.arange(E) % 5 == 0, 2.5, -2.5)  # five-way groups of ties
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    ws = moe.alloc_workspace(shape)
    ti = torch.empty(T, k, dtype=torch.int32, device="cuda")
    tw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.forward(shape, w, inp["x"].cuda(), lg.cuda(), ws, topk_idx=ti, topk_w=tw)
    assert moe.device_check(ws) == (0, 0)
    idx, wr = O.route(lg.numpy(), k)
    assert np.array_equal(ti.cpu().numpy(), idx)
    np.testing.assert_allclose(tw.cpu().numpy(), wr, rtol=2e-6, atol=1e-7)


# ------------------------------------------------------------------ whole block -------
def test_tiny_workload_full_parity(moe):
    wl = inputs.WORKLOADS["tiny-moe-T64-H256-E8-k2"]
    got, ref = run_block(moe, wl.T, wl.H, wl.I, wl.E, wl.k, seed=0)
    check_all(got, ref)


@pytest.mark.parametrize("T,H,I,E,k,seed,kw", [
    (1, 64, 64, 4, 2, 1, {}),                                  # a single token
    (37, 96, 160, 5, 3, 4, {}),                                # K tails (96, 160, 320), ragged tiles
    (5, 64, 64, 16, 1, 5, {}),                                 # most experts empty
    (200, 128, 64, 4, 4, 6, {"scale_lo": 110, "scale_hi": 140}),  # k == E; scales above 2^1
    (450, 64, 96, 2, 1, 7, {}),                                # several token tiles per expert
    (130, 2880, 2880, 4, 2, 8, {}),                            # gpt-oss widths, few tokens
    (96, 64, 64, 256, 8, 9, {}),                               # E = 256 (the maximum), mostly empty
    (24, 64, 96, 32, 20, 10, {}),                              # k = 20 > 16 selected per token
    (40, 32, 32, 4, 2, 11, {}),                                # H = I = 32: half a k-step
    (33, 32, 96, 3, 2, 12, {}),                                # H = 32 forward, K = 192 back
])
def test_edge_cases(moe, T, H, I, E, k, seed, kw):
    got, ref = run_block(moe, T, H, I, E, k, seed, **kw)
    check_all(got, ref)


@pytest.mark.parametrize("T,H,I,E,k,seed,tokens", [
    (64, 256, 256, 8, 2, 0, None),        # the tiny workload, every token
    (37, 96, 160, 5, 3, 4, None),         # K tails, ragged tiles
    (300, 2880, 2880, 32, 4, 13, None),   # gpt-oss-20b widths, every token
])
def test_block_scaled_gate_up_parity(moe, T, H, I, E, k, seed, tokens):
    """The forward with the block-scaled gate_up (E2M1 weights as stored against the E4M3
    hi / lo split of the token rows): the whole block against the oracle, like the bf16 form."""
    got, ref = run_block(moe, T, H, I, E, k, seed, tokens=tokens, gate_up_format=1)
    check_all(got, ref)


@pytest.mark.parametrize("T", [1, 64, 256])
def test_small_token_gpt_oss_20b_every_token(moe, T):
    """The small-token (decode-sized) batches of the gpt-oss-20b layer (H=I=2880, E=32, k=4),
    every token checked: a handful of rows per expert, most experts with a single token tile
    far below the tile height."""
    got, ref = run_block(moe, T, 2880, 2880, 32, 4, seed=40 + T)
    check_all(got, ref)


def test_small_token_skewed_gpt_oss_20b_every_token(moe):
    """T=512 with Zipf-skewed routing at gpt-oss-20b widths, every token: hot experts with
    several hundred rows (two or more token tiles) beside cold ones holding a few rows."""
    got, ref = run_block(moe, 512, 2880, 2880, 32, 4, seed=41, zipf_s=1.2)
    check_all(got, ref)


def test_expert_gradient_is_not_silent(moe):
    """The pages' silent-gradient trap: dX must carry the expert path (not be zero)."""
    got, ref = run_block(moe, 16, 64, 64, 4, 2, seed=12)
    assert np.abs(got["dx"]).max() > 0.1 * np.abs(ref["dx"]).max() > 0
    check_all(got, ref)


def tile_boundary_tokens(logits, k, cap, seed, tile_rows=256):
    """Tokens whose assignments sit on the first or last row of a grouped-GEMM token tile.

    The GEMMs cut each expert's m expert-sorted rows into ceil(m / tile_rows) equal tiles of
    a multiple of 16 rows (the last one possibly shorter); the rows at those cuts are where a
    tile's TMA box starts or ends.  Returns at most `cap` of those tokens (seeded choice)."""
    idx = O.route(np.asarray(logits, np.float64), k)[0].reshape(-1)
    E = int(np.asarray(logits).shape[1])
    hist = np.bincount(idx, minlength=E)
    off = np.concatenate([[0], np.cumsum(hist)])
    perm = np.argsort(idx, kind="stable")  # sorted row -> slot
    rows = []
    for e in range(E):
        m = int(hist[e])
        if m == 0:
            continue
        n = -(-m // tile_rows)
        per = -(-m // n)
        per = (per + 15) // 16 * 16
        for start in range(0, m, per):
            rows += [off[e] + start, off[e] + min(start + per, m) - 1]
    toks = np.unique(perm[np.asarray(rows)] // k)
    if toks.size > cap:
        toks = np.sort(np.random.default_rng(seed).choice(toks, cap, replace=False))
    return toks


def test_gpt_oss_20b_full_size_sampled_tokens(moe):
    """The benchmarked launch configuration (T=8192, H=I=2880, E=32, k=4), checked on 1024
    seeded random tokens plus tokens whose rows sit on token-tile boundaries: every token is
    independent, so the oracle runs on the sample only.  Every token's output spans all 2880
    features, the last 128-feature block (rows 2816..2879 of the weights) half full."""
    wl = inputs.WORKLOADS["gpt-oss-20b-moe-T8192"]
    lg = inputs.make_workload(wl, 0, with_dy=False)["logits"].numpy()
    rnd = np.random.default_rng(0).choice(wl.T, 1024, replace=False)
    sel = np.union1d(rnd, tile_boundary_tokens(lg, wl.k, 256, 0))
    got, ref = run_block(moe, wl.T, wl.H, wl.I, wl.E, wl.k, seed=0, tokens=sel)
    check_all(got, ref)


def test_zipf_skew_full_size_sampled_tokens(moe):
    """Skewed routing at T=16384 (hottest expert ~25% of assignments, eight experts under 16
    rows): 256 seeded tokens, one token of each of the four coldest experts and tokens on
    token-tile boundaries."""
    wl = inputs.WORKLOADS["gpt-oss-20b-moe-zipf-T16384"]
    lg = inputs.make_workload(wl, 0, with_dy=False)["logits"]
    idx = torch.topk(lg, wl.k, dim=1).indices
    cold = torch.bincount(idx.flatten(), minlength=wl.E).argsort()[:4]
    extra = [int((idx == e).any(dim=1).nonzero()[0]) for e in cold.tolist()]
    rnd = np.random.default_rng(1).choice(wl.T, 256, replace=False).tolist()
    sel = np.unique(np.concatenate([np.asarray(rnd + extra),
                                    tile_boundary_tokens(lg.numpy(), wl.k, 64, 1)]))
    got, ref = run_block(moe, wl.T, wl.H, wl.I, wl.E, wl.k, seed=0, tokens=sel, zipf_s=wl.zipf_s)
    check_all(got, ref)


def test_gpt_oss_120b_full_size_sampled_tokens(moe):
    """128 experts of ~512 rows (T=16384): many small expert groups, 1.69 GB of packed
    weights streamed per pass; 256 seeded tokens plus token-tile boundaries."""
    wl = inputs.WORKLOADS["gpt-oss-120b-moe-T16384"]
    lg = inputs.make_workload(wl, 0, with_dy=False)["logits"].numpy()
    rnd = np.random.default_rng(2).choice(wl.T, 256, replace=False)
    sel = np.union1d(rnd, tile_boundary_tokens(lg, wl.k, 64, 2))
    got, ref = run_block(moe, wl.T, wl.H, wl.I, wl.E, wl.k, seed=0, tokens=sel)
    check_all(got, ref)


def test_run_to_run_deterministic(moe):
    T, H, I, E, k = 300, 256, 256, 8, 2
    inp = inputs.make_layer(T, H, I, E, k, 13)
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    wt = moe.transpose_weights(shape, w)
    outs = []
    for _ in range(2):
        ws = moe.alloc_workspace(shape)
        y = moe.forward(shape, w, inp["x"].cuda(), inp["logits"].cuda(), ws)
        dx, dtw, dl = moe.backward_input(shape, w, wt, inp["dy"].cuda(), ws)
        outs.append([t.clone() for t in (y, dx, dtw, dl)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_interleave_helper_restores_the_shipped_row_order(moe):
    """Layout helper: a stacked checkpoint ([gates; ups]) converts to exactly the interleaved
    tensors the block expects (bytes, scales and bias copied unchanged)."""
    T, H, I, E, k = 16, 256, 288, 3, 2
    inp = inputs.make_layer(T, H, I, E, k, 17)

    def stacked(t):
        return torch.cat([t[:, 0::2], t[:, 1::2]], dim=1).contiguous()

    shape = moe.MoeShape(T, H, I, E, k)
    ob, os_, obias = moe.interleave_gate_up(shape, stacked(inp["gu_blocks"]).cuda(),
                                            stacked(inp["gu_scales"]).cuda(),
                                            stacked(inp["gu_bias"]).cuda())
    assert torch.equal(ob.cpu(), inp["gu_blocks"])
    assert torch.equal(os_.cpu(), inp["gu_scales"])
    assert torch.equal(obias.cpu(), inp["gu_bias"])


def _sfb_stride(H):
    """Row stride of the activation scales: one byte per 32 elements, padded to whole 64-element
    k-steps and to 32 bytes."""
    return (2 * (-(-H // 64)) + 31) // 32 * 32


def _sfb_natural(sfb):
    """The activation scales in block order: the library stores byte b of row r in 32-bit word
    (b // 4) ^ ((r // 4) % 8), byte b % 4."""
    A, st = sfb.shape
    b = np.arange(st)
    r = np.arange(A)[:, None]
    pos = 4 * ((b[None, :] >> 2) ^ ((r >> 2) & 7)) + (b[None, :] & 3)
    return np.take_along_axis(sfb, pos, axis=1)


def _ws_offsets(T, E, k, H=None, I=None):
    """Offsets of the regions of the forward's workspace (the library's layout: each region
    starts 256-byte aligned, in the order error word, offsets, idx, w, perm, inv, w_row, routing
    scratch (the 32-token segments' expert histograms, their scans over the segments and the
    column totals), activation scales, GLU factors, act, dH, rows)."""
    def up(v):
        return (v + 255) // 256 * 256
    A = T * k
    sizes = [("err", 16), ("off", 4 * (E + 1)), ("idx", 4 * A), ("w", 4 * A), ("perm", 4 * A),
             ("inv", 4 * A), ("w_row", 4 * A), ("blk_hist", 4 * (2 * (-(-T // 32)) * E + E))]
    if H is not None:
        sizes += [("sfb", A * _sfb_stride(H)), ("dgu", 4 * A * I), ("act", 2 * A * I),
                  ("dh", 2 * A * max(2 * I, H)), ("rows", 2 * A * H)]
    o, out = 0, {}
    for name, size in sizes:
        out[name] = o
        o = up(o + size)
    return out


def _e4m3_values(b):
    """E4M3 bytes -> values (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
    exponent field 0 is subnormal with spacing 2^-9)."""
    b = np.asarray(b, np.int64)
    e, m = (b >> 3) & 15, b & 7
    mag = np.where(e > 0, np.ldexp(1.0 + m / 8.0, e - 7), np.ldexp(m / 8.0, -6))
    return np.where(b & 0x80, -mag, mag)


def test_activation_split_matches_the_mx_definition(moe):
    """The gather feeding the block-scaled gate_up GEMM: each expert-sorted row of x, split per
    32 elements into hi + lo E4M3 parts with a UE8M0 scale 2^S, bit for bit the oracle's
    mx_split of the same row (S stored as the UE8M0 byte S + 127)."""
    T, H, I, E, k = 300, 352, 96, 7, 3
    inp = inputs.make_layer(T, H, I, E, k, 41)
    x = inp["x"].clone()
    x[5, :32] = 0.0         # an all-zero block
    x[7, 32:64] *= 2 ** 40  # a large block
    x[9, 64:96] *= 2 ** -40  # a small block, elements far below the rest of the row
    shape = moe.MoeShape(T, H, I, E, k, gate_up_format=1)
    w = moe.weights_to(inp, "cuda")
    ws = moe.alloc_workspace(shape)
    moe.forward(shape, w, x.cuda(), inp["logits"].cuda(), ws)
    assert moe.device_check(ws) == (0, 0)
    o, A = _ws_offsets(T, E, k, H, I), T * k
    wsn = ws.cpu().numpy()
    perm = wsn[o["perm"]:o["perm"] + 4 * A].view(np.int32)
    hi = wsn[o["dh"]:o["dh"] + A * H].reshape(A, H)  # the forward leaves them in the dH region
    lo = wsn[o["dh"] + A * H:o["dh"] + 2 * A * H].reshape(A, H)
    st = _sfb_stride(H)
    sfb = _sfb_natural(wsn[o["sfb"]:o["sfb"] + A * st].reshape(A, st))
    xs = O.bf16_bits_to_f64(x.view(torch.int16).numpy().view(np.uint16))[perm // k]
    rhi, rlo, S = O.mx_split(xs)
    S = S.reshape(A, H // 32)
    zero = np.abs(xs).reshape(A, H // 32, 32).max(axis=2) == 0
    assert np.array_equal(_e4m3_values(hi), rhi) and np.array_equal(_e4m3_values(lo), rlo)
    assert np.array_equal(sfb[:, :H // 32][~zero].astype(np.int64) - 127, S[~zero])
    assert np.all(sfb[:, H // 32:] == 0)


def test_permutation_is_the_stable_expert_sort(moe):
    """K2 exactly: off is the prefix sum of the expert histogram, perm lists each expert's
    (token, slot) assignments in slot order, and inv is its inverse."""
    T, H, I, E, k = 300, 64, 64, 7, 3
    inp = inputs.make_layer(T, H, I, E, k, 31)
    shape = moe.MoeShape(T, H, I, E, k)
    w = moe.weights_to(inp, "cuda")
    ws = moe.alloc_workspace(shape)
    moe.forward(shape, w, inp["x"].cuda(), inp["logits"].cuda(), ws)
    assert moe.device_check(ws) == (0, 0)
    o, A = _ws_offsets(T, E, k), T * k

    def region(name, n):
        return ws[o[name]:o[name] + 4 * n].cpu().view(torch.int32).numpy()

    idx = O.route(inp["logits"].numpy().astype(np.float64), k)[0].reshape(-1)
    assert np.array_equal(region("idx", A), idx)
    hist = np.bincount(idx, minlength=E)
    assert np.array_equal(region("off", E + 1), np.concatenate([[0], np.cumsum(hist)]))
    perm = region("perm", A)
    assert np.array_equal(perm, np.argsort(idx, kind="stable"))
    assert np.array_equal(region("inv", A)[perm], np.arange(A))
