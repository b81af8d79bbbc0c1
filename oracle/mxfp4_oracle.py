"""Plain fp64 CPU restatement of the MXFP4 MoE expert block (forward + input gradients).

TEST INFRASTRUCTURE ONLY: see the package docstring.  Slow on purpose: an
expert-major loop over weights dequantized on the fly, numpy matmuls in fp64, no
blocking, no fusion.  It shares no code, table or constant generator with the
CUDA path.

What it follows
---------------
* "Add MXFP4 training support via a dequantize-on-the-fly fallback"
  (huggingface/transformers #47464), section "What this does": the eager
  reference math (top-k router + GptOssExperts-style expert loop) over weights
  dequantized per expert, the packed MXFP4 storage left untouched; section
  "Relation to the backward triton kernels": that eager math is the numerical
  reference the backward kernels are validated against, and the frozen base
  weights get no weight gradient (only the input path needs gradients).
* "Integrate finegrained kernels: SOTA performance and per-module quantization"
  (huggingface/transformers #49658), commit "gate|up row-interleaved": gate j sits
  at row 2j and up j at row 2j+1, and the GLU de-interleaves with a stride-2
  split; commit "per-expert bias as a bias= operand": the bias rides the same
  output-row axis as the weight (so it is in interleaved order for gate_up) and
  is added inside both GEMMs, while the host keeps only the routing-weighted
  reduce; the `mxfp4` format pins UE8M0 scales and group-32 blocks.
* MXFP4 element and scale encodings: OCP Microscaling Formats (MX) v1.0,
  E2M1 elements (1 sign, 2 exponent bits with bias 1, 1 mantissa bit; exponent
  field 0 is subnormal) and UE8M0 scales (2^(s-127), s = 255 is NaN), 32
  elements per block.
* The GPT-OSS expert activation: g' = min(g, limit), u' = clamp(u, -limit,
  limit), act = (u' + 1) * g' * sigmoid(alpha * g'), alpha = 1.702, limit = 7.

Readings where the pages are silent (each pinned by a test):
* nibble order: element 2i is the low nibble of byte i, element 2i+1 the high;
* routing: top-k on the raw logits (ties to the lower expert index), then a
  softmax over the k selected logits; slot j of a token holds its j-th largest;
* bias placement: added before the GLU clamp (gate_up) and before the routing
  weight multiply (down), so the routing weight scales the down bias too;
* clamp derivative: inclusive mask (gradient passes at g == limit, |u| == limit),
  decided on the gate_up pre-activation rounded to bf16.  The eager reference runs the
  GPT-OSS expert loop on bf16 tensors (its dequantized transients are bf16), so autograd's
  clamp backward sees h as a bf16 tensor; the mask is a yes/no decision and is taken in
  that precision.  Everything else stays fp64.
"""

from __future__ import annotations

import numpy as np

# E2M1 magnitudes for the 3-bit code (exponent e = bits 2..1, mantissa m = bit 0):
# e == 0 is subnormal (m * 0.5), otherwise 2^(e-1) * (1 + m/2).  Built from the
# encoding rule, not typed in, so that the golden table pins it.
E2M1_MAGNITUDES = np.array(
    [(0.5 * (c & 1)) if (c >> 1) == 0 else 2.0 ** ((c >> 1) - 1) * (1.0 + 0.5 * (c & 1))
     for c in range(8)],
    dtype=np.float64,
)

BLOCK = 32  # elements per UE8M0 scale (MX block size)


# --------------------------------------------------------------------------------------
# MXFP4 decode (OCP MX v1.0: E2M1 elements, UE8M0 scales, 32-element blocks)
# --------------------------------------------------------------------------------------
def decode_e2m1(codes) -> np.ndarray:
    """E2M1 code (0..15) -> value, fp64.  Bit 3 is the sign; code 8 is -0.0."""
    codes = np.asarray(codes, dtype=np.int64)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where((codes >> 3) & 1, -mag, mag)


def decode_ue8m0(s) -> np.ndarray:
    """UE8M0 scale byte -> 2^(s-127) in fp64; s == 255 encodes NaN."""
    s = np.asarray(s, dtype=np.int64)
    val = np.ldexp(1.0, s - 127)
    return np.where(s == 255, np.nan, val)


def dequantize(blocks, scales) -> np.ndarray:
    """Packed MXFP4 rows -> fp64 values.

    ``blocks``: uint8 [..., R, K/2]; byte i of a row holds element 2i in its low
    nibble and element 2i+1 in its high nibble.  ``scales``: uint8 [..., R, K/32],
    one UE8M0 scale per 32 consecutive elements of a row.  Returns [..., R, K].
    """
    blocks = np.asarray(blocks, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    lo = blocks & 0x0F
    hi = blocks >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*blocks.shape[:-1], blocks.shape[-1] * 2)
    K = codes.shape[-1]
    if scales.shape[-1] * BLOCK != K:
        raise ValueError(f"scales last dim {scales.shape[-1]} does not cover K={K}")
    scale = np.repeat(decode_ue8m0(scales), BLOCK, axis=-1)
    return decode_e2m1(codes) * scale


# --------------------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even; subnormals kept; overflow -> inf)
# --------------------------------------------------------------------------------------
def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values to bf16 (RNE) and return the 16-bit patterns."""
    with np.errstate(over="ignore", invalid="ignore"):
        return _f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def _f64_to_bf16_bits(x):
    sign = np.signbit(x).astype(np.uint32) << 15
    a = np.abs(x)
    out = np.zeros(x.shape, dtype=np.uint32)
    finite = np.isfinite(a) & (a > 0)
    af = np.where(finite, a, 1.0)
    _, ex = np.frexp(af)  # af = m * 2^ex, m in [0.5, 1)
    k = ex.astype(np.int64) - 1  # af in [2^k, 2^(k+1))
    q = np.maximum(k - 7, -133)  # quantum: 7 fraction bits, or the subnormal step 2^-133
    n = np.ldexp(af, -q)  # exact power-of-two rescale
    r = np.rint(n)  # numpy rint rounds half to even
    v = np.ldexp(r, q)
    # encode v
    _, ev = np.frexp(np.where(v > 0, v, 1.0))
    kv = ev.astype(np.int64) - 1
    normal = v >= 2.0 ** -126
    E = kv + 127
    mant_n = np.ldexp(np.where(normal, v, 2.0 ** -126), -(np.where(normal, kv, -126) - 7)) - 128.0
    mant_s = np.ldexp(np.where(normal, 0.0, v), 133)
    mant = np.where(normal, mant_n, mant_s).astype(np.int64)
    bits = np.where(normal, (E << 7) | mant, mant)
    bits = np.where(normal & (E >= 255), 0x7F80, bits)
    bits = np.where(v == 0, 0, bits)
    out = np.where(finite, bits, out)
    out = np.where(np.isinf(a), 0x7F80, out)
    out = np.where(np.isnan(a), 0x7FC0, out)
    out = np.where(np.isnan(a), out, out | sign)
    return out.astype(np.uint16)


def round_bf16(x) -> np.ndarray:
    """fp64 values rounded to the nearest bf16 (ties to even), as fp64."""
    return bf16_bits_to_f64(f64_to_bf16_bits(x))


def bf16_bits_to_f64(bits) -> np.ndarray:
    """16-bit bf16 patterns -> fp64 values (exact)."""
    b = np.asarray(bits, dtype=np.int64) & 0xFFFF
    s = (b >> 15) & 1
    E = (b >> 7) & 0xFF
    m = b & 0x7F
    mag = np.where(E == 0, np.ldexp(m.astype(np.float64), -133),
                   np.ldexp((128 + m).astype(np.float64), E - 134))
    mag = np.where(E == 255, np.where(m == 0, np.inf, np.nan), mag)
    return np.where(s == 1, -mag, mag)


# --------------------------------------------------------------------------------------
# Routing: top-k on logits, softmax over the k selected
# --------------------------------------------------------------------------------------
def route(logits, k: int):
    """Return (idx [T,k] int64, w [T,k] fp64).

    The k largest logits of each token, largest first; equal logits go to the
    lower expert index.  w is the softmax over those k logits, in fp64.
    """
    logits = np.asarray(logits)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    lg = logits.astype(np.float64)
    idx = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(lg, idx, axis=1)
    z = np.exp(sel - sel[:, :1])
    w = z / z.sum(axis=1, keepdims=True)
    return idx.astype(np.int64), w


# --------------------------------------------------------------------------------------
# Clamped GLU on interleaved gate/up columns
# --------------------------------------------------------------------------------------
def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def glu(h, alpha: float = 1.702, limit: float = 7.0):
    """act[..., j] from h[..., 2j] (gate) and h[..., 2j+1] (up)."""
    h = np.asarray(h, dtype=np.float64)
    g = h[..., 0::2]
    u = h[..., 1::2]
    gc = np.minimum(g, limit)
    uc = np.clip(u, -limit, limit)
    return (uc + 1.0) * gc * _sigmoid(alpha * gc)


def glu_backward(h, dact, alpha: float = 1.702, limit: float = 7.0, h_mask=None):
    """d(act)/d(h) applied to dact; returns dh with the same interleaved layout as h.

    The clamps pass the gradient where g <= limit and -limit <= u <= limit (inclusive).
    ``h_mask`` (default: h) is the tensor those two decisions are taken on.
    """
    h = np.asarray(h, dtype=np.float64)
    dact = np.asarray(dact, dtype=np.float64)
    hm = h if h_mask is None else np.asarray(h_mask, dtype=np.float64)
    g = h[..., 0::2]
    u = h[..., 1::2]
    gm = hm[..., 0::2]
    um = hm[..., 1::2]
    gc = np.minimum(g, limit)
    uc = np.clip(u, -limit, limit)
    s = _sigmoid(alpha * gc)
    d_gc = (uc + 1.0) * (s + alpha * gc * s * (1.0 - s))
    d_uc = gc * s
    dg = dact * d_gc * (gm <= limit)
    du = dact * d_uc * ((um >= -limit) & (um <= limit))
    dh = np.empty(h.shape, dtype=np.float64)
    dh[..., 0::2] = dg
    dh[..., 1::2] = du
    return dh


# --------------------------------------------------------------------------------------
# Expert loop (forward and input-gradient backward)
# --------------------------------------------------------------------------------------
def _expert_weights(W, e):
    wgu = dequantize(W["gu_blocks"][e], W["gu_scales"][e])  # [2I, H]
    wd = dequantize(W["dn_blocks"][e], W["dn_scales"][e])  # [H, I]
    return wgu, wd


def _weights_of(W, e):
    """Dequantized weights of expert e.  When the caller puts a dict under
    W["_dequant_cache"], each expert is dequantized once and reused (same values)."""
    cache = W.get("_dequant_cache")
    if cache is None:
        return _expert_weights(W, e)
    if e not in cache:
        cache[e] = _expert_weights(W, e)
    return cache[e]


def moe_forward(x, logits, W, k: int, alpha: float = 1.702, limit: float = 7.0):
    """Forward of the expert block.

    x [T,H] (values of the bf16 activations), logits [T,E] fp32, W a dict with
    gu_blocks [E,2I,H/2], gu_scales [E,2I,H/32], gu_bias [E,2I] (interleaved rows),
    dn_blocks [E,H,I/2], dn_scales [E,H,I/32], dn_bias [E,H].

    Returns a dict: out [T,H], idx [T,k], w [T,k], and the per-slot
    pre-activations h [T,k,2I] and expert outputs y [T,k,H] kept for the backward.
    """
    x = np.asarray(x, dtype=np.float64)
    T, H = x.shape
    E = logits.shape[1]
    idx, w = route(logits, k)
    I2 = W["gu_blocks"].shape[1]
    h_slot = np.zeros((T, k, I2), dtype=np.float64)
    y_slot = np.zeros((T, k, H), dtype=np.float64)
    gu_bias = np.asarray(W["gu_bias"], dtype=np.float64)
    dn_bias = np.asarray(W["dn_bias"], dtype=np.float64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)  # slot order t*k + j
        if tt.size == 0:
            continue
        wgu, wd = _weights_of(W, e)
        h = x[tt] @ wgu.T + gu_bias[e]
        act = glu(h, alpha, limit)
        y = act @ wd.T + dn_bias[e]
        h_slot[tt, jj] = h
        y_slot[tt, jj] = y
    out = np.einsum("tj,tjh->th", w, y_slot)
    return {"out": out, "idx": idx, "w": w, "h": h_slot, "y": y_slot}


def moe_backward(dY, fwd, W, alpha: float = 1.702, limit: float = 7.0):
    """Input-gradient backward through the frozen quantized weights (no dW).

    Returns (dX [T,H], d_w [T,k], d_logits [T,E]).
    d_w[t,j] = <dY_t, y_{t,j}> (y including the down bias); d_logits is the
    softmax-over-k Jacobian applied to d_w, zero for unselected experts.
    """
    dY = np.asarray(dY, dtype=np.float64)
    idx, w = fwd["idx"], fwd["w"]
    T, k = idx.shape
    E = int(W["gu_blocks"].shape[0])
    H = dY.shape[1]
    dX = np.zeros((T, H), dtype=np.float64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)
        if tt.size == 0:
            continue
        wgu, wd = _weights_of(W, e)
        dy = w[tt, jj][:, None] * dY[tt]
        dact = dy @ wd  # [n, I]
        h = fwd["h"][tt, jj]
        # clamp masks decided on the pre-activation as the eager bf16 model holds it
        dh = glu_backward(h, dact, alpha, limit, h_mask=round_bf16(h))  # [n, 2I]
        dx = dh @ wgu  # [n, H]
        np.add.at(dX, tt, dx)
    d_w = np.einsum("th,tjh->tj", dY, fwd["y"])
    s = (w * d_w).sum(axis=1, keepdims=True)
    d_sel = w * (d_w - s)
    d_logits = np.zeros((T, E), dtype=np.float64)
    np.put_along_axis(d_logits, idx, d_sel, axis=1)
    return dX, d_w, d_logits


# --------------------------------------------------------------------------------------
# Residual stack of blocks (the caller's side: router linear and residual add)
# --------------------------------------------------------------------------------------
def stack_forward(x, layers, k: int, alpha: float = 1.702, limit: float = 7.0):
    """x_{l+1} = x_l + block_l(x_l, logits_l), logits_l = x_l W_r^l + b_r^l, all in fp64.

    layers: list of dicts {"W": block weights as for moe_forward, "w_r": [H,E], "b_r": [E]}.
    Returns (x_L, records) with records[l] = {"x": x_l, "logits": logits_l, "fwd": ...}.
    """
    x = np.asarray(x, dtype=np.float64)
    recs = []
    for L in layers:
        logits = x @ np.asarray(L["w_r"], np.float64) + np.asarray(L["b_r"], np.float64)
        f = moe_forward(x, logits, L["W"], k, alpha, limit)
        recs.append({"x": x, "logits": logits, "fwd": f})
        x = x + f["out"]
    return x, recs


def stack_backward(dY, recs, layers, alpha: float = 1.702, limit: float = 7.0):
    """dL/dx_0 of the stack: walking the blocks backwards, the gradient of block l's input
    is the residual path plus the block's input gradient plus the router path,
        g_l = g_{l+1} + dX_l + d_logits_l (W_r^l)^T,
    where (dX_l, d_logits_l) are the block's input gradients for upstream g_{l+1}.
    Returns (g_0, per-layer (g_{l+1}, dX_l, d_w_l, d_logits_l), in layer order)."""
    g = np.asarray(dY, dtype=np.float64)
    per = [None] * len(layers)
    for l in range(len(layers) - 1, -1, -1):
        dX, d_w, d_logits = moe_backward(g, recs[l]["fwd"], layers[l]["W"], alpha, limit)
        per[l] = (g, dX, d_w, d_logits)
        g = g + dX + d_logits @ np.asarray(layers[l]["w_r"], np.float64).T
    return g, per


# --------------------------------------------------------------------------------------
# MXFP8 (E4M3) activations: the split a block-scaled forward would feed the tensor cores.
# Not used by the current GPU path; these functions state the reading such a path is held to.
# --------------------------------------------------------------------------------------
E4M3_MAX = 448.0  # exponent field 15 with mantissa 110 (mantissa 111 there is NaN)


def round_e4m3(v) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to even (OCP MX v1.0 E4M3: 1 sign bit, 4 exponent
    bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal with spacing 2^-9).
    Magnitudes above the largest finite value, 448, give NaN (the format has no infinity)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = m * 2^ex, m in [0.5, 1)
    lead = np.maximum(ex - 1, -6)               # binade of the leading bit; subnormals share -6
    q = np.ldexp(1.0, lead - 3)                 # spacing: 3 mantissa bits
    r = np.round(a / q) * q                     # a / q is exact; np.round ties to even
    out = np.copysign(r, v)
    return np.where(r > E4M3_MAX, np.nan, out)


def mx_split(x, block: int = BLOCK):
    """Split each `block`-element run of x (along the last axis) into two E4M3 parts with a
    shared power-of-two scale: x = (hi + lo) * 2^S up to the rounding of lo, where 2^S is the
    smallest power of two that brings the run's largest magnitude to at most 448,
    hi = e4m3(x / 2^S) and lo = e4m3(x / 2^S - hi).  Returns (hi, lo, S) with S per run."""
    x = np.asarray(x, dtype=np.float64)
    shp = x.shape
    xb = x.reshape(-1, block)
    amax = np.abs(xb).max(axis=1)
    m, ex = np.frexp(np.where(amax > 0, amax / E4M3_MAX, 1.0))
    S = np.where(m == 0.5, ex - 1, ex)          # ceil(log2(amax / 448)), exactly
    S = np.where(amax > 0, S, 0).astype(np.int64)
    y = np.ldexp(xb, -S[:, None])
    hi = round_e4m3(y)
    lo = round_e4m3(y - hi)
    return hi.reshape(shp), lo.reshape(shp), S
