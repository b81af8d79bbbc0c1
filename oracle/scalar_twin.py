"""Brute-force twin of the oracle for tiny cases (TEST INFRASTRUCTURE ONLY).

Pure-Python loops, token-major, no numpy linear algebra and no permutation: for
each token it picks the k experts by repeated selection, decodes each weight
element from its nibble and scale as it is used, and sums products one by one.
It restates the same definitions as ``mxfp4_oracle`` in a different structure,
so that a slip in the oracle's routing, permutation, combine or matmul operand
order shows up as a mismatch.  Use it only for T*E*H*I up to a few hundred
thousand (it takes seconds there).

Definitions followed: OCP Microscaling Formats (MX) v1.0 for E2M1/UE8M0; the
eager expert loop of "Add MXFP4 training support via a dequantize-on-the-fly
fallback" (section "What this does"); the interleaved gate/up rows and the
per-expert bias operand of "Integrate finegrained kernels: SOTA performance and
per-module quantization"; the GPT-OSS clamped GLU.
"""

from __future__ import annotations

import math


def _e2m1(code: int) -> float:
    sign = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        return sign * 0.5 * m
    return sign * math.ldexp(1.0 + 0.5 * m, e - 1)


def _scale(s: int) -> float:
    return math.nan if s == 255 else math.ldexp(1.0, s - 127)


def weight(blocks, scales, e: int, row: int, col: int) -> float:
    """Element (row, col) of expert e's packed matrix."""
    byte = int(blocks[e][row][col // 2])
    code = (byte >> 4) if (col & 1) else (byte & 15)
    return _e2m1(code) * _scale(int(scales[e][row][col // 32]))


def _matrix(blocks, scales, e, rows, cols):
    return [[weight(blocks, scales, e, r, c) for c in range(cols)] for r in range(rows)]


def _topk(row, k):
    chosen = []
    for _ in range(k):
        best = -1
        for i, v in enumerate(row):
            if i in chosen:
                continue
            if best < 0 or v > row[best]:
                best = i
        chosen.append(best)
    return chosen


def _bf16(v: float) -> float:
    """Round to the nearest bf16 (8 significant bits, ties to even); normal range only."""
    if v == 0.0 or math.isinf(v) or math.isnan(v):
        return v
    m, e = math.frexp(v)  # v = m * 2^e, 0.5 <= |m| < 1
    return math.ldexp(round(m * 256.0), e - 8)  # Python round() is half-to-even


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def forward_backward(x, logits, dY, W, k, alpha=1.702, limit=7.0):
    """Returns dict(out, idx, w, dX, d_w, d_logits) as nested Python lists."""
    T = len(x)
    H = len(x[0])
    E = len(logits[0])
    I2 = len(W["gu_blocks"][0])
    I = I2 // 2
    cache = {}

    def mats(e):
        if e not in cache:
            cache[e] = (_matrix(W["gu_blocks"], W["gu_scales"], e, I2, H),
                        _matrix(W["dn_blocks"], W["dn_scales"], e, H, I))
        return cache[e]

    out, idx_all, w_all, dX, dW, dL = [], [], [], [], [], []
    for t in range(T):
        sel = _topk([float(v) for v in logits[t]], k)
        m = max(float(logits[t][e]) for e in sel)
        z = [math.exp(float(logits[t][e]) - m) for e in sel]
        zs = sum(z)
        w = [v / zs for v in z]
        o = [0.0] * H
        dx_t = [0.0] * H
        dw_t = []
        for j, e in enumerate(sel):
            wgu, wd = mats(e)
            bgu = W["gu_bias"][e]
            bd = W["dn_bias"][e]
            hrow = [sum(x[t][c] * wgu[n][c] for c in range(H)) + bgu[n] for n in range(I2)]
            act, dgc, duc, gm, um = [], [], [], [], []
            for i in range(I):
                g, u = hrow[2 * i], hrow[2 * i + 1]
                gc = g if g < limit else limit
                uc = -limit if u < -limit else (limit if u > limit else u)
                s = _sig(alpha * gc)
                act.append((uc + 1.0) * gc * s)
                dgc.append((uc + 1.0) * (s + alpha * gc * s * (1.0 - s)))
                duc.append(gc * s)
                gb, ub = _bf16(g), _bf16(u)  # clamp masks decided on bf16 pre-activations
                gm.append(1.0 if gb <= limit else 0.0)
                um.append(1.0 if -limit <= ub <= limit else 0.0)
            y = [sum(act[i] * wd[hh][i] for i in range(I)) + bd[hh] for hh in range(H)]
            for hh in range(H):
                o[hh] += w[j] * y[hh]
            dw_t.append(sum(dY[t][hh] * y[hh] for hh in range(H)))
            dy = [w[j] * dY[t][hh] for hh in range(H)]
            dact = [sum(dy[hh] * wd[hh][i] for hh in range(H)) for i in range(I)]
            dh = [0.0] * I2
            for i in range(I):
                dh[2 * i] = dact[i] * dgc[i] * gm[i]
                dh[2 * i + 1] = dact[i] * duc[i] * um[i]
            for c in range(H):
                dx_t[c] += sum(dh[n] * wgu[n][c] for n in range(I2))
        s_w = sum(w[j] * dw_t[j] for j in range(k))
        dl = [0.0] * E
        for j, e in enumerate(sel):
            dl[e] = w[j] * (dw_t[j] - s_w)
        out.append(o)
        idx_all.append(sel)
        w_all.append(w)
        dX.append(dx_t)
        dW.append(dw_t)
        dL.append(dl)
    return {"out": out, "idx": idx_all, "w": w_all, "dX": dX, "d_w": dW, "d_logits": dL}
