"""The dequantizer fused into the grouped GEMMs, checked bit for bit.

mxfp4_moe_grouped_matmul runs the grouped GEMM the block is built on with a plain epilogue:
out[r] = bf16(x[r] W_e^T), fp32 accumulation.  A row of x that is zero except for one
power-of-two value v at column c picks v * W_e[:, c]: one nonzero product per output, exact
in fp32 and exactly representable in bf16 (v only moves the exponent), so the output equals
the dequantized weight column scaled by v, bit for bit.  That pins the converter warps'
expansion (E2M1 code * 2^(s-127) written to tensor memory) through the tensor-core path,
for both weight layouts:

* the stored rows (forward GEMMs): scales per row and 32-element block along K;
* the transposed copy (backward GEMMs): scales per 32 rows along N, one per element of K.

Scales cover {1, 2, 8, 100} (v = 2^10), {119, 127, 128, 129} (v = 1) and {200, 250, 252}
(v = 2^-10), so both converter factor paths (s <= 128 and s > 128) and the subnormal E2M1
code at s = 1 are hit without leaving fp32's normal range.  A NaN scale (255) must turn every
output of its weight row into NaN (0 * NaN = NaN in the accumulation), as the fp64 reference
matmul does.  Shapes leave a half k-step tail (K = 352) and a partial feature tile (N = 288),
and each expert gets K rows, more than one token tile.
"""

import numpy as np
import pytest
import torch

from mxfp4_quantized_moe_b200 import inputs
from oracle import mxfp4_oracle as O

pytestmark = pytest.mark.gpu

SCALE_SETS = ([1, 2, 8, 100], [119, 127, 128, 129], [200, 250, 252])
V = (2.0 ** 10, 1.0, 2.0 ** -10)


@pytest.fixture(scope="module")
def moe():
    from mxfp4_quantized_moe_b200 import moe as m
    return m


def _packed(E, R, C, seed):
    rng = np.random.default_rng(seed)
    blocks = rng.integers(0, 256, (E, R, C // 2), dtype=np.uint8)
    scales = np.empty((E, R, C // 32), dtype=np.uint8)
    for e in range(E):
        scales[e] = rng.choice(SCALE_SETS[e], (R, C // 32))
    return blocks, scales


def _one_hot_rows(E, K):
    """Expert e gets K rows; row c of its range is v_e at column c, zero elsewhere."""
    x = np.zeros((E * K, K), dtype=np.float32)
    for e in range(E):
        x[e * K + np.arange(K), np.arange(K)] = V[e]
    off = np.arange(E + 1, dtype=np.int32) * K
    return torch.from_numpy(x).to(torch.bfloat16), torch.from_numpy(off)


def _expected(W, E, K):
    """Row c of expert e: v_e * W_e[:, c] (W: fp64 [E][N][K]), as bf16 bit patterns."""
    out = np.concatenate([V[e] * W[e].T for e in range(E)], axis=0)  # [E*K][N]
    return O.f64_to_bf16_bits(out)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _same(got_bits, ref_bits):
    """Bit-for-bit, except that +0 and -0 compare equal (the accumulator adds signed zeros)."""
    zero = ((got_bits & 0x7FFF) == 0) & ((ref_bits & 0x7FFF) == 0)
    return np.all((got_bits == ref_bits) | zero)


def test_converter_stored_rows_bit_exact(moe):
    E, N, K = 3, 288, 352
    blocks, scales = _packed(E, N, K, 1)
    x, off = _one_hot_rows(E, K)
    out = moe.grouped_matmul(off.cuda(), x.cuda(), torch.from_numpy(blocks).cuda(),
                             torch.from_numpy(scales).cuda(), N, transposed=False)
    torch.cuda.synchronize()
    W = O.dequantize(blocks, scales)  # [E][N][K]
    assert _same(_bits(out), _expected(W, E, K))


def test_converter_transposed_copy_bit_exact(moe):
    """The backward reads the transposed copy: element (i, h) of W_d^T with the scale of
    W_d[h][i // 32 block]; one-hot rows over h pick rows h of the stored W_d."""
    H, I, E = 352, 288, 3
    dn_blocks, dn_scales = _packed(E, H, I, 2)  # W_d [E][H][I]
    gu_blocks, gu_scales = _packed(E, 2 * I, H, 3)
    shape = moe.MoeShape(8, H, I, E, 2)
    w = {"gu_blocks": torch.from_numpy(gu_blocks).cuda(), "gu_scales": torch.from_numpy(gu_scales).cuda(),
         "gu_bias": torch.zeros(E, 2 * I, dtype=torch.bfloat16, device="cuda"),
         "dn_blocks": torch.from_numpy(dn_blocks).cuda(), "dn_scales": torch.from_numpy(dn_scales).cuda(),
         "dn_bias": torch.zeros(E, H, dtype=torch.bfloat16, device="cuda")}
    wt = moe.transpose_weights(shape, w)
    def up(v):
        return -(-v // 256) * 256
    n_dn = E * I * H // 2
    dn_t = wt[:n_dn]
    o = up(up(n_dn) + E * H * I)  # the gate_up copy follows, then the down scales
    dn_st = wt[o:o + E * (I // 32) * H]
    x, off = _one_hot_rows(E, H)
    out = moe.grouped_matmul(off.cuda(), x.cuda(), dn_t, dn_st, I, transposed=True)
    torch.cuda.synchronize()
    Wd = O.dequantize(dn_blocks, dn_scales)  # [E][H][I]; (W_d^T)[e][i][h] = Wd[e][h][i]
    assert _same(_bits(out), _expected(Wd.transpose(0, 2, 1), E, H))


def test_converter_nan_scale_poisons_its_row(moe):
    E, N, K = 1, 64, 128
    blocks, scales = _packed(E, N, K, 4)
    scales[0, 5, 2] = 255  # weight row 5, elements 64..95: NaN
    x, off = _one_hot_rows(E, K)
    out = moe.grouped_matmul(off.cuda(), x.cuda(), torch.from_numpy(blocks).cuda(),
                             torch.from_numpy(scales).cuda(), N, transposed=False)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    ref = x.double().numpy() @ O.dequantize(blocks, scales)[0].T  # NaN where 0 * NaN enters
    assert np.isnan(ref[:, 5]).all() and not np.isnan(np.delete(ref, 5, axis=1)).any()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], O.bf16_bits_to_f64(O.f64_to_bf16_bits(ref[ok])))
