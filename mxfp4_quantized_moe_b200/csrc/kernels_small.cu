// Routing, permutation, gather/combine, routing backward, standalone dequant and the
// one-time weight transpose.  All of these are memory- or latency-bound; the grouped
// GEMMs live in grouped_gemm.cu.
#include "common.cuh"
#include "kernels.h"
#include "aux_kernels.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------------------------------
// Router: top-k over the E logits of a token (largest first, equal logits -> lower expert
// index), softmax over the k selected, expert histogram.  One thread per token.
// Source: the top-k router of the eager expert loop ("Add MXFP4 training support via a
// dequantize-on-the-fly fallback", section "What this does"); softmax over the k values.
// ---------------------------------------------------------------------------------------
__global__ void router_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                   int32_t* __restrict__ idx, float* __restrict__ w,
                                   int32_t* __restrict__ hist, int32_t* __restrict__ user_idx,
                                   float* __restrict__ user_w) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  uint32_t taken[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // E <= 256
  int sel[16];
  float val[16];
  float m0 = 0.f, zsum = 0.f;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    float bv = 0.f;
    for (int e = 0; e < E; ++e) {
      if (taken[e >> 5] & (1u << (e & 31))) continue;
      const float v = __ldg(row + e);
      if (best < 0 || v > bv) {
        best = e;
        bv = v;
      }
    }
    taken[best >> 5] |= 1u << (best & 31);
    if (j == 0) m0 = bv;
    const float z = __expf(bv - m0);
    zsum += z;
    if (j < 16) {
      sel[j] = best;
      val[j] = z;
    }
    atomicAdd(hist + best, 1);
    idx[(size_t)t * k + j] = best;
    w[(size_t)t * k + j] = z;  // normalized below
  }
  const float inv = 1.f / zsum;
  for (int j = 0; j < k; ++j) {
    const float z = (j < 16) ? val[j] : w[(size_t)t * k + j];
    const int e = (j < 16) ? sel[j] : idx[(size_t)t * k + j];
    const float wj = z * inv;
    w[(size_t)t * k + j] = wj;
    if (user_idx) user_idx[(size_t)t * k + j] = e;
    if (user_w) user_w[(size_t)t * k + j] = wj;
  }
}

// ---------------------------------------------------------------------------------------
// Stable counting sort of the A = T*k slots by expert.  Block e owns expert e: it scans
// the slots in order and gives each slot of expert e the next row of [off[e], off[e+1]).
// perm[row] = slot, inv[slot] = row.  Block 0 also publishes off[0..E].
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) build_perm_kernel(const int32_t* __restrict__ idx, int A,
                                                          int E, const int32_t* __restrict__ hist,
                                                          int32_t* __restrict__ off,
                                                          int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ inv, int* err) {
  __shared__ int s_base;
  __shared__ int s_warp[32];
  __shared__ int s_run;
  const int e = blockIdx.x;
  if (threadIdx.x == 0) {
    int base = 0;
    for (int i = 0; i < e; ++i) base += hist[i];
    s_base = base;
    s_run = 0;
    if (e == 0) {
      int acc = 0;
      for (int i = 0; i < E; ++i) {
        off[i] = acc;
        acc += hist[i];
      }
      off[E] = acc;
      if (acc != A) DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x100);
    }
  }
  __syncthreads();
  const int base = s_base;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int c = 0; c < A; c += blockDim.x) {
    const int slot = c + threadIdx.x;
    const bool f = slot < A && idx[slot] == e;
    const unsigned b = __ballot_sync(kFull, f);
    if (lane == 0) s_warp[wid] = __popc(b);
    __syncthreads();
    if (wid == 0) {
      const int v = (lane < (int)(blockDim.x >> 5)) ? s_warp[lane] : 0;
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      s_warp[lane] = incl - v;  // exclusive prefix over the block's warps
    }
    __syncthreads();
    const int pos = s_run + s_warp[wid] + __popc(b & ((1u << lane) - 1u));
    if (f) {
      const int row = base + pos;
      if (row < A) {
        perm[row] = slot;
        inv[slot] = row;
      } else {
        DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x101);
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_run = pos + (f ? 1 : 0);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------
// dst[row] = src[perm[row] / k] for every expert-sorted row (one warp per row, 16-byte
// vectors).  With `bias`, also dot_out[row] = <src row, bias[e(row)]> in fp32, e(row) the
// expert owning the row (the down-bias term of the routing-weight gradient).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int expert_of_row(const int32_t* off, int E, int row) {
  int lo = 0, hi = E;  // off[lo] <= row < off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(off + mid) <= row) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void gather_rows_kernel(const uint16_t* __restrict__ src, int H, int k,
                                   const int32_t* __restrict__ perm, int A,
                                   uint16_t* __restrict__ dst, const int32_t* __restrict__ off,
                                   int E, const uint16_t* __restrict__ bias,
                                   float* __restrict__ dot_out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= A) return;
  const int row = warp;
  const int t = perm[row] / k;
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)t * H);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)row * H);
  const int nv = H / 8;
  float acc = 0.f;
  const uint4* bv = nullptr;
  if (bias) bv = reinterpret_cast<const uint4*>(bias + (size_t)expert_of_row(off, E, row) * H);
  for (int i = lane; i < nv; i += 32) {
    const uint4 v = __ldg(s + i);
    d[i] = v;
    if (bias) {
      const uint4 b = __ldg(bv + i);
      acc += bf16_lo(v.x) * bf16_lo(b.x) + bf16_hi(v.x) * bf16_hi(b.x);
      acc += bf16_lo(v.y) * bf16_lo(b.y) + bf16_hi(v.y) * bf16_hi(b.y);
      acc += bf16_lo(v.z) * bf16_lo(b.z) + bf16_hi(v.z) * bf16_hi(b.z);
      acc += bf16_lo(v.w) * bf16_lo(b.w) + bf16_hi(v.w) * bf16_hi(b.w);
    }
  }
  if (bias) {
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) dot_out[row] = acc;
  }
}

// out[t] = sum_j slots[t*k + j] in fp32, rounded to bf16 once.  8 bf16 per thread.
__global__ void combine_kernel(const uint16_t* __restrict__ slots, int T, int k, int H,
                               uint16_t* __restrict__ out) {
  const int nv = H / 8;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)T * nv) return;
  const int t = (int)(i / nv), c = (int)(i % nv);
  float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(slots + ((size_t)t * k + j) * H) + c);
    a[0] += bf16_lo(v.x); a[1] += bf16_hi(v.x);
    a[2] += bf16_lo(v.y); a[3] += bf16_hi(v.y);
    a[4] += bf16_lo(v.z); a[5] += bf16_hi(v.z);
    a[6] += bf16_lo(v.w); a[7] += bf16_hi(v.w);
  }
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]);
  o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]);
  o.w = pack_bf16x2(a[6], a[7]);
  reinterpret_cast<uint4*>(out + (size_t)t * H)[c] = o;
}

// Routing-weight gradient per expert-sorted row: dw[r] = <dY_t, b_d[e]> + sum of the GEMM's
// per-32-feature partial <dZ_r, act_r>; written to its slot.  Reads of the [P][A] partials
// are coalesced across threads (consecutive rows).
__global__ void reduce_dw_kernel(const float* __restrict__ cbias, const float* __restrict__ dw_part,
                                 int nparts, int A, const int32_t* __restrict__ perm,
                                 float* __restrict__ dw, float* __restrict__ d_topk_w) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= A) return;
  float v = cbias[r];
  for (int q = 0; q < nparts; ++q) v += __ldg(dw_part + (size_t)q * A + r);
  dw[r] = v;
  d_topk_w[perm[r]] = v;
}

// d_logits through the softmax over the k selected logits:
// d_l[idx_j] = w_j (d_w_j - sum_i w_i d_w_i), 0 for the experts not selected.
__global__ void router_backward_kernel(const int32_t* __restrict__ idx,
                                       const float* __restrict__ w,
                                       const float* __restrict__ d_topk_w, int T, int E, int k,
                                       float* __restrict__ d_logits) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float s = 0.f;
  for (int j = 0; j < k; ++j) s += w[t * k + j] * d_topk_w[t * k + j];
  float* dl = d_logits + (size_t)t * E;
  for (int e = 0; e < E; ++e) dl[e] = 0.f;
  for (int j = 0; j < k; ++j) {
    const int slot = t * k + j;
    dl[idx[slot]] = w[slot] * (d_topk_w[slot] - s);
  }
}

// One thread per 8 elements (one 32-bit word of codes, a quarter of an MX block): a warp reads
// 128 contiguous bytes of codes and writes 512 contiguous bytes of bf16.
__global__ void dequant_kernel(const uint8_t* __restrict__ blocks,
                               const uint8_t* __restrict__ scales, int64_t nwords,
                               uint16_t* __restrict__ out) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= nwords) return;
  const uint32_t q = __ldg(reinterpret_cast<const uint32_t*>(blocks) + t);
  const uint32_t s = __ldg(scales + (t >> 2));
  const uint32_t f1 = dup16(ue8m0_f1(s)), f2 = dup16(ue8m0_f2(s));
  uint32_t p[4];
  e2m1x8_to_bf16x2_pattern(q, p);
  uint4 v;
  v.x = bmul2(bmul2(p[0], f1), f2);
  v.y = bmul2(bmul2(p[1], f1), f2);
  v.z = bmul2(bmul2(p[2], f1), f2);
  v.w = bmul2(bmul2(p[3], f1), f2);
  if (s == 255u) v = make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);  // quiet NaN
  reinterpret_cast<uint4*>(out)[t] = v;
}

// Packed nibble transpose: src [E][R][C/2] (packed along C) -> dst [E][C][R/2] (packed
// along R).  One 32x32-element tile per block of 32 threads.
__global__ void transpose_packed_kernel(const uint8_t* __restrict__ src, int R, int C,
                                        uint8_t* __restrict__ dst) {
  __shared__ uint8_t nib[32][33];
  const int e = blockIdx.z, r0 = blockIdx.y * 32, c0 = blockIdx.x * 32, tid = threadIdx.x;
  const uint8_t* s = src + (size_t)e * R * (C / 2);
  // thread tid loads row r0+tid, 16 bytes = 32 nibbles along C
  const uint4 v = *reinterpret_cast<const uint4*>(s + (size_t)(r0 + tid) * (C / 2) + c0 / 2);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t byte = (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    nib[tid][2 * i] = byte & 0xF;
    nib[tid][2 * i + 1] = byte >> 4;
  }
  __syncthreads();
  // thread tid writes output row c0+tid, 16 bytes = 32 nibbles along R
  uint32_t o[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t byte = nib[2 * i][tid] | (nib[2 * i + 1][tid] << 4);
    o[i >> 2] |= byte << (8 * (i & 3));
  }
  uint8_t* d = dst + (size_t)e * C * (R / 2);
  *reinterpret_cast<uint4*>(d + (size_t)(c0 + tid) * (R / 2) + r0 / 2) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Scale transpose: src [E][R][C/32] -> dst [E][C/32][R].
__global__ void transpose_scales_kernel(const uint8_t* __restrict__ src, int R, int CB,
                                        uint8_t* __restrict__ dst, int64_t total) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int r = (int)(i % R);
  const int64_t eb = i / R;
  const int b = (int)(eb % CB);
  const int64_t e = eb / CB;
  dst[i] = src[((size_t)e * R + r) * CB + b];
}

}  // namespace

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               int32_t* hist, int32_t* user_idx, float* user_w, int* err,
                               cudaStream_t st) {
  (void)err;
  router_topk_kernel<<<(T + 127) / 128, 128, 0, st>>>(logits, T, E, k, idx, w, hist, user_idx,
                                                      user_w);
  return cudaGetLastError();
}

cudaError_t launch_build_perm(const int32_t* idx, int A, int E, const int32_t* hist, int32_t* off,
                              int32_t* perm, int32_t* inv, int* err, cudaStream_t st) {
  build_perm_kernel<<<E, 1024, 0, st>>>(idx, A, E, hist, off, perm, inv, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* src, int H, int k, const int32_t* perm, int A,
                               uint16_t* dst, const int32_t* off, int E, const uint16_t* bias,
                               float* dot_out, cudaStream_t st) {
  const int threads = 256;
  const long long blocks = ((long long)A * 32 + threads - 1) / threads;
  gather_rows_kernel<<<(unsigned)blocks, threads, 0, st>>>(src, H, k, perm, A, dst, off, E, bias,
                                                           dot_out);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* slots, int T, int k, int H, uint16_t* out,
                           cudaStream_t st) {
  const size_t n = (size_t)T * (H / 8);
  combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(slots, T, k, H, out);
  return cudaGetLastError();
}

cudaError_t launch_reduce_dw(const float* cbias, const float* dw_part, int nparts, int A,
                             const int32_t* perm, float* dw, float* d_topk_w, cudaStream_t st) {
  reduce_dw_kernel<<<(A + 255) / 256, 256, 0, st>>>(cbias, dw_part, nparts, A, perm, dw, d_topk_w);
  return cudaGetLastError();
}

cudaError_t launch_router_backward(const int32_t* idx, const float* w, const float* d_topk_w,
                                   int T, int E, int k, float* d_logits, cudaStream_t st) {
  if (!d_logits) return cudaSuccess;
  router_backward_kernel<<<(T + 127) / 128, 128, 0, st>>>(idx, w, d_topk_w, T, E, k, d_logits);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                           uint16_t* out, cudaStream_t st) {
  const int64_t nw = rows * (K / 8);  // 32-bit words of codes
  if (nw == 0) return cudaSuccess;
  dequant_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(blocks, scales, nw, out);
  return cudaGetLastError();
}

// Stacked gate_up rows (gate j at row j, up j at row I + j) to the interleaved order (gate j
// at row 2j, up j at row 2j + 1): one block per output row copies its packed bytes (16 bytes
// per thread step), its scale bytes and its bias.
__global__ void interleave_rows_kernel(const uint8_t* __restrict__ sb, const uint8_t* __restrict__ ss,
                                       const uint16_t* __restrict__ sbias, int I, int K,
                                       uint8_t* __restrict__ db, uint8_t* __restrict__ ds,
                                       uint16_t* __restrict__ dbias) {
  const int e = blockIdx.y;
  const int r = blockIdx.x;              // output row in [0, 2I)
  const int src = (r & 1) ? I + (r >> 1) : (r >> 1);
  const size_t orow = (size_t)e * 2 * I + r, irow = (size_t)e * 2 * I + src;
  const int nb = K / 2, ns = K / 32;     // packed bytes and scales per row
  const uint4* bi = reinterpret_cast<const uint4*>(sb + irow * nb);
  uint4* bo = reinterpret_cast<uint4*>(db + orow * nb);
  for (int i = threadIdx.x; i < nb / 16; i += blockDim.x) bo[i] = bi[i];
  for (int i = threadIdx.x; i < ns; i += blockDim.x) ds[orow * ns + i] = ss[irow * ns + i];
  if (threadIdx.x == 0) dbias[orow] = sbias[irow];
}

cudaError_t launch_interleave_gate_up(const uint8_t* sb, const uint8_t* ss, const uint16_t* sbias,
                                      int E, int I, int K, uint8_t* db, uint8_t* ds,
                                      uint16_t* dbias, cudaStream_t st) {
  dim3 grid(2 * I, E);
  interleave_rows_kernel<<<grid, 64, 0, st>>>(sb, ss, sbias, I, K, db, ds, dbias);
  return cudaGetLastError();
}

cudaError_t launch_transpose_packed(const uint8_t* src, int E, int R, int C, uint8_t* dst,
                                    cudaStream_t st) {
  dim3 grid(C / 32, R / 32, E);
  transpose_packed_kernel<<<grid, 32, 0, st>>>(src, R, C, dst);
  return cudaGetLastError();
}

cudaError_t launch_transpose_scales(const uint8_t* src, int E, int R, int C, uint8_t* dst,
                                    cudaStream_t st) {
  const int64_t total = (int64_t)E * R * (C / 32);
  transpose_scales_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(src, R, C / 32, dst,
                                                                          total);
  return cudaGetLastError();
}

}  // namespace moe
