// Routing, permutation, gather/combine, routing backward, standalone dequant and the
// one-time weight transpose.  All of these are memory- or latency-bound; the grouped
// GEMMs live in grouped_gemm.cu.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "aux_kernels.h"

namespace moe {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------------------------------
// Router: top-k over the E logits of a token (largest first, equal logits -> lower expert
// index) and softmax over the k selected.  One warp per token, one block per 32-token
// segment.  Lane l holds logits l, l+32, ... (NG = ceil(E/32) of them) as order-preserving
// 32-bit keys; each of the k rounds takes the lane's best remaining key, the warp's largest
// key (one redux.sync) and the lowest expert index among the lanes holding it (a second).
// NaN logits never win (they rank as -inf), and -0 ranks with +0.  Lane j keeps selection j
// and counts it in the segment's expert histogram in shared memory, which the block stores as
// row t / 32 of `hist`; the segment scan and the permutation kernel place every segment's
// slots from these rows without another pass over the routing.
// Source: the top-k router of the eager expert loop ("Add MXFP4 training support via a
// dequantize-on-the-fly fallback", section "What this does"); softmax over the k values.
// ---------------------------------------------------------------------------------------
constexpr int kRouteTokens = 32;                  // tokens per histogram segment
constexpr int kRouteThreads = 32 * kRouteTokens;  // one warp per token
constexpr int kPermThreads = 256;                 // permutation block (one segment)
constexpr int kScanThreads = 512;                 // segment scan (one expert column)

// float -> unsigned key with the same order (x assumed not NaN); the inverse below
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int NG>
__global__ void __launch_bounds__(kRouteThreads) router_topk_kernel(
    const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ idx,
    float* __restrict__ w, int32_t* __restrict__ hist, int32_t* __restrict__ user_idx,
    float* __restrict__ user_w) {
  __shared__ int s_hist[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < E; e += kRouteThreads) s_hist[e] = 0;
  __syncthreads();
  const int seg = blockIdx.x;
  const int t = seg * kRouteTokens + warp;
  if (t < T) {  // warp-uniform
    const float* row = logits + (size_t)t * E;
    uint32_t key[NG];  // 0: absent or already selected (every present logit's key is larger)
#pragma unroll
    for (int i = 0; i < NG; ++i) {
      const int e = lane + 32 * i;
      float x = (e < E) ? __ldg(row + e) : 0.f;
      x = (x != x) ? -INFINITY : x + 0.f;  // NaN ranks as -inf; -0 + 0 = +0
      key[i] = (e < E) ? order_key(x) : 0u;
    }
    float m0 = 0.f, zsum = 0.f;
    float myz = 0.f;  // selection `lane` (k <= 32); lane j % 32 parks selections j >= 32 in
    int myi = 0;      // idx / w until the softmax denominator is known
    for (int j = 0; j < k; ++j) {
      uint32_t hk = 0;
      int hi = 0x7FFFFFFF;
#pragma unroll
      for (int i = 0; i < NG; ++i)  // strictly larger: the lower expert wins a tie
        if (key[i] > hk) {
          hk = key[i];
          hi = lane + 32 * i;
        }
      const uint32_t mk = __reduce_max_sync(kFull, hk);
      const int bi = (int)__reduce_min_sync(kFull, hk == mk ? (uint32_t)hi : 0x7FFFFFFFu);
      if ((bi & 31) == lane) {
#pragma unroll
        for (int i = 0; i < NG; ++i)
          if (i == (bi >> 5)) key[i] = 0u;
      }
      const float bv = key_value(mk);
      if (j == 0) m0 = bv;
      const float z = __expf(bv - m0);
      zsum += z;
      if (lane == (j & 31)) {
        if (j < 32) {
          myz = z;
          myi = bi;
        } else {
          w[(size_t)t * k + j] = z;
          idx[(size_t)t * k + j] = bi;
        }
      }
    }
    const float inv = 1.f / zsum;
    for (int j = lane; j < k; j += 32) {
      const size_t o = (size_t)t * k + j;
      const float z = (j < 32) ? myz : w[o];
      const int e = (j < 32) ? myi : idx[o];
      const float wj = z * inv;
      idx[o] = e;
      w[o] = wj;
      if (user_idx) user_idx[o] = e;
      if (user_w) user_w[o] = wj;
      atomicAdd(s_hist + e, 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kRouteThreads) hist[(size_t)seg * E + e] = s_hist[e];
}

// Exclusive scan of one expert's column of the segment histograms (block e):
// seg_pre[s][e] = sum of hist[s'][e] over s' < s, tot[e] = the column's sum.
__global__ void __launch_bounds__(kScanThreads) seg_scan_kernel(
    const int32_t* __restrict__ hist, int nseg, int E, int32_t* __restrict__ seg_pre,
    int32_t* __restrict__ tot) {
  __shared__ int s_warp[kScanThreads / 32];
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int carry = 0;
  for (int c = 0; c < nseg; c += kScanThreads) {
    const int s = c + threadIdx.x;
    const int v = s < nseg ? __ldg(hist + (size_t)s * E + e) : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int wbase = 0, chunk = 0;
    for (int i = 0; i < kScanThreads / 32; ++i) {
      const int x = s_warp[i];
      wbase += (i < warp) ? x : 0;
      chunk += x;
    }
    if (s < nseg) seg_pre[(size_t)s * E + e] = carry + wbase + incl - v;
    carry += chunk;
    __syncthreads();  // s_warp is rewritten by the next chunk
  }
  if (threadIdx.x == 0) tot[e] = carry;
}

// ---------------------------------------------------------------------------------------
// Stable counting sort of the A = T*k slots by expert, one block per routing segment.  The
// expert offsets off[e] are the exclusive scan of the column sums over the experts; the
// segment's first expert-e row is off[e] + seg_pre[b][e].  The block's slots are then ranked
// in slot order: each warp counts a contiguous share of them per expert (warp-level match on
// the expert id), a scan over the warps gives each share's first row, and a second pass
// assigns the rows.  perm[row] = slot, inv[slot] = row, w_row[row] = w[slot]; block 0
// publishes off[0..E].
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kPermThreads) build_perm_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, int A, int E, int k,
    const int32_t* __restrict__ seg_pre, const int32_t* __restrict__ tot,
    int32_t* __restrict__ off, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    float* __restrict__ w_row, int* err) {
  constexpr int kWarps = kPermThreads / 32;
  static_assert(kPermThreads >= 256, "one thread per expert (E <= 256)");
  __shared__ int s_cnt[kWarps][256];
  __shared__ int s_tot[256];
  __shared__ int s_scan[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int e = threadIdx.x;
  const int total = (e < E) ? __ldg(tot + e) : 0;
  // exclusive scan of the totals over experts (E <= 256 = one value per thread)
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int i = 0; i < warp; ++i) wbase += s_scan[i];
  const int off_e = wbase + incl - total;
  if (e < E) s_tot[e] = off_e + __ldg(seg_pre + (size_t)b * E + e);  // first row of this block's expert-e slots
  if (b == 0) {
    if (e < E) off[e] = off_e;
    if (e == E - 1) {
      off[E] = off_e + total;
      if (off_e + total != A) DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x100);
    }
  }
  // this block's slots, split into kWarps contiguous shares of whole 32-slot steps
  const int s0 = b * kRouteTokens * k, s1 = min(A, s0 + kRouteTokens * k);
  const int steps = (s1 - s0 + 31) / 32;
  const int per = (steps + kWarps - 1) / kWarps;
  const int w0 = s0 + 32 * min(steps, warp * per), w1 = min(s1, s0 + 32 * min(steps, (warp + 1) * per));
  for (int i = lane; i < E; i += 32) s_cnt[warp][i] = 0;
  __syncwarp();
  for (int c = w0; c < w1; c += 32) {  // pass 1: per-warp counts
    const int slot = c + lane;
    const int ex = slot < w1 ? idx[slot] : -1;
    const unsigned m = __match_any_sync(kFull, ex);
    if (ex >= 0 && lane == 31 - __clz(m)) s_cnt[warp][ex] += __popc(m);
    __syncwarp();
  }
  __syncthreads();
  if (e < E) {  // scan over the warps' shares
    int run = s_tot[e];
    for (int i = 0; i < kWarps; ++i) {
      const int c = s_cnt[i][e];
      s_cnt[i][e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int c = w0; c < w1; c += 32) {  // pass 2: rows in slot order
    const int slot = c + lane;
    const int ex = slot < w1 ? idx[slot] : -1;
    const unsigned m = __match_any_sync(kFull, ex);
    if (ex >= 0) {
      const int row = s_cnt[warp][ex] + __popc(m & ((1u << lane) - 1u));
      if (row < A) {
        perm[row] = slot;
        inv[slot] = row;
        w_row[row] = w[slot];
      } else {
        DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x101);
      }
    }
    __syncwarp();
    if (ex >= 0 && lane == 31 - __clz(m)) s_cnt[warp][ex] += __popc(m);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------------------
// dst[r] = src[perm[r] / k] for every expert-sorted row r (one warp per row, 16-byte
// vectors).  With `dot_w` (the backward's gather of dY), the row of `dst` first holds the
// forward's expert output y_r (unweighted, bias included), read in place before it is
// overwritten: dot_w[perm[r]] = <dY_t, y_r> in fp32, the routing-weight gradient.  Each lane
// reads a 16-byte chunk of y_r and then writes the same chunk, and no other lane or warp
// touches that chunk, so reading and writing one buffer is safe.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16x8_dot(const uint4& a, const uint4& b) {
  float acc = bf16_lo(a.x) * bf16_lo(b.x) + bf16_hi(a.x) * bf16_hi(b.x);
  acc += bf16_lo(a.y) * bf16_lo(b.y) + bf16_hi(a.y) * bf16_hi(b.y);
  acc += bf16_lo(a.z) * bf16_lo(b.z) + bf16_hi(a.z) * bf16_hi(b.z);
  acc += bf16_lo(a.w) * bf16_lo(b.w) + bf16_hi(a.w) * bf16_hi(b.w);
  return acc;
}

__global__ void gather_rows_kernel(const uint16_t* __restrict__ src, int H, int k,
                                   const int32_t* __restrict__ perm, int A, uint16_t* dst,
                                   float* __restrict__ dot_w, int* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= A) return;
  const int row = warp;
  const int slot = perm[row];
  if (MXFP4_MOE_DEBUG && (slot < 0 || slot >= A)) {  // warp-uniform
    if (lane == 0) DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x110);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(slot / k) * H);
  uint4* d = reinterpret_cast<uint4*>(dst + (size_t)row * H);
  const int nv = H / 8;
  float acc = 0.f;
  // four 16-byte chunks per lane in flight: all loads of a group are issued before its stores
  // (the chunks are distinct, so reading y and writing dY in place keeps its order per chunk)
  constexpr int kG = 4;
  for (int i0 = lane; i0 < nv; i0 += 32 * kG) {
    uint4 v[kG], y[kG];
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int i = i0 + 32 * g;
      if (i < nv) {
        v[g] = __ldg(s + i);
        if (dot_w) y[g] = d[i];
      }
    }
#pragma unroll
    for (int g = 0; g < kG; ++g) {
      const int i = i0 + 32 * g;
      if (i < nv) {
        if (dot_w) acc += bf16x8_dot(v[g], y[g]);
        d[i] = v[g];
      }
    }
  }
  if (dot_w) {
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) dot_w[slot] = acc;
  }
}

// ---------------------------------------------------------------------------------------
// Gather with the split into two E4M3 parts that the block-scaled gate_up GEMM consumes.
// For every expert-sorted row r (token t = perm[r] / k) and 32-element block b of x[t]:
//   S  = the smallest integer with max|x_block| <= 448 * 2^S (clamped to [-126, 121]),
//   hi = e4m3(x / 2^S), lo = e4m3(x / 2^S - hi)   (round to nearest even, exact residual),
//   sfb[r][b] = S + 127: the UE8M0 scale 2^S the MMA applies to both parts.
// x / 2^S has at most 8 significant bits; hi keeps the top 4 and lo the next 4 (the remainder
// is exact in fp32), so hi + lo equals x / 2^S for every element within 2^9 of the block
// maximum that stays above the E4M3 subnormal floor; smaller elements keep an absolute error
// below 2^-10 * 2^S.  A block holding inf or NaN gets the NaN scale (255).  Bytes of sfb past
// the row's H/32 blocks are zero.  One warp per row; a lane takes whole blocks (64 bytes of
// x in, 32 bytes of hi and of lo out).
// Source: "Integrate finegrained kernels: SOTA performance and per-module quantization", the
// commits on the activation format and input recipe (MX activations with UE8M0 block scales
// feeding block-scaled tensor-core GEMMs).
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float a_lo, float a_hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(a_hi), "f"(a_lo));
  return d;
}
__device__ __forceinline__ void f32x2_from_e4m3x2(uint32_t v, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "h"((uint16_t)v));
  __half2 hh = *reinterpret_cast<__half2*>(&h2);
  lo = __low2float(hh);
  hi = __high2float(hh);
}

__global__ void gather_quant_kernel(const uint16_t* __restrict__ x, int H, int k,
                                    const int32_t* __restrict__ perm, int A,
                                    uint8_t* __restrict__ hi, uint8_t* __restrict__ lo,
                                    uint8_t* __restrict__ sfb, int sfb_stride, int* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= A) return;
  const int row = warp;
  if (MXFP4_MOE_DEBUG && (perm[row] < 0 || perm[row] >= A)) {  // warp-uniform
    if (lane == 0) DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x111);
    return;
  }
  const int t = perm[row] / k;
  const int nb = H / 32;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  // scale byte b of the row lives in 32-bit word (b / 4) ^ ((row / 4) % 8), byte b % 4: the
  // GEMM's converter lanes read one word of 32 consecutive rows and so hit 32 different banks
  // (the stride is a multiple of 32 bytes, so the exchange stays inside the row)
  uint8_t* srow = sfb + (size_t)row * sfb_stride;
  const int rsw = (row >> 2) & 7;
  for (int b = lane; b < sfb_stride; b += 32) {
    const int pos = 4 * ((b >> 2) ^ rsw) + (b & 3);
    if (b >= nb) {
      srow[pos] = 0;
      continue;
    }
    uint32_t v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = __ldg(src + 4 * b + i);
      v[4 * i + 0] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
    }
    uint32_t amax = 0;  // largest bf16 magnitude pattern (ordered like the magnitudes)
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = max(amax, max(v[i] & 0x7FFFu, (v[i] >> 16) & 0x7FFFu));
    uint32_t hw[8], lw[8];
    int sbyte;
    if (amax >= 0x7F80u) {  // inf or NaN in the block
      sbyte = 255;
#pragma unroll
      for (int i = 0; i < 8; ++i) hw[i] = lw[i] = 0;
    } else {
      const int E = (int)(amax >> 7), m7 = (int)(amax & 0x7F);
      const int S = (E == 0) ? -126 : max(-126, E - 135 + (m7 > 0x60 ? 1 : 0));
      sbyte = S + 127;
      const float inv = __uint_as_float((uint32_t)(127 - S) << 23);  // 2^-S, exact
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // elements 4i .. 4i+3
        const float y0 = bf16_lo(v[2 * i]) * inv, y1 = bf16_hi(v[2 * i]) * inv;
        const float y2 = bf16_lo(v[2 * i + 1]) * inv, y3 = bf16_hi(v[2 * i + 1]) * inv;
        const uint32_t h01 = e4m3x2_from_f32(y0, y1), h23 = e4m3x2_from_f32(y2, y3);
        float g0, g1, g2, g3;
        f32x2_from_e4m3x2(h01, g0, g1);
        f32x2_from_e4m3x2(h23, g2, g3);
        const uint32_t l01 = e4m3x2_from_f32(y0 - g0, y1 - g1), l23 = e4m3x2_from_f32(y2 - g2, y3 - g3);
        hw[i] = h01 | (h23 << 16);
        lw[i] = l01 | (l23 << 16);
      }
    }
    uint4* dh = reinterpret_cast<uint4*>(hi + (size_t)row * H + 32 * b);
    uint4* dl = reinterpret_cast<uint4*>(lo + (size_t)row * H + 32 * b);
    dh[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    dh[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    dl[0] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    dl[1] = make_uint4(lw[4], lw[5], lw[6], lw[7]);
    srow[pos] = (uint8_t)sbyte;
  }
}

// out[t] = sum_j w[t*k+j] * rows[inv[t*k+j]] in fp32 (w == nullptr: weight 1), rounded to
// bf16 once.  8 bf16 per thread.
__global__ void combine_kernel(const uint16_t* __restrict__ rows, const int32_t* __restrict__ inv,
                               const float* __restrict__ w, int T, int k, int H,
                               uint16_t* __restrict__ out, int* err) {
  const int nv = H / 8;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)T * nv) return;
  const int t = (int)(i / nv), c = (int)(i % nv);
  float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const size_t slot = (size_t)t * k + j;
    const float wj = w ? __ldg(w + slot) : 1.f;
    const int32_t r = __ldg(inv + slot);
    if (MXFP4_MOE_DEBUG && (r < 0 || r >= T * k)) {
      DevErr{err}.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x112);
      continue;
    }
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(rows + (size_t)r * H) + c);
    a[0] += wj * bf16_lo(v.x); a[1] += wj * bf16_hi(v.x);
    a[2] += wj * bf16_lo(v.y); a[3] += wj * bf16_hi(v.y);
    a[4] += wj * bf16_lo(v.z); a[5] += wj * bf16_hi(v.z);
    a[6] += wj * bf16_lo(v.w); a[7] += wj * bf16_hi(v.w);
  }
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]);
  o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]);
  o.w = pack_bf16x2(a[6], a[7]);
  reinterpret_cast<uint4*>(out + (size_t)t * H)[c] = o;
}

// d_logits through the softmax over the k selected logits:
// d_l[idx_j] = w_j (d_w_j - sum_i w_i d_w_i), 0 for the experts not selected.  One warp per
// token: the k selections are read once (lane j % 32 takes selection j), the sum is a warp
// reduction, and the row of E outputs is stored by the 32 lanes together (coalesced).
__global__ void router_backward_kernel(const int32_t* __restrict__ idx,
                                       const float* __restrict__ w,
                                       const float* __restrict__ d_topk_w, int T, int E, int k,
                                       float* __restrict__ d_logits) {
  const int lane = threadIdx.x & 31;
  const int t = (int)(((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (t >= T) return;  // warp-uniform
  const int32_t* it = idx + (size_t)t * k;
  const float* wt = w + (size_t)t * k;
  const float* dt = d_topk_w + (size_t)t * k;
  // s = sum_j w_j d_w_j over the k selections (lane j % 32 takes selection j)
  float s = 0.f;
  for (int j = lane; j < k; j += 32) s += __ldg(wt + j) * __ldg(dt + j);
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
  // lane l writes experts l, l+32, ...: the selected ones get w_j (d_w_j - s)
  float out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j0 = 0; j0 < k; j0 += 32) {
    const int j = j0 + lane;
    const int ej = j < k ? __ldg(it + j) : -1;
    const float gj = j < k ? __ldg(wt + j) * (__ldg(dt + j) - s) : 0.f;
    const int n = min(32, k - j0);
    for (int q = 0; q < n; ++q) {
      const int e = __shfl_sync(kFull, ej, q);
      const float g = __shfl_sync(kFull, gj, q);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (e == lane + 32 * i) out[i] = g;
    }
  }
  float* dl = d_logits + (size_t)t * E;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i < E) dl[lane + 32 * i] = out[i];
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

int route_blocks(int T) { return (T + kRouteTokens - 1) / kRouteTokens; }

size_t route_scratch_words(int T, int E) { return 2 * (size_t)route_blocks(T) * E + E; }

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               int32_t* scratch, int32_t* user_idx, float* user_w,
                               cudaStream_t st) {
  const int ng = (E + 31) / 32;
  auto kern = ng <= 1 ? router_topk_kernel<1> : ng <= 2 ? router_topk_kernel<2>
            : ng <= 4 ? router_topk_kernel<4> : router_topk_kernel<8>;
  kern<<<route_blocks(T), kRouteThreads, 0, st>>>(logits, T, E, k, idx, w, scratch, user_idx,
                                                   user_w);
  return cudaGetLastError();
}

cudaError_t launch_seg_scan(int T, int E, int32_t* scratch, cudaStream_t st) {
  const int nseg = route_blocks(T);
  int32_t* seg_pre = scratch + (size_t)nseg * E;
  seg_scan_kernel<<<E, kScanThreads, 0, st>>>(scratch, nseg, E, seg_pre, seg_pre + (size_t)nseg * E);
  return cudaGetLastError();
}

cudaError_t launch_build_perm(const int32_t* idx, const float* w, int T, int E, int k,
                              const int32_t* scratch, int32_t* off, int32_t* perm, int32_t* inv,
                              float* w_row, int* err, cudaStream_t st) {
  const int nseg = route_blocks(T);
  const int32_t* seg_pre = scratch + (size_t)nseg * E;
  build_perm_kernel<<<nseg, kPermThreads, 0, st>>>(idx, w, T * k, E, k, seg_pre,
                                                   seg_pre + (size_t)nseg * E, off, perm, inv,
                                                   w_row, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* src, int H, int k, const int32_t* perm, int A,
                               uint16_t* dst, float* dot_w, int* err, cudaStream_t st) {
  const int threads = 256;
  const long long blocks = ((long long)A * 32 + threads - 1) / threads;
  gather_rows_kernel<<<(unsigned)blocks, threads, 0, st>>>(src, H, k, perm, A, dst, dot_w, err);
  return cudaGetLastError();
}

cudaError_t launch_gather_quant(const uint16_t* x, int H, int k, const int32_t* perm, int A,
                                uint8_t* hi, uint8_t* lo, uint8_t* sfb, int sfb_stride,
                                int* err, cudaStream_t st) {
  const int threads = 256;
  const long long blocks = ((long long)A * 32 + threads - 1) / threads;
  gather_quant_kernel<<<(unsigned)blocks, threads, 0, st>>>(x, H, k, perm, A, hi, lo, sfb,
                                                            sfb_stride, err);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* rows, const int32_t* inv, const float* w, int T, int k,
                           int H, uint16_t* out, int* err, cudaStream_t st) {
  const size_t n = (size_t)T * (H / 8);
  combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(rows, inv, w, T, k, H, out, err);
  return cudaGetLastError();
}

cudaError_t launch_router_backward(const int32_t* idx, const float* w, const float* d_topk_w,
                                   int T, int E, int k, float* d_logits, cudaStream_t st) {
  if (!d_logits) return cudaSuccess;
  const size_t n = (size_t)T * 32;  // one warp per token
  router_backward_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(idx, w, d_topk_w, T, E, k,
                                                                     d_logits);
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
