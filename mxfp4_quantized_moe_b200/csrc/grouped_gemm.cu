// Persistent grouped GEMM over expert-sorted token rows with MXFP4 weights dequantized
// straight into tensor memory (sm_100a, tcgen05).
//
// For expert e with rows [off[e], off[e+1]) of the expert-sorted token matrix X (bf16,
// [A][K]) and packed weights W[e] ([N][K], MXFP4), each tile computes
//     D^T[n, r] = sum_k W[e][n, k] * X[r, k]
// for 128 output features n (the MMA's M side) and up to kBN token rows r (its N side).
//
// Why this shape: the dequantized weights never touch shared memory.  Converter warps read
// the packed tile (TMA -> smem, 0.53 B/element), expand it to bf16 in registers and write
// it to tensor memory with tcgen05.st, where tcgen05.mma reads it as the A operand
// (A-from-TMEM form).  Shared memory carries only the token tile (TMA, 128B swizzle, B
// operand) and the packed bytes, so its bandwidth goes to the MMA, not to the converter.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: token tile + packed weight tile per k-step, scales per tile
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2-5   converters: packed MXFP4 -> bf16 -> TMEM (one TMEM lane quarter each)
//   warps 6-9   epilogue: TMEM -> registers -> fused bias / GLU / routing / scatter
// TMEM (512 columns): two fp32 accumulators of kBN columns (double buffered across tiles)
// and a 4-stage ring of A operands (32 columns = 64 bf16 of K each).
//
// Which weights: the forward GEMMs read the stored rows (scales per row and 32-element
// block of K).  The backward GEMMs contract over the stored rows' output axis, so they
// read the transposed copy (element (n, k) of W^T); there the 32-element scale blocks run
// along n, and the scale of element (n, k) is scales_t[n/32][k].
//
// Sources: "Integrate finegrained kernels: SOTA performance and per-module quantization"
// (commits on the gate|up row interleave and on the per-expert bias operand, which the
// epilogue indexes by the tile's expert id); "Add MXFP4 training support via a
// dequantize-on-the-fly fallback" (section "What this does": the expert math over weights
// dequantized on the fly; section "Relation to the backward triton kernels": input
// gradients through the frozen weights, no weight gradient).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kStages = 4;        // token + packed-weight ring depth
constexpr int kAStages = 4;       // TMEM A ring depth
constexpr int kThreads = 320;
constexpr int kTokBytes = kBN * kBK * 2;      // 24 KB
constexpr int kWBytes = kBM * (kBK / 2);      // 4 KB of packed nibbles
constexpr int kAccCols = kBN;                 // fp32 accumulator columns per buffer
constexpr int kACol0 = 2 * kAccCols;          // first TMEM column of the A ring
constexpr int kTmemCols = 512;
static_assert(kACol0 + kAStages * (kBK / 2) <= kTmemCols, "TMEM budget");
static_assert(kBN % 32 == 0 && kBN <= 256, "token tile");

constexpr unsigned kFull = 0xFFFFFFFFu;

struct __align__(8) Barriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t a_full[kAStages];
  uint64_t a_empty[kAStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sc_full[2];
  uint64_t sc_empty[2];
  uint64_t drain;
};

struct SmemLayout {
  // offsets from the 1024-aligned dynamic smem base
  static constexpr int tok = 0;
  static constexpr int w = tok + kStages * kTokBytes;
  static constexpr int bars = w + kStages * kWBytes;
  static constexpr int misc = bars + 256;  // tmem slot, abort flag
  static constexpr int cw = misc + 64;     // per converter warp: 2 x 2 x 32 scale words
  static constexpr int tables = cw + 4 * 2 * 2 * 32 * 4;  // off[257], tile_start[257]
  static constexpr int sc = ((tables + 2 * 257 * 4) + 127) / 128 * 128;  // 2 scale buffers
};

struct Tile {
  int e, fb, row0, n_valid, feat0;
};

__device__ __forceinline__ void decode_tile(int t, const int* s_tstart, const int* s_off, int E,
                                            int nfb, Tile& o) {
  int lo = 0, hi = E;  // s_tstart[lo] <= t < s_tstart[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  // skip experts with no tiles (equal starts)
  while (lo + 1 <= E && s_tstart[lo + 1] <= t) ++lo;
  const int local = t - s_tstart[lo];
  const int tt = local / nfb;
  o.e = lo;
  o.fb = local - tt * nfb;
  o.row0 = s_off[lo] + tt * kBN;
  o.n_valid = min(kBN, s_off[lo + 1] - o.row0);
  o.feat0 = o.fb * kBM;
}

__device__ __forceinline__ float sigmoidf_fast(float z) { return 1.f / (1.f + __expf(-z)); }

// In-register transpose-reduction: on entry v[c] is this lane's term for column c; on
// exit v[0] holds, in lane l, the sum over the 32 lanes of the terms for column l.
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, off);
    }
  }
  return v[0];
}

template <int EPI, bool COLT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_tok,
                        const __grid_constant__ CUtensorMap tmap_w, const GemmArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Barriers* bar = reinterpret_cast<Barriers*>(smem + SmemLayout::bars);
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + SmemLayout::misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 8);
  int* s_off = reinterpret_cast<int*>(smem + SmemLayout::tables);
  int* s_tstart = s_off + 257;
  const int sc_bytes = 4 * p.K;  // 128 rows x K/32 (per-row) or 4 x K (transposed)
  uint8_t* s_sc = smem + SmemLayout::sc;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DevErr err{p.err};
  const int E = p.E, K = p.K, N = p.N;
  const int nk = (K + kBK - 1) / kBK;
  const int nfb = (N + kBM - 1) / kBM;
  const int kb32 = K / 32;  // scale blocks per row

  // ---- set-up: expert offsets and tile starts, barriers, TMEM ----------------------
  for (int i = threadIdx.x; i <= E; i += kThreads) s_off[i] = p.off[i];
  if (threadIdx.x == 0) {
    *s_abort = 0;
    mbar_init(smem_u32(&bar->drain), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bar->full[s]), 1);
      mbar_init(smem_u32(&bar->empty[s]), 1 + 4);  // MMA commit + 4 converter warps
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(smem_u32(&bar->a_full[s]), 4);
      mbar_init(smem_u32(&bar->a_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar->acc_full[s]), 1);
      mbar_init(smem_u32(&bar->acc_empty[s]), 4);
      mbar_init(smem_u32(&bar->sc_full[s]), 1);
      mbar_init(smem_u32(&bar->sc_empty[s]), 4);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)s_tmem), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      s_tstart[e] = acc;
      const int m = s_off[e + 1] - s_off[e];
      acc += ((m + kBN - 1) / kBN) * nfb;
    }
    s_tstart[E] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int total = s_tstart[E];

  if (warp == 0) {
    // ================================ TMA producer ==================================
    int issued = 0, sc_issued = 0;
    if (lane == 0) {
      prefetch_tmap(&tmap_tok);
      prefetch_tmap(&tmap_w);
      int s = 0;
      uint32_t ph = 0;
      int lt = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
        Tile tl;
        decode_tile(t, s_tstart, s_off, E, nfb, tl);
        const int rows = min(kBM, N - tl.feat0);
        const int sb = lt & 1;
        if (!mbar_wait(smem_u32(&bar->sc_empty[sb]), ((lt >> 1) & 1) ^ 1, err, 0x200, s_abort)) break;
        uint32_t bytes;
        const uint8_t* src;
        if (COLT) {
          bytes = (uint32_t)(rows / 32) * K;
          src = p.scales + ((size_t)tl.e * (N / 32) + tl.feat0 / 32) * K;
        } else {
          bytes = (uint32_t)rows * kb32;
          src = p.scales + ((size_t)tl.e * N + tl.feat0) * kb32;
        }
        mbar_arrive_expect_tx(smem_u32(&bar->sc_full[sb]), bytes);
        bulk_load(smem_u32(s_sc + sb * sc_bytes), src, bytes, smem_u32(&bar->sc_full[sb]));
        ++sc_issued;
        bool ok = true;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(smem_u32(&bar->empty[s]), ph ^ 1, err, 0x201, s_abort)) { ok = false; break; }
          const uint32_t fb = smem_u32(&bar->full[s]);
          mbar_arrive_expect_tx(fb, kTokBytes + kWBytes);
          tma_load_2d(smem_u32(smem + SmemLayout::tok + s * kTokBytes), &tmap_tok, ks * kBK,
                      tl.row0, fb);
          tma_load_2d(smem_u32(smem + SmemLayout::w + s * kWBytes), &tmap_w, ks * (kBK / 2),
                      tl.e * N + tl.feat0, fb);
          ++issued;
          if (++s == kStages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
    }
    __syncwarp();
    // Drain: wait until every copy issued into a stage has landed before the CTA exits.
    __syncthreads();
    if (lane == 0) {
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int last = s + kStages * ((issued - 1 - s) / kStages);
        mbar_wait(smem_u32(&bar->full[s]), (last / kStages) & 1, err, 0x2F0, nullptr);
      }
      for (int sb = 0; sb < 2 && sb < sc_issued; ++sb) {
        const int last = sb + 2 * ((sc_issued - 1 - sb) / 2);
        mbar_wait(smem_u32(&bar->sc_full[sb]), (last / 2) & 1, err, 0x2F1, nullptr);
      }
    }
  } else if (warp == 1) {
    // ================================ MMA issuer ====================================
    if (lane == 0) {
      int s = 0, sa = 0;
      uint32_t ph = 0, aph = 0;
      int lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        Tile tl;
        decode_tile(t, s_tstart, s_off, E, nfb, tl);
        const int acc = lt & 1;
        if (!mbar_wait(smem_u32(&bar->acc_empty[acc]), ((lt >> 1) & 1) ^ 1, err, 0x300, s_abort)) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_m128((tl.n_valid + 15) & ~15);
        const uint32_t d_tmem = tmem + acc * kAccCols;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(smem_u32(&bar->full[s]), ph, err, 0x301, s_abort) ||
              !mbar_wait(smem_u32(&bar->a_full[sa]), aph, err, 0x302, s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc =
              smem_desc_kmajor_sw128(smem_u32(smem + SmemLayout::tok + s * kTokBytes));
          const uint32_t a_tmem = tmem + kACol0 + sa * (kBK / 2);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ts(d_tmem, a_tmem + kk * 8, bdesc + (uint64_t)(kk * 2), idesc,
                        (ks | kk) != 0);
          mma_commit(smem_u32(&bar->empty[s]));
          mma_commit(smem_u32(&bar->a_empty[sa]));
          if (++s == kStages) { s = 0; ph ^= 1; }
          if (++sa == kAStages) { sa = 0; aph ^= 1; }
        }
        if (ok) mma_commit(smem_u32(&bar->acc_full[acc]));
      }
      // every MMA issued by this thread has completed once `drain` flips
      mma_commit(smem_u32(&bar->drain));
      mbar_wait(smem_u32(&bar->drain), 0, err, 0x3F0, nullptr);
    }
    __syncwarp();
    __syncthreads();
  } else if (warp < 6) {
    // ================================ converters ====================================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t* cw = reinterpret_cast<uint32_t*>(smem + SmemLayout::cw) + (warp - 2) * 128;
    int s = 0, sa = 0;
    uint32_t ph = 0, aph = 0;
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
      Tile tl;
      decode_tile(t, s_tstart, s_off, E, nfb, tl);
      const bool active = tl.feat0 + 32 * q < N;  // warp-uniform: N % 32 == 0
      const int sb = lt & 1;
      if (!mbar_wait(smem_u32(&bar->sc_full[sb]), (lt >> 1) & 1, err, 0x400, s_abort)) break;
      const uint8_t* scb = s_sc + sb * sc_bytes;
      const int r = 32 * q + lane;  // row of the 128-row weight tile
      for (int ks = 0; ks < nk; ++ks) {
        if (!mbar_wait(smem_u32(&bar->full[s]), ph, err, 0x401, s_abort)) { ok = false; break; }
        uint32_t qw[8];
        {
          const uint4* wp =
              reinterpret_cast<const uint4*>(smem + SmemLayout::w + s * kWBytes + r * (kBK / 2));
          const uint4 w0 = wp[0], w1 = wp[1];
          qw[0] = w0.x; qw[1] = w0.y; qw[2] = w0.z; qw[3] = w0.w;
          qw[4] = w1.x; qw[5] = w1.y; qw[6] = w1.z; qw[7] = w1.w;
        }
        // scale factors: f1 (and f2 when some scale is above 128), as bf16x2 words
        uint32_t f1a, f1b, f2a = 0x3F803F80u, f2b = 0x3F803F80u;
        bool slow;
        if (!COLT) {
          const uint32_t sa_ = active ? scb[r * kb32 + 2 * ks] : 127u;
          const uint32_t sb_ = (active && 2 * ks + 1 < kb32) ? scb[r * kb32 + 2 * ks + 1] : 127u;
          f1a = dup16(ue8m0_f1(sa_));
          f1b = dup16(ue8m0_f1(sb_));
          slow = __any_sync(kFull, (sa_ > 128u) | (sb_ > 128u));
          if (slow) {
            f2a = dup16(ue8m0_f2(sa_));
            f2b = dup16(ue8m0_f2(sb_));
          }
        } else {
          // lane l computes the factors of K elements 2l, 2l+1 of this k-step; the
          // warp shares them through shared memory (same scale row for all 32 lanes).
          const int k0 = ks * kBK + 2 * lane;
          uint32_t s0 = 127u, s1 = 127u;
          if (active && k0 < K) {
            s0 = scb[q * K + k0];
            s1 = (k0 + 1 < K) ? scb[q * K + k0 + 1] : 127u;
          }
          slow = __any_sync(kFull, (s0 > 128u) | (s1 > 128u));
          uint32_t* cwb = cw + (ks & 1) * 64;
          cwb[lane] = ue8m0_f1(s0) | (ue8m0_f1(s1) << 16);
          if (slow) cwb[32 + lane] = ue8m0_f2(s0) | (ue8m0_f2(s1) << 16);
          f1a = f1b = 0;
        }
        // the packed bytes are in registers: release the stage's weight half
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->empty[s]));

        uint32_t out[32];
        if (active) {
          if (!COLT) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t pt[4];
              e2m1x8_to_bf16x2_pattern(qw[i], pt);
              const uint32_t f1 = i < 4 ? f1a : f1b;
#pragma unroll
              for (int m = 0; m < 4; ++m) out[4 * i + m] = bmul2(pt[m], f1);
            }
            if (slow) {
#pragma unroll
              for (int m = 0; m < 32; ++m) out[m] = bmul2(out[m], m < 16 ? f2a : f2b);
            }
          } else {
            const uint32_t* cwb = cw + (ks & 1) * 64;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              uint32_t pt[4];
              e2m1x8_to_bf16x2_pattern(qw[i], pt);
              const uint4 f = *reinterpret_cast<const uint4*>(cwb + 4 * i);
              out[4 * i + 0] = bmul2(pt[0], f.x);
              out[4 * i + 1] = bmul2(pt[1], f.y);
              out[4 * i + 2] = bmul2(pt[2], f.z);
              out[4 * i + 3] = bmul2(pt[3], f.w);
            }
            if (slow) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint4 f = *reinterpret_cast<const uint4*>(cwb + 32 + 4 * i);
                out[4 * i + 0] = bmul2(out[4 * i + 0], f.x);
                out[4 * i + 1] = bmul2(out[4 * i + 1], f.y);
                out[4 * i + 2] = bmul2(out[4 * i + 2], f.z);
                out[4 * i + 3] = bmul2(out[4 * i + 3], f.w);
              }
            }
          }
        }
        if (!mbar_wait(smem_u32(&bar->a_empty[sa]), aph ^ 1, err, 0x402, s_abort)) { ok = false; break; }
        tc_fence_after();
        if (active) {
          tmem_st32(tmem + ((uint32_t)(32 * q) << 16) + kACol0 + sa * (kBK / 2), out);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->a_full[sa]));
        if (++s == kStages) { s = 0; ph ^= 1; }
        if (++sa == kAStages) { sa = 0; aph ^= 1; }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->sc_empty[sb]));
    }
    __syncwarp();
    __syncthreads();
  } else {
    // ================================ epilogue ======================================
    const int q = warp & 3;
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      Tile tl;
      decode_tile(t, s_tstart, s_off, E, nfb, tl);
      const int acc = lt & 1;
      if (!mbar_wait(smem_u32(&bar->acc_full[acc]), (lt >> 1) & 1, err, 0x500, s_abort)) break;
      tc_fence_after();
      const int f = tl.feat0 + 32 * q + lane;  // output feature of this thread
      const bool active = tl.feat0 + 32 * q < N;
      float bias_f = 0.f;
      if ((EPI == kEpiGateUp || EPI == kEpiDown) && active)
        bias_f = bf16_to_f(p.bias[(size_t)tl.e * N + f]);
      for (int c0 = 0; c0 < tl.n_valid; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + acc * kAccCols + c0, r);
        tmem_wait_ld();
        if (!active) continue;
        const int ncol = min(32, tl.n_valid - c0);
        const int rbase = tl.row0 + c0;
        if (EPI == kEpiGateUp) {
          // h = acc + bias (interleaved: even f = gate, odd f = up); act from the pair
          const int I = N >> 1;
          const bool gate = (lane & 1) == 0;
          const int jf = f >> 1;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float v0 = __uint_as_float(r[j]) + bias_f;
            const float v1 = __uint_as_float(r[j + 1]) + bias_f;
            if (j < ncol) p.out0[(size_t)(rbase + j) * N + f] = f_to_bf16(v0);
            if (j + 1 < ncol) p.out0[(size_t)(rbase + j + 1) * N + f] = f_to_bf16(v1);
            const float recv = __shfl_xor_sync(kFull, gate ? v1 : v0, 1);
            const float g = gate ? v0 : recv;
            const float u = gate ? recv : v1;
            const int col = j + (gate ? 0 : 1);
            const float gc = fminf(g, p.limit);
            const float uc = fminf(fmaxf(u, -p.limit), p.limit);
            const float a = (uc + 1.f) * gc * sigmoidf_fast(p.alpha * gc);
            if (col < ncol) p.out1[(size_t)(rbase + col) * I + jf] = f_to_bf16(a);
          }
        } else {
          int my_slot = 0;
          float my_w = 0.f;
          if (lane < ncol) {
            my_slot = p.perm[rbase + lane];
            if (EPI == kEpiDown || EPI == kEpiDact) my_w = p.topk_w[my_slot];
          }
          if (EPI == kEpiDown || EPI == kEpiDx) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int slot = __shfl_sync(kFull, my_slot, j);
              float v = __uint_as_float(r[j]);
              if (EPI == kEpiDown) v = __shfl_sync(kFull, my_w, j) * (v + bias_f);
              if (j < ncol) p.out0[(size_t)slot * N + f] = f_to_bf16(v);
            }
          } else {  // kEpiDact
            const int I = N;
            float part[32];
            const uint32_t* hw = reinterpret_cast<const uint32_t*>(p.hsaved);
            uint32_t* dh = reinterpret_cast<uint32_t*>(p.out0);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float wr = __shfl_sync(kFull, my_w, j);
              part[j] = 0.f;
              if (j < ncol) {
                const uint32_t hv = hw[(size_t)(rbase + j) * I + f];
                const float g = bf16_lo(hv), u = bf16_hi(hv);
                const float dz = __uint_as_float(r[j]);
                const float gc = fminf(g, p.limit);
                const float uc = fminf(fmaxf(u, -p.limit), p.limit);
                const float sg = sigmoidf_fast(p.alpha * gc);
                part[j] = dz * ((uc + 1.f) * gc * sg);
                const float dact = wr * dz;
                const float dg = (g <= p.limit)
                                     ? dact * (uc + 1.f) * (sg + p.alpha * gc * sg * (1.f - sg))
                                     : 0.f;
                const float du = (u >= -p.limit && u <= p.limit) ? dact * gc * sg : 0.f;
                dh[(size_t)(rbase + j) * I + f] = pack_bf16x2(dg, du);
              }
            }
            const float sum = warp_transpose_reduce(part, lane);
            if (lane < ncol) p.dw_part[(size_t)((tl.feat0 >> 5) + q) * p.A + rbase + lane] = sum;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->acc_empty[acc]));
    }
    __syncwarp();
    __syncthreads();
  }

  // ---- teardown: every role has left its loop and drained its async copies / MMAs ----
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

template <int EPI, bool COLT>
cudaError_t launch_one(const CUtensorMap& tt, const CUtensorMap& tw, const GemmArgs& a, int grid,
                       size_t smem, cudaStream_t st) {
  auto kern = grouped_gemm_kernel<EPI, COLT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(tt, tw, a);
  return cudaGetLastError();
}

}  // namespace

size_t grouped_gemm_smem_bytes(int K) {
  return 1024 + SmemLayout::sc + 2 * (size_t)(4 * K);
}

cudaError_t launch_grouped_gemm(int epi, bool transposed_scales, const uint16_t* tokens,
                                const uint8_t* wq, const GemmArgs& a, int num_sms,
                                cudaStream_t st) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tt, tw;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.A};
    const cuuint64_t strides[1] = {(cuuint64_t)a.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(tokens), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(a.K / 2), (cuuint64_t)a.E * (cuuint64_t)a.N};
    const cuuint64_t strides[1] = {(cuuint64_t)(a.K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kBK / 2), (cuuint32_t)kBM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(wq), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = grouped_gemm_smem_bytes(a.K);
  const int grid = num_sms;
  switch (epi * 2 + (transposed_scales ? 1 : 0)) {
    case kEpiGateUp * 2 + 0: return launch_one<kEpiGateUp, false>(tt, tw, a, grid, smem, st);
    case kEpiDown * 2 + 0: return launch_one<kEpiDown, false>(tt, tw, a, grid, smem, st);
    case kEpiDact * 2 + 1: return launch_one<kEpiDact, true>(tt, tw, a, grid, smem, st);
    case kEpiDx * 2 + 1: return launch_one<kEpiDx, true>(tt, tw, a, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
