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
// Warp roles (512 threads, registers rebalanced per warpgroup with setmaxnreg):
//   warp 0      TMA producer of the token ring (released by the MMA)
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warp 2      TMA producer of the packed-weight ring (released by the converters) and of
//               the per-tile scales
//   warps 4-11  converters: packed MXFP4 -> bf16 -> TMEM; two warps per TMEM lane quarter,
//               taking alternate k-steps
//   warps 12-15 epilogue: TMEM -> registers -> fused bias / GLU / routing / scatter
// The token and weight rings are separate so that the converters can run ahead of the MMA
// by the depth of the TMEM A ring without pinning token stages.
// TMEM (512 columns): one fp32 accumulator of kBN = 256 columns and a 4-stage ring of A
// operands (32 columns = 64 bf16 of K each).  The epilogue releases the accumulator as soon as
// it holds the tile in registers (rounded to bf16, two columns per word), so the next tile's
// MMAs overlap the processing and stores of this one; dact, which multiplies the fp32 values,
// releases it after its last chunk.  An MMA instruction costs time in proportion to N from
// N = 128 up (half a cycle per column per K=16 step), and a k-step's fixed costs (barrier
// round trips, conversion) do not grow with N, so the widest tile amortizes them best.
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

// MMA-facing ring: stage s holds the token tile (shared memory) and the bf16 A operand
// (TMEM) of one k-step; the MMA waits once and commits once per k-step.
constexpr int kStages = 4;        // even: a stage always belongs to the same converter parity
// packed-weight ring depth (even, same reason): 8 stages, 4 in the block-scaled form, whose
// per-tile token scales take the shared memory the other four would
constexpr int kWStagesMax = 8;
template <bool BS>
__host__ __device__ constexpr int wstages() { return BS ? 4 : kWStagesMax; }
constexpr int kThreads = 512;
constexpr int kConvWarps = 8;
constexpr int kTokBytes = kBN * kBK * 2;      // 32 KB
constexpr int kWBytes = kBM * (kBK / 2);      // 4 KB of packed nibbles
constexpr int kAccCols = kBN;                 // fp32 accumulator columns per buffer
// One accumulator of kBN = 256 columns: the epilogue releases it as soon as it holds the tile
// in registers (two accumulators of 256 columns would leave no room for the A ring).
constexpr int kAccBufs = 1;
constexpr int kACol0 = kAccBufs * kAccCols;   // first TMEM column of the A ring
constexpr int kTmemCols = 512;
// Registers per thread by warpgroup after setmaxnreg: control (producers, MMA, warpgroup 0),
// converters (warpgroups 1-2), epilogue (warpgroup 3).  setmaxnreg.inc draws only on what the
// other warpgroups released from the block's launch allocation (kThreads x kLaunchRegs), so
// every warpgroup sets its count explicitly and the four shares must fit that allocation;
// launch_one also refuses to launch if ptxas allocated fewer than kLaunchRegs per thread.
constexpr int kLaunchRegs = 65536 / kThreads;  // 128: what __launch_bounds__(512, 1) allows
constexpr int kRegsCtl = 56, kRegsConv = 112, kRegsEpi = 232;
static_assert(kRegsCtl <= kLaunchRegs && kRegsConv <= kLaunchRegs && kRegsEpi >= kLaunchRegs,
              "control and converter warpgroups only release registers; the epilogue takes");
static_assert(128 * kRegsCtl + 2 * 128 * kRegsConv + 128 * kRegsEpi <= kThreads * kLaunchRegs,
              "register split exceeds the block's launch allocation: setmaxnreg.inc would wait forever");
static_assert(kRegsCtl % 8 == 0 && kRegsConv % 8 == 0 && kRegsEpi % 8 == 0, "setmaxnreg granularity");
static_assert(kACol0 + kStages * (kBK / 2) <= kTmemCols, "TMEM budget");
// Block-scaled variant (E2M1 weights in 8-bit containers against E4M3 tokens, UE8M0 scales):
// A stages of 64 bytes (16 columns), then per stage the scale-factor columns of A (4) and of
// the token tile (8, of which kBN/32 are used).
constexpr int kAColsBS = kBK / 4;
constexpr int kSfaCol0 = kACol0 + kStages * kAColsBS;
constexpr int kSfbCols = kBN / 32;
constexpr int kSfbCol0 = kSfaCol0 + kStages * 4;
static_assert(kSfbCol0 + kStages * 8 <= kTmemCols, "TMEM budget (block-scaled)");
static_assert(kSfbCols <= 8, "scale-factor columns of the token tile");
static_assert(kBN % 64 == 0 && kBN <= 256, "token tile (whole pairs of 32-column chunks)");
static_assert(wstages<false>() % 2 == 0 && wstages<true>() % 2 == 0 && kStages % 2 == 0,
              "ring depths must be even");

constexpr unsigned kFull = 0xFFFFFFFFu;

struct __align__(8) Barriers {
  uint64_t full[kStages];   // token bytes landed + 4 converter warps stored the A operand
  uint64_t empty[kStages];  // MMA commit: token stage and A stage free again
  uint64_t w_full[kWStagesMax];
  uint64_t w_empty[kWStagesMax];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t sc_full[2];
  uint64_t sc_empty[2];
  uint64_t drain;
};
static_assert(sizeof(Barriers) <= 512, "barrier block");

template <bool BS>
struct SmemLayoutT {
  // offsets from the 1024-aligned dynamic smem base
  static constexpr int tok = 0;                                  // 1024-aligned (128B swizzle)
  static constexpr int w = tok + kStages * kTokBytes;            // 256-aligned (32B swizzle)
  static constexpr int bars = w + wstages<BS>() * kWBytes;
  static constexpr int misc = bars + 512;                        // tmem slot, abort flag
  static constexpr int cw = misc + 64;                           // 8 warps x 4 x 32 scale words
  static constexpr int tables = cw + kConvWarps * 4 * 32 * 4;    // off[257], tile_start[257]
  static constexpr int sc = ((tables + 2 * 257 * 4) + 127) / 128 * 128;  // 2 scale buffers
};
static_assert(SmemLayoutT<false>::w % 1024 == 0 && SmemLayoutT<true>::w % 1024 == 0,
              "weight ring alignment");

template <uint32_t N>
MOE_DEV void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
MOE_DEV void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

struct Tile {
  int e, fb, row0, n_valid, feat0;
};

// An expert's m rows are split into equal token tiles of at most kBN rows (a multiple of 16),
// so that no tile is a small remainder: a k-step's fixed costs are the same for a tile of 32
// rows as for one of 256.
MOE_DEV int token_tile_rows(int m) {
  const int n = (m + kBN - 1) / kBN;
  const int rows = (m + n - 1) / n;
  return (rows + 15) & ~15;
}
MOE_DEV int token_tiles(int m) {
  if (m <= 0) return 0;
  const int rows = token_tile_rows(m);
  return (m + rows - 1) / rows;
}

__device__ __forceinline__ void decode_tile(int t, const int* s_tstart, const int* s_off, int E,
                                            int nfb, Tile& o) {
  int lo = 0, hi = E;  // largest lo with s_tstart[lo] <= t (s_tstart[E] = total > t)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tstart[mid] <= t) lo = mid; else hi = mid;
  }
  const int local = t - s_tstart[lo];
  const int tt = local / nfb;
  const int m = s_off[lo + 1] - s_off[lo];
  const int rows = token_tile_rows(m);
  o.e = lo;
  o.fb = local - tt * nfb;
  o.row0 = s_off[lo] + tt * rows;
  o.n_valid = min(rows, m - tt * rows);
  o.feat0 = o.fb * kBM;
}

// Last-phase parity of a ring stage after `issued` uses in total (for the exit drains).
MOE_DEV bool drain_ring(uint64_t* full, int stages, int issued, const DevErr& err, int where) {
  bool ok = true;
  for (int s = 0; s < stages && s < issued; ++s) {
    const int last = s + stages * ((issued - 1 - s) / stages);
    ok &= mbar_wait(smem_u32(&full[s]), (last / stages) & 1, err, where, nullptr);
  }
  return ok;
}

template <int EPI, bool COLT, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_tok,
                        const __grid_constant__ CUtensorMap tmap_lo,
                        const __grid_constant__ CUtensorMap tmap_w, const GemmArgs p) {
  static_assert(!BS || (EPI == kEpiGateUp && !COLT), "block-scaled form: gate_up only");
  using SmemLayout = SmemLayoutT<BS>;
  constexpr int kWStages = wstages<BS>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Barriers* bar = reinterpret_cast<Barriers*>(smem + SmemLayout::bars);
  volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(smem + SmemLayout::misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 8);
  int* s_off = reinterpret_cast<int*>(smem + SmemLayout::tables);
  int* s_tstart = s_off + 257;
  // per tile: 128 rows x K/32 (per-row) or 4 x K (transposed) weight scales; the block-scaled
  // form appends the token tile's activation scales (kBN rows x sfb_stride)
  const int sc_bytes = 4 * p.K + (BS ? kBN * p.sfb_stride : 0);
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
      mbar_init(smem_u32(&bar->full[s]), 1 + 4);  // token producer + 4 converter warps
      mbar_init(smem_u32(&bar->empty[s]), 1);     // MMA commit
    }
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(smem_u32(&bar->w_full[s]), 1);
      mbar_init(smem_u32(&bar->w_empty[s]), 4);  // the 4 converter warps of this parity
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bar->acc_full[s]), 1);
      mbar_init(smem_u32(&bar->acc_empty[s]), 4);
      mbar_init(smem_u32(&bar->sc_full[s]), 1);
      mbar_init(smem_u32(&bar->sc_empty[s]), kConvWarps);
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
    bool bad = MXFP4_MOE_DEBUG && s_off[0] != 0;
    for (int e = 0; e < E; ++e) {
      s_tstart[e] = acc;
      if (MXFP4_MOE_DEBUG && (s_off[e + 1] < s_off[e] || s_off[e + 1] > p.A)) bad = true;
      acc += token_tiles(s_off[e + 1] - s_off[e]) * nfb;
    }
    if (bad) {  // debug build: offsets that do not partition [0, A) -> no tiles at all
      err.set(MXFP4_MOE_ERR_DEVICE_BOUNDS, 0x600);
      for (int e = 0; e < E; ++e) s_tstart[e] = 0;
      acc = 0;
    }
    s_tstart[E] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int total = s_tstart[E];
  const int wg = warp >> 2;

  if (wg == 0) {
    setmaxnreg_dec<kRegsCtl>();
    if (warp == 0) {
      // ============================ token producer ==================================
      int issued = 0;
      if (lane == 0) {
        prefetch_tmap(&tmap_tok);
        if (BS) prefetch_tmap(&tmap_lo);
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
          Tile tl;
          decode_tile(t, s_tstart, s_off, E, nfb, tl);
          for (int ks = 0; ks < nk; ++ks) {
            if (!mbar_wait_sleep(smem_u32(&bar->empty[s]), ph ^ 1, err, 0x201, s_abort, 64)) { ok = false; break; }
            const uint32_t fb = smem_u32(&bar->full[s]);
            mbar_arrive_expect_tx(fb, kTokBytes);
            if (BS) {  // hi and lo E4M3 parts: 64 bytes per row each, half a stage apiece
              tma_load_2d(smem_u32(smem + SmemLayout::tok + s * kTokBytes), &tmap_tok, ks * kBK,
                          tl.row0, fb);
              tma_load_2d(smem_u32(smem + SmemLayout::tok + s * kTokBytes + kTokBytes / 2),
                          &tmap_lo, ks * kBK, tl.row0, fb);
            } else {
              tma_load_2d(smem_u32(smem + SmemLayout::tok + s * kTokBytes), &tmap_tok, ks * kBK,
                          tl.row0, fb);
            }
            ++issued;
            if (++s == kStages) { s = 0; ph ^= 1; }
          }
        }
      }
      __syncwarp();
      __syncthreads();
      // exit drain: every token copy issued has landed.  `full` also counts converter
      // arrivals, so wait on the copies' own completion: the stage's phase can only
      // complete once its bytes are in (or the CTA aborted, which the drain bound covers).
      if (lane == 0) drain_ring(bar->full, kStages, issued, err, 0x2F0);
    } else if (warp == 2) {
      // ============================ weight + scale producer =========================
      int issued = 0, sc_issued = 0;
      if (lane == 0) {
        prefetch_tmap(&tmap_w);
        bool ok = true;
        int lt = 0, ws = 0;
        uint32_t wph = 0;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
          Tile tl;
          decode_tile(t, s_tstart, s_off, E, nfb, tl);
          const int rows = min(kBM, N - tl.feat0);
          const int sb = lt & 1;
          if (!mbar_wait_sleep(smem_u32(&bar->sc_empty[sb]), ((lt >> 1) & 1) ^ 1, err, 0x200, s_abort, 128)) break;
          uint32_t bytes;
          const uint8_t* src;
          if (COLT) {
            bytes = (uint32_t)(rows / 32) * K;
            src = p.scales + ((size_t)tl.e * (N / 32) + tl.feat0 / 32) * K;
          } else {
            bytes = (uint32_t)rows * kb32;
            src = p.scales + ((size_t)tl.e * N + tl.feat0) * kb32;
          }
          const uint32_t sfb_bytes = BS ? (uint32_t)(tl.n_valid * p.sfb_stride) : 0u;
          mbar_arrive_expect_tx(smem_u32(&bar->sc_full[sb]), bytes + sfb_bytes);
          bulk_load(smem_u32(s_sc + sb * sc_bytes), src, bytes, smem_u32(&bar->sc_full[sb]));
          if (BS)
            bulk_load(smem_u32(s_sc + sb * sc_bytes + 4 * K),
                      p.sfb + (size_t)tl.row0 * p.sfb_stride, sfb_bytes,
                      smem_u32(&bar->sc_full[sb]));
          ++sc_issued;
          for (int ks = 0; ks < nk; ++ks) {
            if (!mbar_wait_sleep(smem_u32(&bar->w_empty[ws]), wph ^ 1, err, 0x202, s_abort, 64)) { ok = false; break; }
            const uint32_t fb = smem_u32(&bar->w_full[ws]);
            mbar_arrive_expect_tx(fb, kWBytes);
            tma_load_2d(smem_u32(smem + SmemLayout::w + ws * kWBytes), &tmap_w, ks * (kBK / 2),
                        tl.e * N + tl.feat0, fb);
            ++issued;
            if (++ws == kWStages) { ws = 0; wph ^= 1; }
          }
        }
      }
      __syncwarp();
      __syncthreads();
      if (lane == 0) {
        drain_ring(bar->w_full, kWStages, issued, err, 0x2F1);
        drain_ring(bar->sc_full, 2, sc_issued, err, 0x2F2);
      }
    } else if (warp == 1) {
      // ============================ MMA issuer ======================================
      if (lane == 0) {
        int s = 0;
        uint32_t ph = 0;
        const uint32_t tok_base = smem_u32(smem + SmemLayout::tok);
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
          Tile tl;
          decode_tile(t, s_tstart, s_off, E, nfb, tl);
          const int acc = lt % kAccBufs;
          if (!mbar_wait(smem_u32(&bar->acc_empty[acc]), ((lt / kAccBufs) & 1) ^ 1, err, 0x300, s_abort)) break;
          tc_fence_after();
          const uint32_t idesc = idesc_bf16_m128((tl.n_valid + 15) & ~15);
          const uint32_t d_tmem = tmem + acc * kAccCols;
          // one k-step per round: wait for its stage, issue its MMAs, release it on completion
          const int npad = (tl.n_valid + 15) & ~15;
          for (int ks = 0; ks < nk; ++ks) {
            if (!mbar_wait(smem_u32(&bar->full[s]), ph, err, 0x301, s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t tbase = tok_base + s * kTokBytes;
            if (BS) {
              const uint64_t bhi = smem_desc_kmajor_sw64(tbase);
              const uint64_t blo = smem_desc_kmajor_sw64(tbase + kTokBytes / 2);
              const uint32_t a_tmem = tmem + kACol0 + s * kAColsBS;
              const uint32_t sfa = tmem + kSfaCol0 + s * 4, sfb = tmem + kSfbCol0 + s * 8;
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const uint32_t id = idesc_mxf4a_m128(npad, (uint32_t)kk);
                mma_mxf8_ts(d_tmem, a_tmem + kk * 8, bhi + (uint64_t)(kk * 2), id, sfa, sfb,
                            (ks | kk) != 0);
                mma_mxf8_ts(d_tmem, a_tmem + kk * 8, blo + (uint64_t)(kk * 2), id, sfa, sfb, 1u);
              }
            } else {
              const uint64_t bdesc = smem_desc_kmajor_sw128(tbase);
              const uint32_t a_tmem = tmem + kACol0 + s * (kBK / 2);
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                mma_bf16_ts(d_tmem, a_tmem + kk * 8, bdesc + (uint64_t)(kk * 2), idesc,
                            (ks | kk) != 0);
            }
            mma_commit(smem_u32(&bar->empty[s]));
            if (++s == kStages) { s = 0; ph ^= 1; }
          }
          if (ok) mma_commit(smem_u32(&bar->acc_full[acc]));
        }
        // every MMA issued by this thread has completed once `drain` flips
        mma_commit(smem_u32(&bar->drain));
        mbar_wait(smem_u32(&bar->drain), 0, err, 0x3F0, nullptr);
      }
      __syncwarp();
      __syncthreads();
    } else {
      __syncthreads();
    }
  } else if (wg < 3) {
    // ================================ converters ====================================
    if (kRegsConv < kLaunchRegs) setmaxnreg_dec<kRegsConv>();
    // Converter warp c (0..7) serves TMEM lane quarter q = warp % 4.  A tile's k-steps are
    // converted in pairs (2u, 2u+1) that share their scale set-up; the two warps of a quarter
    // take alternate pairs (running pair index parity = c / 4) and publish each k-step as soon
    // as it is stored.
    const int q = warp & 3;
    const int cidx = warp - 4;
    const int par = cidx >> 2;
    // per-warp scale-factor words (transposed scales): f1 of k-steps 0/1, then f2 of 0/1
    uint32_t* cw = reinterpret_cast<uint32_t*>(smem + SmemLayout::cw) + cidx * 128;
    const int r = 32 * q + lane;  // row of the 128-row weight tile
    // 32B-swizzled packed tile: the two 16-byte halves of row r swap when bit 2 of r is set
    const int swz = (r >> 2) & 1;
    const int npair = (nk + 1) >> 1;
    int g = 0;   // running index of the current tile's first k-step
    int it = 0;  // running pair index
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt, g += nk) {
      Tile tl;
      decode_tile(t, s_tstart, s_off, E, nfb, tl);
      const bool active = tl.feat0 + 32 * q < N;  // warp-uniform: N % 32 == 0
      const int sb = lt & 1;
      if (!mbar_wait_sleep(smem_u32(&bar->sc_full[sb]), (lt >> 1) & 1, err, 0x400, s_abort, 64)) break;
      const uint8_t* scb = s_sc + sb * sc_bytes;
      for (int u = 0; u < npair; ++u, ++it) {
        if ((it & 1) != par) continue;
        const int ks0 = 2 * u;
        const bool two = ks0 + 1 < nk;
        const int ga = g + ks0;  // running index of the pair's first k-step
        // scale factors: f1 (and f2 when some scale is above 128), as bf16x2 words
        // (per row, forward: the pair's four 32-element blocks; the rare second factor is
        // re-derived from the scale bytes where it is needed)
        uint32_t f1[4] = {0, 0, 0, 0};
        bool slow = false;
        // block-scaled form: the token tile's activation scales of the pair's four 32-element
        // blocks, one 32-bit word per token (word u of the token's row, stored at word
        // u ^ ((row / 4) % 8) so that the 32 lanes' loads hit 32 different banks)
        uint32_t sfb4[kSfbCols];
        if (BS) {
          // the block-scaled MMA applies the UE8M0 scales itself (scale-factor columns)
          const uint8_t* sfbb = scb + 4 * K;
#pragma unroll
          for (int j = 0; j < kSfbCols; ++j) {
            const int tok = 32 * j + lane;
            const int wsw = u ^ (((tl.row0 + tok) >> 2) & 7);
            sfb4[j] = tok < tl.n_valid
                          ? *reinterpret_cast<const uint32_t*>(sfbb + tok * p.sfb_stride + 4 * wsw)
                          : 0u;
          }
        } else if (!COLT) {
          uint32_t mx = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int blk = 2 * ks0 + j;
            const uint32_t sv = (active && blk < kb32) ? scb[r * kb32 + blk] : 127u;
            mx = max(mx, sv);
            f1[j] = dup16(ue8m0_f1(sv));
          }
          slow = __any_sync(kFull, mx > 128u);
        } else {
          // lane l computes the factors of K elements 2l, 2l+1 of each k-step; the warp
          // shares them through shared memory (one scale row for all 32 lanes).
          uint32_t mx = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int k0 = (ks0 + h) * kBK + 2 * lane;
            const uint32_t s0 = (active && k0 < K) ? scb[q * K + k0] : 127u;
            const uint32_t s1 = (active && k0 + 1 < K) ? scb[q * K + k0 + 1] : 127u;
            mx = max(mx, max(s0, s1));
            cw[32 * h + lane] = ue8m0_f1(s0) | (ue8m0_f1(s1) << 16);
          }
          slow = __any_sync(kFull, mx > 128u);
          if (slow) {  // rare: scales above 128 need the second factor
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int k0 = (ks0 + h) * kBK + 2 * lane;
              const uint32_t s0 = (active && k0 < K) ? scb[q * K + k0] : 127u;
              const uint32_t s1 = (active && k0 + 1 < K) ? scb[q * K + k0 + 1] : 127u;
              cw[64 + 32 * h + lane] = ue8m0_f2(s0) | (ue8m0_f2(s1) << 16);
            }
          }
          __syncwarp();  // cw written before any lane reads it
        }

        // each k-step: wait for its packed bytes, expand them to bf16 in registers, wait for
        // its A stage to be free (the MMA consumed the k-step kStages earlier) and store it
        const uint32_t lanes = (uint32_t)(32 * q) << 16;
        // k-step j converted and stored: release its packed bytes and publish its A stage
        // (the warp's reads of cw for it are ordered before any later write by the syncwarp)
        auto publish_stage = [&](int j, bool stored) {
          if (stored) tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(smem_u32(&bar->w_empty[j % kWStages]));
            mbar_arrive(smem_u32(&bar->full[j % kStages]));
          }
        };
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && !two) break;
          const int s = (ga + h) % kWStages;
          if (!mbar_wait_sleep(smem_u32(&bar->w_full[s]), ((ga + h) / kWStages) & 1, err, 0x401,
                         s_abort, 32)) {
            ok = false;
            break;
          }
          uint32_t qw[8];
          {
            const uint8_t* row = smem + SmemLayout::w + s * kWBytes + r * (kBK / 2);
            const uint4 w0 = *reinterpret_cast<const uint4*>(row + (swz << 4));
            const uint4 w1 = *reinterpret_cast<const uint4*>(row + ((swz ^ 1) << 4));
            qw[0] = w0.x; qw[1] = w0.y; qw[2] = w0.z; qw[3] = w0.w;
            qw[4] = w1.x; qw[5] = w1.y; qw[6] = w1.z; qw[7] = w1.w;
          }
          if (BS) {
            // E2M1 codes into 8-bit containers (the MMA decodes them with the scales)
            uint32_t out16[16];
            if (active) {
#pragma unroll
              for (int i = 0; i < 8; ++i) e2m1x8_to_containers(qw[i], out16[2 * i], out16[2 * i + 1]);
            }
            // scale factors of the k-step's two 32-element blocks, bytes 0 and 1 of a column.
            // The MMA reads weight row m's from lane m, column m / 32: this warp's rows are
            // its own lanes, column q.  The token tile's are read from lane n % 32, column
            // n / 32; every lane quarter gets the same copy.
            const int blk0 = 2 * (ks0 + h);
            uint32_t sfa1;
            {
              const bool rv = r < min(kBM, N - tl.feat0);
              const uint32_t b0 = (rv && blk0 < kb32) ? scb[r * kb32 + blk0] : 0u;
              const uint32_t b1 = (rv && blk0 + 1 < kb32) ? scb[r * kb32 + blk0 + 1] : 0u;
              sfa1 = b0 | (b1 << 8);
            }
            uint32_t sfb8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) sfb8[j] = j < kSfbCols ? (h ? sfb4[j] >> 16 : sfb4[j] & 0xFFFFu) : 0u;
            const int sa = (ga + h) % kStages;
            if (!mbar_wait(smem_u32(&bar->empty[sa]), (((ga + h) / kStages) & 1) ^ 1, err, 0x402,
                           s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (active) tmem_st16(tmem + lanes + kACol0 + sa * kAColsBS, out16);
            tmem_st1(tmem + lanes + kSfaCol0 + sa * 4 + q, sfa1);
            tmem_st8(tmem + lanes + kSfbCol0 + sa * 8, sfb8);
            publish_stage(ga + h, true);
            continue;
          }
          uint32_t out[32];
          if (active) {
            if (!COLT) {
              const uint32_t fa0 = h ? f1[2] : f1[0];
              const uint32_t fa1 = h ? f1[3] : f1[1];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                uint32_t pt[4];
                e2m1x8_to_bf16x2_pattern(qw[i], pt);
                const uint32_t fa = i < 4 ? fa0 : fa1;
#pragma unroll
                for (int m = 0; m < 4; ++m) out[4 * i + m] = bmul2(pt[m], fa);
              }
              if (slow) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const int blk = 2 * (ks0 + h) + j;
                  const uint32_t f2 =
                      dup16(ue8m0_f2(blk < kb32 ? scb[r * kb32 + blk] : 127u));
#pragma unroll
                  for (int m = 16 * j; m < 16 * j + 16; ++m) out[m] = bmul2(out[m], f2);
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                uint32_t pt[4];
                e2m1x8_to_bf16x2_pattern(qw[i], pt);
                const uint4 f = *reinterpret_cast<const uint4*>(cw + 32 * h + 4 * i);
                out[4 * i + 0] = bmul2(pt[0], f.x);
                out[4 * i + 1] = bmul2(pt[1], f.y);
                out[4 * i + 2] = bmul2(pt[2], f.z);
                out[4 * i + 3] = bmul2(pt[3], f.w);
              }
              if (slow) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const uint4 f = *reinterpret_cast<const uint4*>(cw + 64 + 32 * h + 4 * i);
                  out[4 * i + 0] = bmul2(out[4 * i + 0], f.x);
                  out[4 * i + 1] = bmul2(out[4 * i + 1], f.y);
                  out[4 * i + 2] = bmul2(out[4 * i + 2], f.z);
                  out[4 * i + 3] = bmul2(out[4 * i + 3], f.w);
                }
              }
            }
          }
          const int sa = (ga + h) % kStages;
          if (!mbar_wait(smem_u32(&bar->empty[sa]), (((ga + h) / kStages) & 1) ^ 1, err, 0x402,
                         s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (active) tmem_st32(tmem + lanes + kACol0 + sa * (kBK / 2), out);
          publish_stage(ga + h, active);
        }
        if (!ok) break;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->sc_empty[sb]));
    }
    // an aborted pair may leave TMEM stores in flight: none may outlive the allocation
    __syncwarp();
    tmem_wait_st();
    __syncthreads();
  } else {
    // ================================ epilogue ======================================
    setmaxnreg_inc<kRegsEpi>();
    const int q = warp & 3;
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      Tile tl;
      decode_tile(t, s_tstart, s_off, E, nfb, tl);
      const int acc = lt % kAccBufs;
      const int f = tl.feat0 + 32 * q + lane;  // output feature of this thread
      const bool active = tl.feat0 + 32 * q < N;
      // dact: the saved GLU factors of the tile's first 32 rows are requested before the
      // accumulator is ready; each chunk then requests the next chunk's while it computes
      uint32_t dnext[32];
      if (EPI == kEpiDact && active) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          dnext[j] = __ldg(p.dgu + (size_t)min(tl.row0 + j, p.A - 1) * N + f);
      }
      // the bias (gate_up, down) and dact's routing weights of the tile's rows (lane l holds
      // row 32 c + l of chunk c) are requested before the accumulator is ready, so that no
      // global load sits between the accumulator and its release
      float bias_f = 0.f;
      if ((EPI == kEpiGateUp || EPI == kEpiDown) && active)
        bias_f = bf16_to_f(p.bias[(size_t)tl.e * N + f]);
      float wrow[kBN / 32];
      if (EPI == kEpiDact) {
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
          wrow[c] = (32 * c + lane < tl.n_valid) ? p.w_row[tl.row0 + 32 * c + lane] : 0.f;
      }
      if (!mbar_wait_sleep(smem_u32(&bar->acc_full[acc]), (lt / kAccBufs) & 1, err, 0x500, s_abort, 256)) break;
      tc_fence_after();
      const uint32_t acc_tmem = tmem + ((uint32_t)(32 * q) << 16) + acc * kAccCols;
      const bool odd = (lane & 1) != 0;
      if (EPI != kEpiDact) {
        // Early release: the tile's accumulator, bias added and rounded to bf16 (two columns
        // per word), moves into registers first; the MMA may start the next tile as soon as
        // every epilogue warp holds its rows, while the values are processed and stored.
        // down and dx store exactly these bf16 values; gate_up evaluates the GLU on them
        // (h rounded to bf16, as the eager bf16 model holds it).
        uint32_t pk[kBN / 32][16];
        // two chunks per TMEM round trip (the release waits for all of them)
#pragma unroll
        for (int c = 0; c < kBN / 32; c += 2) {
          if (32 * c < tl.n_valid) {
            uint32_t r0[32], r1[32];
            tmem_ld32(acc_tmem + 32 * c, r0);
            tmem_ld32(acc_tmem + 32 * (c + 1), r1);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              pk[c][jj] = pack_bf16x2(__uint_as_float(r0[2 * jj]) + bias_f,
                                      __uint_as_float(r0[2 * jj + 1]) + bias_f);
              pk[c + 1][jj] = pack_bf16x2(__uint_as_float(r1[2 * jj]) + bias_f,
                                          __uint_as_float(r1[2 * jj + 1]) + bias_f);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->acc_empty[acc]));
        if (active) {
          // the work on one chunk of 32 columns (the tile's rows rbase .. rbase + ncol - 1)
          auto chunk = [&](const uint32_t (&cur)[16], int ncol, int rbase) {
            if (EPI == kEpiGateUp) {
              // Columns j (even lane) and j+1 (odd lane) of each pair: the lanes of an
              // interleaved (gate, up) feature pair swap one value so that each holds (g, u)
              // of its own column.  Stored per (row, j): act = (u'+1) g' sigmoid(a g') and,
              // for the backward, the GLU derivative factors d act/d g and d act/d u as one
              // bf16x2 word.
              const int I = N >> 1;
              const int jf = f >> 1;
              uint32_t dw16[16];
              float av[16];
              // two columns per step with the paired fp32 instructions (same operations and
              // rounding as one column at a time)
              const uint64_t kOne = f2(1.f, 1.f);
              const uint64_t kHalfAlpha = f2(0.5f * p.alpha, 0.5f * p.alpha);
              const uint64_t kHalf = f2(0.5f, 0.5f), kAlpha = f2(p.alpha, p.alpha);
              const uint64_t kMinusOne = f2(-1.f, -1.f);
#pragma unroll
              for (int jj = 0; jj < 16; jj += 2) {
                const uint32_t wa = cur[jj], wb = cur[jj + 1];  // columns 2jj, 2jj+1 | +2, +3
                const float v0a = bf16_lo(wa), v0b = bf16_lo(wb), v1a = bf16_hi(wa), v1b = bf16_hi(wb);
                const float ra = __shfl_xor_sync(kFull, odd ? v0a : v1a, 1);
                const float rb = __shfl_xor_sync(kFull, odd ? v0b : v1b, 1);
                const float ga = odd ? ra : v0a, ua = odd ? v1a : ra;
                const float gb = odd ? rb : v0b, ub = odd ? v1b : rb;
                const uint64_t gc = f2(fminf(ga, p.limit), fminf(gb, p.limit));
                const uint64_t uc = f2(fminf(fmaxf(ua, -p.limit), p.limit), fminf(fmaxf(ub, -p.limit), p.limit));
                // sigmoid(a g') = (1 + tanh(a g' / 2)) / 2
                const uint64_t z = f2mul(kHalfAlpha, gc);
                float ta, tb;
                asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(f2lo(z)));
                asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(f2hi(z)));
                const uint64_t sg = f2fma(kHalf, f2(ta, tb), kHalf);
                const uint64_t t1 = f2mul(gc, sg);
                const uint64_t up1 = f2add(uc, kOne);
                const uint64_t act = f2mul(up1, t1);
                av[jj] = f2lo(act);
                av[jj + 1] = f2hi(act);
                // d act / d g' = (u'+1) (s + a t1 (1 - s)); d act / d u' = t1
                const uint64_t om = f2fma(sg, kMinusOne, kOne);
                const uint64_t dg = f2mul(up1, f2fma(f2mul(kAlpha, t1), om, sg));
                // bf16(g) <= limit  <=>  g <= mask_limit (and likewise for |bf16(u)|)
                const float dga = (ga <= p.mask_limit) ? f2lo(dg) : 0.f;
                const float dgb = (gb <= p.mask_limit) ? f2hi(dg) : 0.f;
                const float dua = (fabsf(ua) <= p.mask_limit) ? f2lo(t1) : 0.f;
                const float dub = (fabsf(ub) <= p.mask_limit) ? f2hi(t1) : 0.f;
                dw16[jj] = pack_bf16x2(dga, dua);
                dw16[jj + 1] = pack_bf16x2(dgb, dub);
              }
              uint32_t* dgu_out = reinterpret_cast<uint32_t*>(p.out0);
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int col = 2 * jj + (odd ? 1 : 0);
                if (col < ncol) {
                  const size_t o = (size_t)(rbase + col) * I + jf;
                  dgu_out[o] = dw16[jj];
                  p.out1[o] = f_to_bf16(av[jj]);
                }
              }
            } else {
              // Feature pairs (f, f+1) live in lanes (2m, 2m+1), each lane holding its feature
              // for the columns (2jj, 2jj+1): after one swap of whole words the even lane
              // holds both features of column 2jj, the odd lane both of column 2jj+1.  Rows
              // are stored in expert-sorted order (down: y = act W_d^T + b_d, not yet
              // weighted; the combine applies the routing weights).
              uint32_t* orow = reinterpret_cast<uint32_t*>(p.out0);
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const uint32_t w = cur[jj];
                const uint32_t wp = __shfl_xor_sync(kFull, w, 1);
                const uint32_t ow = odd ? prmt(wp, w, 0x7632u) : prmt(w, wp, 0x5410u);
                const int col = 2 * jj + (odd ? 1 : 0);
                if (col < ncol) orow[((size_t)(rbase + col) * N + (f & ~1)) >> 1] = ow;
              }
            }
          };
          if (EPI == kEpiGateUp) {
            // one chunk per pass, always from pk[0]: the chunks move down one slot per pass,
            // so the GLU is emitted once (eight unrolled copies would crowd the instruction
            // cache that the converters and the MMA issuer run from)
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
              if (32 * c >= tl.n_valid) break;
              chunk(pk[0], min(32, tl.n_valid - 32 * c), tl.row0 + 32 * c);
#pragma unroll
              for (int cc = 0; cc + 1 < kBN / 32; ++cc)
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) pk[cc][jj] = pk[cc + 1][jj];
            }
          } else {
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c) {
              if (32 * c >= tl.n_valid) break;
              chunk(pk[c], min(32, tl.n_valid - 32 * c), tl.row0 + 32 * c);
            }
          }
        }
      } else {
        // dact keeps the fp32 accumulator through its multiply: chunk by chunk, then release
        // one chunk per pass (rolled, as for the GLU): the routing weights move down one slot
        // per pass, so the current chunk's are always in wrow[0]
#pragma unroll 1
        for (int c0 = 0; c0 < tl.n_valid; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(acc_tmem + c0, r);
          const float my_w = wrow[0];
#pragma unroll
          for (int cc = 0; cc + 1 < kBN / 32; ++cc) wrow[cc] = wrow[cc + 1];
          tmem_wait_ld();
          if (!active) continue;
          const int ncol = min(32, tl.n_valid - c0);
          const int rbase = tl.row0 + c0;
          // dZ = dY W_d for this row; dact = w dZ; dH = (dact * dact/dg, dact * dact/du)
          // from the factors the forward saved.
          const int I = N;
          uint32_t* dh = reinterpret_cast<uint32_t*>(p.out0);
          uint32_t dcur[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) dcur[j] = dnext[j];
          if (c0 + 32 < tl.n_valid) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              dnext[j] = __ldg(p.dgu + (size_t)min(rbase + 32 + j, p.A - 1) * I + f);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float dact = __shfl_sync(kFull, my_w, j) * __uint_as_float(r[j]);
            const uint32_t dh2 = pack_bf16x2(dact * bf16_lo(dcur[j]), dact * bf16_hi(dcur[j]));
            if (j < ncol) dh[(size_t)(rbase + j) * I + f] = dh2;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->acc_empty[acc]));
      }
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

template <int EPI, bool COLT, bool BS>
cudaError_t launch_one(const CUtensorMap& tt, const CUtensorMap& tl, const CUtensorMap& tw,
                       const GemmArgs& a, int grid, size_t smem, cudaStream_t st) {
  auto kern = grouped_gemm_kernel<EPI, COLT, BS>;
  // the setmaxnreg split assumes kLaunchRegs registers per thread at launch
  cudaFuncAttributes fa;
  cudaError_t fe = cudaFuncGetAttributes(&fa, kern);
  if (fe != cudaSuccess) return fe;
  if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(tt, tl, tw, a);
  return cudaGetLastError();
}

// 2-D tiled map over a row-major [rows][cols] array of `elem`-byte elements.
bool encode_2d(EncodeTiledFn enc, CUtensorMap* m, CUtensorMapDataType type, const void* base,
               int elem, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t grouped_gemm_smem_bytes(int K, int sfb_stride) {
  return 1024 + (sfb_stride ? SmemLayoutT<true>::sc : SmemLayoutT<false>::sc) +
         2 * ((size_t)(4 * K) + (size_t)kBN * sfb_stride);
}

cudaError_t launch_grouped_gemm(int epi, bool transposed_scales, const void* tokens,
                                const uint8_t* wq, const GemmArgs& a, int num_sms,
                                cudaStream_t st) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const bool bs = a.tok_lo != nullptr;
  CUtensorMap tt, tl, tw;
  if (bs) {  // E4M3 hi / lo parts: [A][K] bytes each, 64-byte rows per k-step
    if (epi != kEpiGateUp || transposed_scales || !a.sfb || a.sfb_stride % 32 ||
        a.sfb_stride < 2 * ((a.K + kBK - 1) / kBK))
      return cudaErrorInvalidValue;
    if (!encode_2d(enc, &tt, CU_TENSOR_MAP_DATA_TYPE_UINT8, tokens, 1, a.K, a.A, kBK, kBN,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_2d(enc, &tl, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.tok_lo, 1, a.K, a.A, kBK, kBN,
                   CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  } else {
    if (!encode_2d(enc, &tt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, tokens, 2, a.K, a.A, kBK, kBN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    tl = tt;
  }
  if (!encode_2d(enc, &tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, wq, 1, a.K / 2,
                 (uint64_t)a.E * (uint64_t)a.N, kBK / 2, kBM, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  const size_t smem = grouped_gemm_smem_bytes(a.K, bs ? a.sfb_stride : 0);
  const int grid = num_sms;
  if (bs) return launch_one<kEpiGateUp, false, true>(tt, tl, tw, a, grid, smem, st);
  switch (epi * 2 + (transposed_scales ? 1 : 0)) {
    case kEpiGateUp * 2 + 0: return launch_one<kEpiGateUp, false, false>(tt, tl, tw, a, grid, smem, st);
    case kEpiDown * 2 + 0: return launch_one<kEpiDown, false, false>(tt, tl, tw, a, grid, smem, st);
    case kEpiDact * 2 + 1: return launch_one<kEpiDact, true, false>(tt, tl, tw, a, grid, smem, st);
    case kEpiDx * 2 + 1: return launch_one<kEpiDx, true, false>(tt, tl, tw, a, grid, smem, st);
    // plain product over the stored rows (the grouped matmul entry point)
    case kEpiDx * 2 + 0: return launch_one<kEpiDx, false, false>(tt, tl, tw, a, grid, smem, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
