// The residual stream around stacked MoE blocks, the caller's side of the block boundary,
// in two kernels:
//   residual_router  x_out = bf16(x + y) (fp32 sum, rounded once) and the next block's router
//                    logits = x_out W_r + b_r (fp32 accumulation) from one read of x and y;
//   grad_chain       g_out = bf16(g + dx + d_logits W_r^T) (fp32) from one read of g and dx.
// Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", section "What
// this does" (decoder layers trained with gradient checkpointing: the residual stream, the
// router linear and the MoE block).
#include <cuda_bf16.h>

#include "aux_kernels.h"
#include "common.cuh"

namespace moe {

namespace {

// Both kernels take 64 tokens per CTA (4 warps x 16 rows of an m16n8k16 bf16 mma.sync tile,
// fp32 accumulation) through H in chunks of 64.
constexpr int kTok = 64;
constexpr int kChunk = 64;
constexpr int kThreads = 128;

MOE_DEV void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four 8x8 bf16 matrices, transposed: thread i gives the address of row i % 8 of matrix i / 8.
MOE_DEV void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

MOE_DEV uint32_t add_bf16x2_rn(uint32_t a, uint32_t b) {  // fp32 sums rounded once
  return pack_bf16x2(bf16_lo(a) + bf16_lo(b), bf16_hi(a) + bf16_hi(b));
}

// ---- residual_router ------------------------------------------------------------------
// Per chunk: x_out = x + y for the CTA's 64 tokens (16-byte vectors: x_out to memory and to
// shared memory as the A operand) and the chunk of W_r as stored ([h][e], 16-byte vectors),
// whose B fragments ldmatrix.trans reads; the next chunk's loads are in flight while the MMAs
// of this one run.  Experts go in passes of 32 (E <= 32: four n-tiles) or 64 (eight; only
// tiles below E are computed); a second pass recomputes x_out's chunks from x and y without
// storing them.  Up to 120 registers a thread, so that four CTAs share an SM.
constexpr int kRRE = 64;           // expert columns of W_r staged per chunk (a pass uses 8 NT)
constexpr int kXPitch = kChunk + 8;  // bf16: 144-byte rows, conflict-free 32-bit fragment loads
constexpr int kWPitch = kRRE + 8;    // bf16: 144-byte rows, conflict-free ldmatrix rows

template <int NT>  // n-tiles of 8 experts per pass: 4 (E <= 32) or 8
__global__ void __launch_bounds__(kThreads, 4) residual_router_kernel(
    int T, int H, int E, const uint16_t* __restrict__ x, const uint16_t* __restrict__ y,
    const uint16_t* __restrict__ w_r, const uint16_t* __restrict__ b_r,
    uint16_t* __restrict__ x_out, float* __restrict__ logits) {
  __shared__ __align__(16) uint16_t s_x[kTok * kXPitch];     // x_out chunk [token][h]
  __shared__ __align__(16) uint16_t s_w[kChunk * kWPitch];   // W_r chunk [h][e]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int t0 = blockIdx.x * kTok;
  const int nchunk = (H + kChunk - 1) / kChunk;
  const bool vec_w = (E & 7) == 0;  // rows of W_r in whole 16-byte vectors
  constexpr int kPassE = 8 * NT;  // experts per pass
  const int passes = logits ? (E + kPassE - 1) / kPassE : 1;
  // this thread's share of a chunk: 4 vectors of x (and y), up to 4 vectors of W_r
  uint4 px[4], py[4], pw[4];
  auto load_chunk = [&](int kc, int e0) {
    const int h0 = kc * kChunk;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int v = threadIdx.x + kThreads * i;
      const int r = v >> 3, cv = v & 7;
      const int t = t0 + r, h = h0 + 8 * cv;
      px[i] = py[i] = make_uint4(0u, 0u, 0u, 0u);
      if (t < T && h < H) {
        const size_t at = ((size_t)t * H + h) / 8;
        px[i] = __ldg(reinterpret_cast<const uint4*>(x) + at);
        if (y) py[i] = __ldg(reinterpret_cast<const uint4*>(y) + at);
      }
    }
    if (logits && vec_w) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int v = threadIdx.x + kThreads * i;
        const int hh = v >> 3, cv = v & 7;  // 8 vectors of 8 experts per row
        const int h = h0 + hh, e = e0 + 8 * cv;
        pw[i] = make_uint4(0u, 0u, 0u, 0u);
        if (h < H && e < E) pw[i] = __ldg(reinterpret_cast<const uint4*>(w_r + (size_t)h * E + e));
      }
    }
  };
  auto store_chunk = [&](int kc, int e0, bool write_out) {
    const int h0 = kc * kChunk;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int v = threadIdx.x + kThreads * i;
      const int r = v >> 3, cv = v & 7;
      uint4 o = px[i];
      if (y) {
        o.x = add_bf16x2_rn(o.x, py[i].x);
        o.y = add_bf16x2_rn(o.y, py[i].y);
        o.z = add_bf16x2_rn(o.z, py[i].z);
        o.w = add_bf16x2_rn(o.w, py[i].w);
        const int t = t0 + r, h = h0 + 8 * cv;
        if (write_out && t < T && h < H) reinterpret_cast<uint4*>(x_out)[((size_t)t * H + h) / 8] = o;
      }
      *reinterpret_cast<uint4*>(s_x + r * kXPitch + 8 * cv) = o;
    }
    if (!logits) return;
    if (vec_w) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int v = threadIdx.x + kThreads * i;
        *reinterpret_cast<uint4*>(s_w + (v >> 3) * kWPitch + 8 * (v & 7)) = pw[i];
      }
    } else {
      for (int i = threadIdx.x; i < kChunk * kRRE; i += kThreads) {
        const int hh = i / kRRE, e = i % kRRE;
        const int h = h0 + hh, ee = e0 + e;
        s_w[hh * kWPitch + e] = (h < H && ee < E) ? __ldg(w_r + (size_t)h * E + ee) : (uint16_t)0;
      }
    }
  };
  for (int pass = 0; pass < passes; ++pass) {
    const int e0 = pass * kPassE;
    const int ntiles = logits ? min(kPassE, E - e0 + 7) / 8 : 0;  // n-tiles holding experts
    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    load_chunk(0, e0);
    for (int kc = 0; kc < nchunk; ++kc) {
      __syncthreads();  // every warp is done with the previous chunk's shared memory
      store_chunk(kc, e0, pass == 0);
      __syncthreads();
      if (kc + 1 < nchunk) load_chunk(kc + 1, e0);  // in flight during this chunk's MMAs
      if (!logits) continue;
      const uint16_t* xa = s_x + (16 * warp) * kXPitch;
      const uint32_t wbase = (uint32_t)__cvta_generic_to_shared(s_w);
#pragma unroll
      for (int kk = 0; kk < kChunk; kk += 16) {
        uint32_t a[4];
        a[0] = *reinterpret_cast<const uint32_t*>(xa + g * kXPitch + kk + 2 * c);
        a[1] = *reinterpret_cast<const uint32_t*>(xa + (g + 8) * kXPitch + kk + 2 * c);
        a[2] = *reinterpret_cast<const uint32_t*>(xa + g * kXPitch + kk + 8 + 2 * c);
        a[3] = *reinterpret_cast<const uint32_t*>(xa + (g + 8) * kXPitch + kk + 8 + 2 * c);
#pragma unroll
        for (int n = 0; n < NT; n += 2) {
          if (n >= ntiles) break;  // CTA-uniform
          // matrices: (k 0-7, tile n), (k 8-15, tile n), (k 0-7, tile n+1), (k 8-15, tile n+1)
          const int m = lane >> 3, rr = lane & 7;
          const int k = kk + rr + 8 * (m & 1), col = 8 * (n + (m >> 1));
          uint32_t b[4];
          ldmatrix_x4_trans(b, wbase + 2u * (uint32_t)(k * kWPitch + col));
          mma_16816(acc[n], a, b[0], b[1]);
          mma_16816(acc[n + 1], a, b[2], b[3]);
        }
      }
    }
    if (!logits) break;
    // accumulator tile n: tokens 16 warp + g (+8), experts e0 + 8n + 2c (+1)
#pragma unroll
    for (int n = 0; n < NT; ++n) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int t = t0 + 16 * warp + g + 8 * half;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int e = e0 + 8 * n + 2 * c + j;
          if (t < T && e < E)
            logits[(size_t)t * E + e] = acc[n][2 * half + j] + (b_r ? bf16_to_f(b_r[e]) : 0.f);
        }
      }
    }
  }
}

// ---- grad_chain ------------------------------------------------------------------------
// g_out = bf16(g + dx + d_logits W_r^T): a GEMM over the experts (K = E, up to 256) with the
// tokens as M and the features as N.  d_logits is fp32: each value splits exactly into three
// bf16 parts (hi = bf16(v), mid = bf16(v - hi), lo = v - hi - mid; 8 significant bits each,
// 24 in all), and the three products with the bf16 W_r accumulate in fp32, so the sum keeps
// fp32 operands.  The CTA's d_logits rows stay in shared memory; each chunk of 64 features
// stages its rows of W_r (zero-padded to whole k-steps), whose B fragments are plain 32-bit
// loads ([h][e] rows are k-contiguous).
MOE_DEV void split3(float v, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  const uint16_t h = f_to_bf16(v);
  const float r1 = v - bf16_to_f(h);
  const uint16_t m = f_to_bf16(r1);
  const uint16_t l = f_to_bf16(r1 - bf16_to_f(m));
  hi = h; mid = m; lo = l;
}

__global__ void __launch_bounds__(kThreads) grad_chain_kernel(
    int T, int H, int E, const uint16_t* __restrict__ g, const uint16_t* __restrict__ dx,
    const float* __restrict__ d_logits, const uint16_t* __restrict__ w_r,
    uint16_t* __restrict__ g_out, int ek, int dpitch, int wpitch) {
  // ek: E rounded up to a whole k-step (16); dpitch: fp32 row pitch of d_logits (ek + 8, so
  // that the 64-bit fragment loads of a half-warp hit distinct banks); wpitch: bf16 row pitch
  // of the W_r chunk (ek + 8: 4 (2 ek/16 + 1) words, conflict-free 32-bit fragment loads)
  extern __shared__ __align__(16) float s_dyn[];
  float* s_dl = s_dyn;                                               // [64][dpitch]
  uint16_t* s_w = reinterpret_cast<uint16_t*>(s_dl + kTok * dpitch);  // [64][wpitch]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gr = lane >> 2, c = lane & 3;
  const int t0 = blockIdx.x * kTok;
  for (int i = threadIdx.x; i < kTok * ek; i += kThreads) {
    const int r = i / ek, e = i % ek;
    const int t = t0 + r;
    s_dl[r * dpitch + e] = (t < T && e < E) ? __ldg(d_logits + (size_t)t * E + e) : 0.f;
  }
  const int nchunk = (H + kChunk - 1) / kChunk;
  for (int kc = 0; kc < nchunk; ++kc) {
    const int h0 = kc * kChunk;
    __syncthreads();  // d_logits staged / the previous chunk's W_r rows read
    if ((E & 7) == 0) {  // rows of W_r in whole 16-byte vectors (wpitch keeps rows aligned)
      const int nv = ek / 8;
      for (int i = threadIdx.x; i < kChunk * nv; i += kThreads) {
        const int hh = i / nv, cv = i % nv;
        const int h = h0 + hh, e = 8 * cv;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (h < H && e < E) v = __ldg(reinterpret_cast<const uint4*>(w_r + (size_t)h * E + e));
        *reinterpret_cast<uint4*>(s_w + hh * wpitch + e) = v;
      }
    } else {
      for (int i = threadIdx.x; i < kChunk * ek; i += kThreads) {
        const int hh = i / ek, e = i % ek;
        const int h = h0 + hh;
        s_w[hh * wpitch + e] = (h < H && e < E) ? __ldg(w_r + (size_t)h * E + e) : (uint16_t)0;
      }
    }
    __syncthreads();
    float acc[kChunk / 8][4];
#pragma unroll
    for (int n = 0; n < kChunk / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const float* da = s_dl + (16 * warp) * dpitch;
    for (int kk = 0; kk < ek; kk += 16) {
      // A fragments (rows gr, gr+8; experts kk + 2c (+1), kk + 8 + 2c (+1)) in three parts
      uint32_t ah[4], am[4], al[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = gr + 8 * (q & 1), col = kk + 2 * c + 8 * (q >> 1);
        const float2 v = *reinterpret_cast<const float2*>(da + row * dpitch + col);
        uint32_t h0_, m0_, l0_, h1_, m1_, l1_;
        split3(v.x, h0_, m0_, l0_);
        split3(v.y, h1_, m1_, l1_);
        ah[q] = h0_ | (h1_ << 16);
        am[q] = m0_ | (m1_ << 16);
        al[q] = l0_ | (l1_ << 16);
      }
#pragma unroll
      for (int n = 0; n < kChunk / 8; ++n) {
        const uint16_t* wb = s_w + (8 * n + gr) * wpitch + kk + 2 * c;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wb);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wb + 8);
        mma_16816(acc[n], al, b0, b1);  // smallest part first
        mma_16816(acc[n], am, b0, b1);
        mma_16816(acc[n], ah, b0, b1);
      }
    }
    // g_out for tokens 16 warp + gr (+8), features h0 + 8n + 2c (+1): two bf16 per word
#pragma unroll
    for (int n = 0; n < kChunk / 8; ++n) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int t = t0 + 16 * warp + gr + 8 * half;
        const int h = h0 + 8 * n + 2 * c;
        if (t < T && h < H) {
          const size_t at = ((size_t)t * H + h) / 2;
          const uint32_t gv = reinterpret_cast<const uint32_t*>(g)[at];
          const uint32_t dv = __ldg(reinterpret_cast<const uint32_t*>(dx) + at);
          const float s0 = bf16_lo(gv) + bf16_lo(dv) + acc[n][2 * half];
          const float s1 = bf16_hi(gv) + bf16_hi(dv) + acc[n][2 * half + 1];
          reinterpret_cast<uint32_t*>(g_out)[at] = pack_bf16x2(s0, s1);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_residual_router(int T, int H, int E, const uint16_t* x, const uint16_t* y,
                                   const uint16_t* w_r, const uint16_t* b_r, uint16_t* x_out,
                                   float* logits, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (E <= 32)
    residual_router_kernel<4><<<(T + kTok - 1) / kTok, kThreads, 0, st>>>(T, H, E, x, y, w_r, b_r,
                                                                        x_out, logits);
  else
    residual_router_kernel<8><<<(T + kTok - 1) / kTok, kThreads, 0, st>>>(T, H, E, x, y, w_r, b_r,
                                                                        x_out, logits);
  return cudaGetLastError();
}

size_t grad_chain_smem_bytes(int E) {
  const int ek = (E + 15) / 16 * 16;
  return (size_t)kTok * (ek + 8) * 4 + (size_t)kChunk * (ek + 8) * 2;
}

cudaError_t launch_grad_chain(int T, int H, int E, const uint16_t* g, const uint16_t* dx,
                              const float* d_logits, const uint16_t* w_r, uint16_t* g_out,
                              cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int ek = (E + 15) / 16 * 16;
  const size_t smem = grad_chain_smem_bytes(E);
  cudaError_t e = cudaFuncSetAttribute(grad_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  grad_chain_kernel<<<(T + kTok - 1) / kTok, kThreads, smem, st>>>(T, H, E, g, dx, d_logits, w_r,
                                                                   g_out, ek, ek + 8, ek + 8);
  return cudaGetLastError();
}

}  // namespace moe
