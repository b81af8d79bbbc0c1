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

// Both kernels take 64 tokens per CTA through H in chunks of 64 features.
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
// 4 warps x 16 tokens, each warp's logits on m16n8k16 bf16 mma.sync tiles (fp32 accumulation).
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
// g_out = bf16(g + dx + d_logits W_r^T) in fp32 on the CUDA cores: a CTA takes 64 tokens and
// walks H in chunks of 64 features; thread (tg, hg) forms the 4 x 8 block of tokens 4 tg..+3
// and features 8 hg..+7 of the chunk, summing the experts in ascending order with fp32 FMAs
// from two transposed shared-memory tiles (d_logits [e][token] for the CTA, W_r [e][h] for
// the chunk; per expert one 16-byte load of d_logits and two of W_r feed 32 FMAs), then adds
// g and dx (requested before the FMAs) and rounds once.
constexpr int kGCTok = 64, kGCH = 64;

__global__ void __launch_bounds__(kThreads) grad_chain_kernel(
    int T, int H, int E, const uint16_t* __restrict__ g, const uint16_t* __restrict__ dx,
    const float* __restrict__ d_logits, const uint16_t* __restrict__ w_r,
    uint16_t* __restrict__ g_out) {
  extern __shared__ __align__(16) float s_dyn[];
  float* s_dl = s_dyn;                // [E][kGCTok]
  float* s_w = s_dyn + E * kGCTok;    // [E][kGCH]
  const int t0 = blockIdx.x * kGCTok;
  const int tg = threadIdx.x >> 3, hg = threadIdx.x & 7;  // 16 token groups x 8 feature groups
  for (int i = threadIdx.x; i < kGCTok * E; i += kThreads) {  // consecutive threads: tokens
    const int r = i % kGCTok, e = i / kGCTok;
    const int t = t0 + r;
    s_dl[e * kGCTok + r] = (t < T) ? __ldg(d_logits + (size_t)t * E + e) : 0.f;
  }
  const int nchunk = (H + kGCH - 1) / kGCH;
  for (int kc = 0; kc < nchunk; ++kc) {
    const int h0 = kc * kGCH;
    __syncthreads();  // d_logits staged / the previous chunk's W_r tile read
    if ((E & 7) == 0) {  // 16-byte vectors of 8 experts (w_r is 16-byte aligned)
      for (int i = threadIdx.x; i < kGCH * (E / 8); i += kThreads) {  // consecutive: features
        const int hh = i % kGCH, e = 8 * (i / kGCH);
        const int h = h0 + hh;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (h < H) v = __ldg(reinterpret_cast<const uint4*>(w_r + (size_t)h * E + e));
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          s_w[(e + 2 * q) * kGCH + hh] = bf16_lo(vw[q]);
          s_w[(e + 2 * q + 1) * kGCH + hh] = bf16_hi(vw[q]);
        }
      }
    } else {
      for (int i = threadIdx.x; i < kGCH * E; i += kThreads) {  // consecutive threads: features
        const int hh = i % kGCH, e = i / kGCH;
        const int h = h0 + hh;
        s_w[e * kGCH + hh] = (h < H) ? bf16_to_f(__ldg(w_r + (size_t)h * E + e)) : 0.f;
      }
    }
    __syncthreads();
    // this thread's g and dx vectors of the chunk, requested before the FMAs so that their
    // latency overlaps them (H % 32 == 0: the 8 features are all in range or all out)
    const int h = h0 + 8 * hg;
    uint4 gv[4], dv4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = t0 + 4 * tg + r;
      gv[r] = dv4[r] = make_uint4(0u, 0u, 0u, 0u);
      if (t < T && h < H) {
        const size_t at = ((size_t)t * H + h) / 8;
        gv[r] = reinterpret_cast<const uint4*>(g)[at];
        dv4[r] = __ldg(reinterpret_cast<const uint4*>(dx) + at);
      }
    }
    float acc[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[r][j] = 0.f;
    const float* dl = s_dl + 4 * tg;
    const float* wv = s_w + 8 * hg;
#pragma unroll 4
    for (int e = 0; e < E; ++e) {
      const float4 d = *reinterpret_cast<const float4*>(dl + e * kGCTok);
      const float4 w0 = *reinterpret_cast<const float4*>(wv + e * kGCH);
      const float4 w1 = *reinterpret_cast<const float4*>(wv + e * kGCH + 4);
      const float dv[4] = {d.x, d.y, d.z, d.w};
      const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[r][j] = fmaf(dv[r], ww[j], acc[r][j]);
    }
    if (h >= H) continue;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = t0 + 4 * tg + r;
      if (t >= T) continue;
      const size_t at = ((size_t)t * H + h) / 8;
      const uint32_t gw[4] = {gv[r].x, gv[r].y, gv[r].z, gv[r].w};
      const uint32_t dw[4] = {dv4[r].x, dv4[r].y, dv4[r].z, dv4[r].w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = pack_bf16x2(bf16_lo(gw[q]) + bf16_lo(dw[q]) + acc[r][2 * q],
                           bf16_hi(gw[q]) + bf16_hi(dw[q]) + acc[r][2 * q + 1]);
      reinterpret_cast<uint4*>(g_out)[at] = make_uint4(o[0], o[1], o[2], o[3]);
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

static size_t grad_chain_smem_bytes(int E) { return (size_t)E * (kGCTok + kGCH) * 4; }

cudaError_t launch_grad_chain(int T, int H, int E, const uint16_t* g, const uint16_t* dx,
                              const float* d_logits, const uint16_t* w_r, uint16_t* g_out,
                              cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const size_t smem = grad_chain_smem_bytes(E);
  cudaError_t e = cudaFuncSetAttribute(grad_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  grad_chain_kernel<<<(T + kGCTok - 1) / kGCTok, kThreads, smem, st>>>(T, H, E, g, dx, d_logits,
                                                                       w_r, g_out);
  return cudaGetLastError();
}

}  // namespace moe
