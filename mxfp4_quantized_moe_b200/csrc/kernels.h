// Internal launch interface of the MXFP4 MoE kernels (not part of the public C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

// 1 in the debug build (libmxfp4_moe_debug.so): kernels check workspace indices (common.cuh)
#ifndef MXFP4_MOE_DEBUG
#define MXFP4_MOE_DEBUG 0
#endif

namespace moe {

// Tile shape of the grouped GEMMs: 128 weight rows (output features) in TMEM as the
// MMA's A operand, BN routed tokens per tile in shared memory as the B operand.
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;

enum Epilogue : int { kEpiGateUp = 0, kEpiDown = 1, kEpiDact = 2, kEpiDx = 3 };

struct GemmArgs {
  const uint8_t* scales;   // per-row [E][N][K/32] (forward) or transposed [E][N/32][K] (backward)
  const int32_t* off;      // [E+1] start row of each expert in the expert-sorted order
  int E, K, N, A;          // experts, contraction length, output features, assignments
  const uint16_t* bias;    // bf16 [E][N]: gate_up bias (kEpiGateUp) or down bias (kEpiDown)
  uint16_t* out0;          // dGU [A][I] (bf16x2) | Y [A][H] | dH [A][2I] | dX rows [A][H],
                           // all in expert-sorted row order
  uint16_t* out1;          // act [A][I] (kEpiGateUp)
  const uint32_t* dgu;     // saved GLU derivative factors [A][I] bf16x2 (kEpiDact)
  const float* w_row;      // [A] routing weight of each expert-sorted row (kEpiDact)
  // block-scaled gate_up: the token tile comes as E4M3 hi (`tokens`) and lo parts with one
  // UE8M0 scale per row and 32 elements (sfb [A][sfb_stride]); null for the bf16 form
  const uint8_t* tok_lo;
  const uint8_t* sfb;
  int sfb_stride;
  float alpha, limit;
  float mask_limit;        // largest fp32 x whose bf16 rounding is <= limit (clamp-mask test)
  int* err;
};

// Encodes the tensor maps and launches one persistent grouped GEMM.
// `tokens`: bf16 [A][K] expert-sorted rows (or, with a.tok_lo set, the E4M3 hi part [A][K]
// bytes); `wq`: packed rows uint8 [E*N][K/2].
cudaError_t launch_grouped_gemm(int epi, bool transposed_scales, const void* tokens,
                                const uint8_t* wq, const GemmArgs& a, int num_sms,
                                cudaStream_t st);
// dynamic shared memory of a launch (sfb_stride: 0 for the bf16 form)
size_t grouped_gemm_smem_bytes(int K, int sfb_stride);

// Tokens are routed in segments of a fixed size; the routing scratch holds
// route_scratch_words(T, E) int32: the segments' expert histograms [route_blocks(T)][E], their
// exclusive scans over the segments [route_blocks(T)][E] and the column totals [E].
int route_blocks(int T);
size_t route_scratch_words(int T, int E);
// top-k + softmax over the k selected logits; idx/w in slot order (t*k + j), the segments'
// expert histograms in the scratch
cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               int32_t* scratch, int32_t* user_idx, float* user_w,
                               cudaStream_t st);
// the segments' histograms scanned over the segments, one block per expert column
cudaError_t launch_seg_scan(int T, int E, int32_t* scratch, cudaStream_t st);
// stable expert sort of the slots, one block per segment: off[E+1], perm[row] = slot,
// inv[slot] = row, w_row[row] = w[slot]
cudaError_t launch_build_perm(const int32_t* idx, const float* w, int T, int E, int k,
                              const int32_t* scratch, int32_t* off, int32_t* perm, int32_t* inv,
                              float* w_row, int* err, cudaStream_t st);
// dst[r] = src[perm[r] / k] for every expert-sorted row r.  With `dot_w` (the backward's
// gather of dY), `dst` first holds the forward's expert outputs y in sorted order, which are
// read in place: dot_w[perm[r]] = <src[perm[r] / k], y[r]> before the row is overwritten.
cudaError_t launch_gather_rows(const uint16_t* src, int H, int k, const int32_t* perm, int A,
                               uint16_t* dst, float* dot_w, int* err, cudaStream_t st);
// Gather x into expert-sorted rows as two E4M3 parts with a UE8M0 scale per 32 elements
// (hi, lo [A][H] bytes; sfb [A][sfb_stride] UE8M0 bytes, sfb_stride a multiple of 32; byte b
// of row r at word (b / 4) ^ ((r / 4) % 8), byte b % 4).
cudaError_t launch_gather_quant(const uint16_t* x, int H, int k, const int32_t* perm, int A,
                                uint8_t* hi, uint8_t* lo, uint8_t* sfb, int sfb_stride,
                                int* err, cudaStream_t st);
// out[t] = sum_j w[t*k+j] * rows[inv[t*k+j]] in fp32, rounded to bf16 once (w == nullptr: 1).
// `err` is the workspace error word: the debug build records out-of-range perm / inv entries
// there (DEVICE_BOUNDS) instead of reading through them.
cudaError_t launch_combine(const uint16_t* rows, const int32_t* inv, const float* w, int T, int k,
                           int H, uint16_t* out, int* err, cudaStream_t st);
// d_logits from d_topk_w through the softmax over the k selected logits (one thread per token)
cudaError_t launch_router_backward(const int32_t* idx, const float* w, const float* d_topk_w,
                                   int T, int E, int k, float* d_logits, cudaStream_t st);
cudaError_t launch_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                           uint16_t* out, cudaStream_t st);
cudaError_t launch_transpose_packed(const uint8_t* src, int E, int R, int C, uint8_t* dst,
                                    cudaStream_t st);
cudaError_t launch_transpose_scales(const uint8_t* src, int E, int R, int C, uint8_t* dst,
                                    cudaStream_t st);

}  // namespace moe
