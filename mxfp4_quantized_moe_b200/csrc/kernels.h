// Internal launch interface of the MXFP4 MoE kernels (not part of the public C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

// Tile shape of the grouped GEMMs: 128 weight rows (output features) in TMEM as the
// MMA's A operand, BN routed tokens per tile in shared memory as the B operand.
constexpr int kBM = 128;
constexpr int kBN = 192;
constexpr int kBK = 64;

enum Epilogue : int { kEpiGateUp = 0, kEpiDown = 1, kEpiDact = 2, kEpiDx = 3 };

struct GemmArgs {
  const uint8_t* scales;   // per-row [E][N][K/32] (forward) or transposed [E][N/32][K] (backward)
  const int32_t* off;      // [E+1] start row of each expert in the expert-sorted order
  int E, K, N, A;          // experts, contraction length, output features, assignments
  const uint16_t* bias;    // bf16 [E][N]: gate_up bias (kEpiGateUp) or down bias (kEpiDown)
  uint16_t* out0;          // dGU [A][I] (bf16x2) | Yslot [A][H] | dH [A][2I] | dXslot [A][H]
  uint16_t* out1;          // act [A][I] (kEpiGateUp)
  const uint32_t* dgu;     // saved GLU derivative factors [A][I] bf16x2 (kEpiDact)
  const uint16_t* act;     // saved act [A][I] bf16 (kEpiDact)
  const int32_t* perm;     // [A] sorted row -> slot t*k+j
  const float* topk_w;     // [A] routing weight per slot
  float* dw_part;          // [N/32][A] partial <dZ, act> sums (kEpiDact)
  float alpha, limit;
  float mask_limit;        // largest fp32 x whose bf16 rounding is <= limit (clamp-mask test)
  int* err;
};

// Encodes the two tensor maps and launches one persistent grouped GEMM.
// `tokens`: bf16 [A][K] expert-sorted rows; `wq`: packed rows uint8 [E*N][K/2].
cudaError_t launch_grouped_gemm(int epi, bool transposed_scales, const uint16_t* tokens,
                                const uint8_t* wq, const GemmArgs& a, int num_sms,
                                cudaStream_t st);
size_t grouped_gemm_smem_bytes(int K);

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               int32_t* hist, int32_t* user_idx, float* user_w, int* err,
                               cudaStream_t st);
cudaError_t launch_build_perm(const int32_t* idx, int A, int E, const int32_t* hist, int32_t* off,
                              int32_t* perm, int32_t* inv, int* err, cudaStream_t st);
cudaError_t launch_gather_rows(const uint16_t* src, int H, int k, const int32_t* perm, int A,
                               uint16_t* dst, const int32_t* off, int E, const uint16_t* bias,
                               float* dot_out, cudaStream_t st);
cudaError_t launch_combine(const uint16_t* slots, int T, int k, int H, uint16_t* out,
                           cudaStream_t st);
// dw[r] = cbias[r] + sum_p dw_part[p][r]; d_topk_w[perm[r]] = dw[r]  (one thread per row)
cudaError_t launch_reduce_dw(const float* cbias, const float* dw_part, int nparts, int A,
                             const int32_t* perm, float* dw, float* d_topk_w, cudaStream_t st);
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
