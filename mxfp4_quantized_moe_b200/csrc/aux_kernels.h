// Internal launch interface of the library's auxiliary kernels (layout helper, self-test);
// not part of the public C ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

// Stacked gate_up rows [gates; ups] -> interleaved rows (gate j at 2j, up j at 2j+1) for
// packed bytes [E][2I][K/2], scales [E][2I][K/32] and bias [E][2I]; K = H.
cudaError_t launch_interleave_gate_up(const uint8_t* sb, const uint8_t* ss, const uint16_t* sbias,
                                      int E, int I, int K, uint8_t* db, uint8_t* ds,
                                      uint16_t* dbias, cudaStream_t st);

// The residual stream around stacked blocks: x_out = bf16(x + y) (y null: no residual and no
// x_out) and logits = (y ? x_out : x) W_r + b_r in fp32 (logits null: no router); w_r bf16
// [H][E], b_r bf16 [E] or null.  H % 32 == 0, 1 <= E <= 256.
cudaError_t launch_residual_router(int T, int H, int E, const uint16_t* x, const uint16_t* y,
                                   const uint16_t* w_r, const uint16_t* b_r, uint16_t* x_out,
                                   float* logits, cudaStream_t st);
// g_out = bf16(g + dx + d_logits W_r^T), fp32 arithmetic; g_out may alias g.
cudaError_t launch_grad_chain(int T, int H, int E, const uint16_t* g, const uint16_t* dx,
                              const float* d_logits, const uint16_t* w_r, uint16_t* g_out,
                              cudaStream_t st);

// One CTA whose mbarrier waits nothing completes: exercises the bounded-wait path (tag 0xF00
// in the error word after about one second) without any fault.
cudaError_t launch_wait_timeout_selftest(int* err_word, cudaStream_t st);

}  // namespace moe
