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

// One CTA whose mbarrier waits nothing completes: exercises the bounded-wait path (tag 0xF00
// in the error word after about one second) without any fault.
cudaError_t launch_wait_timeout_selftest(int* err_word, cudaStream_t st);

}  // namespace moe
