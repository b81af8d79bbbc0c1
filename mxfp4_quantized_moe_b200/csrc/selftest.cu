// Self-test of the failure-detection path: a kernel whose mbarrier waits nothing completes.
//
// Every wait in the library's kernels is bounded (mbar_wait: one second of %globaltimer).
// On expiry a wait records MXFP4_MOE_ERR_DEVICE_TIMEOUT and its tag in the workspace error
// word, raises the CTA's abort flag so that the other roles leave their loops, and the kernel
// tears down (TMEM freed) and returns; mxfp4_moe_check then reports the code on the host.
// This kernel drives exactly that path without any fault:
//   warp 0 owns 32 TMEM columns and waits on a barrier that never completes: after the limit
//          it records the timeout (tag 0xF00) and raises the abort flag;
//   warp 1 starts waiting half a second later on another such barrier, so the flag reaches it
//          before its own limit: it must leave through the flag and records that it did in
//          word 2 of the error area;
//   then warp 0 frees its TMEM columns and the kernel returns.
#include "../../include/mxfp4_moe.h"
#include "common.cuh"
#include "kernels.h"
#include "aux_kernels.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(64, 1) wait_timeout_selftest_kernel(int* err_word) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DevErr err{err_word};
  volatile int* abort = &abort_flag;
  if (threadIdx.x == 0) {
    *abort = 0;
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (lane == 0) {
    if (warp == 1) {  // start half a second after warp 0 (bounded by the clock itself)
      const uint64_t t0 = globaltimer();
      while (globaltimer() - t0 < kWaitLimitNs / 2) __nanosleep(100000);
    }
    const bool ok = mbar_wait(smem_u32(&bars[warp]), 0, err, 0xF00 + warp, abort);
    if (warp == 1 && !ok && *abort) err_word[2] = 1;  // left through the abort flag
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*reinterpret_cast<volatile uint32_t*>(&tmem_slot), 32);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int* err_word, cudaStream_t st) {
  wait_timeout_selftest_kernel<<<1, 64, 0, st>>>(err_word);
  return cudaGetLastError();
}

}  // namespace moe
