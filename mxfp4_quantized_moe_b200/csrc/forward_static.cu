// Forward of the expert block for callers that cannot allocate device memory.
//
// Some callers of this library hold no device allocator at the point where they run the
// layer: an inference-engine plugin whose enqueue step receives only input and output
// pointers, a process whose device memory is owned by another framework's pool, or a
// latency-critical serving loop that must not pay for cudaMalloc's implicit device
// synchronization.  For them, mxfp4_moe_forward_static runs the ordinary forward
// (mxfp4_moe_forward, unchanged) with its workspace in a fixed array that lives in this
// file, instead of a caller-provided one.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/mxfp4_moe.h"

// The scratch: MXFP4_MOE_STATIC_SCRATCH_BYTES (64 MiB) of device memory, one copy per GPU
// that loads this code (with the CUDA 12 default of lazy module loading, a GPU gets it the
// first time this entry point runs there), held until the process exits.
static __device__ __align__(256) unsigned char g_forward_scratch[MXFP4_MOE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_forward_scratch on the current device.  In host code the array's
// name only stands in for the symbol, so the address is looked up once per device (with
// that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXFP4_MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MXFP4_MOE_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MXFP4_MOE_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_forward_scratch) != cudaSuccess || p == nullptr)
      return MXFP4_MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MXFP4_MOE_OK;
}

}  // namespace

extern "C" MXFP4_MOE_API int mxfp4_moe_forward_static(const mxfp4_moe_dims* d,
                                                      const mxfp4_moe_weights* w,
                                                      const uint16_t* x, const float* logits,
                                                      uint16_t* y, int32_t* topk_idx,
                                                      float* topk_w, void* stream) {
  size_t need = 0;
  int rc = mxfp4_moe_workspace_size(d, &need);
  if (rc) return rc;
  if (need > MXFP4_MOE_STATIC_SCRATCH_BYTES) return MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc) return rc;
  // the array keeps the previous call's contents: start this call with a clear error word
  // (the forward itself zeroes the routing histogram it accumulates into)
  if (cudaMemsetAsync(scratch, 0, 16, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  return mxfp4_moe_forward(d, w, x, logits, y, topk_idx, topk_w, scratch,
                           MXFP4_MOE_STATIC_SCRATCH_BYTES, stream);
}
