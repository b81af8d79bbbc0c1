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

// The scratch: MXFP4_MOE_STATIC_SCRATCH_BYTES (64 MiB) of device memory, one copy in every
// context that loads this file's module (under the CUDA 12 default of lazy module loading, the
// first time code of this module runs on that device; with CUDA_MODULE_LOADING=EAGER, on every
// device the library is used on), held until the context is destroyed.
static __device__ __align__(256) unsigned char g_forward_scratch[MXFP4_MOE_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
struct ScratchCache {
  void* ctx;  // the CUcontext the address belongs to
  void* ptr;
};
ScratchCache g_scratch[kMaxDevices] = {};

typedef int (*CtxGetCurrentFn)(void**);

// The driver's cuCtxGetCurrent, looked up through the runtime (the library does not link
// libcuda directly).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

// Device address of g_forward_scratch in the current context.  In host code the array's name
// only stands in for the symbol, so the address is looked up with the device current and
// cached together with the context it belongs to: after a cudaDeviceReset (or any other
// teardown of the primary context) the module is loaded again, possibly at another address,
// and the changed context handle triggers a fresh lookup.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MXFP4_MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MXFP4_MOE_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MXFP4_MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MXFP4_MOE_ERR_UNSUPPORTED_DEVICE;
  CtxGetCurrentFn get = ctx_get_current();
  void* ctx = nullptr;
  if (!get || get(&ctx) != 0) return MXFP4_MOE_ERR_CUDA;
  if (ctx == nullptr) {
    // no context bound to this thread yet: the symbol lookup initializes the device's primary
    // context and binds it
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_forward_scratch) != cudaSuccess) return MXFP4_MOE_ERR_CUDA;
    if (get(&ctx) != 0 || ctx == nullptr) return MXFP4_MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  ScratchCache& c = g_scratch[dev];
  if (c.ptr == nullptr || c.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_forward_scratch) != cudaSuccess || p == nullptr)
      return MXFP4_MOE_ERR_CUDA;
    c.ctx = ctx;
    c.ptr = p;
  }
  *out = c.ptr;
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

extern "C" MXFP4_MOE_API int mxfp4_moe_forward_static_check(void* stream, int32_t* where) {
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  return mxfp4_moe_check(scratch, stream, where);
}
