// moe_forward_noalloc: the layer forward for callers that cannot allocate
// device memory, running on a fixed scratch array that lives in the library
// image itself.
//
// Who needs this: callers that record their GPU work ahead of time and
// replay it later (a captured CUDA graph, or an engine that replays
// pre-built command buffers) cannot call cudaMalloc inside the recorded
// region; runtimes that reserve their whole memory budget at start-up, and
// plugins whose host framework owns the device allocator, cannot allocate
// per call either.  They pass only inputs and outputs here.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes that
// every GPU which loads the library holds until the process exits.  In host
// code the array's name is only a host-side stand-in, so the device address
// is looked up with cudaGetSymbolAddress once per device (with that device
// current) on the first call made on that device; make that first call before
// any stream capture.  All calls on a device share the array and it keeps the
// previous call's contents: each call clears the status/counter region it
// needs at zero, and calls whose executions overlap on the GPU (different
// streams without ordering between them) race on the array.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

moe_status_t moe_forward_noalloc(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                                 const float* logit_bias, const void* gate_up_packed, const void* down_packed,
                                 uint16_t* out, cudaStream_t stream) {
  const size_t need = moe_workspace_bytes(shape, T);
  if (need == 0) return shape == nullptr || T < 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  if (need > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;  // batch too large for the fixed scratch
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // the status word and the completion counters must start at zero
  if (cudaMemsetAsync(scratch, 0, kStatusBytes, stream) != cudaSuccess) return MOE_ERR_CUDA;
  return moe_forward(shape, x, T, router_w, logit_bias, gate_up_packed, down_packed, scratch, kNoAllocScratchBytes,
                     out, nullptr, stream);
}

}  // extern "C"
