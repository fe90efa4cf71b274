// moe_forward_noalloc: the layer forward for callers that cannot allocate
// device memory, running on a fixed scratch array that lives in the library
// image itself.
//
// Who needs this: inference runtimes that reserve their whole device-memory
// budget at start-up, plugins whose host framework owns the device allocator,
// and code that records its GPU work for later replay (an allocation inside
// the recorded region is not allowed) cannot call cudaMalloc per call.  They
// pass only inputs and outputs here.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes that
// every GPU which loads the library holds until the process exits.  In host
// code the array's name is only a host-side stand-in, so the device address
// is looked up with cudaGetSymbolAddress, with the device current, on the
// first call made on that device (and again if the device's context was
// re-created since, e.g. after cudaDeviceReset); make that first call before
// any stream capture.  All calls on a device share the array and it keeps the
// previous call's contents: each call clears the device counters it needs at
// zero, and calls whose executions overlap on the GPU (different streams
// without ordering between them) race on the array.  The status word at the
// start of the array is not cleared by a call: an expired bounded wait stays
// recorded there until moe_noalloc_status reports it.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchEntry {
  unsigned long long ctx_id;  // the context the address belongs to (0: unknown)
  void* ptr;
};

std::mutex g_noalloc_mutex;
ScratchEntry g_noalloc[kMaxDevices] = {};

// Driver calls that identify the current context (resolved once; null when the
// driver does not offer them, in which case the address is looked up once per
// device and not refreshed).
struct CtxCalls {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxCalls& ctx_calls() {
  static const CtxCalls calls = [] {
    CtxCalls c;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    return c;
  }();
  return calls;
}

// Unique id of the current context, 0 if there is none or it cannot be read.
unsigned long long current_ctx_id() {
  const CtxCalls& c = ctx_calls();
  if (!c.get_current || !c.get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (c.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (c.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace

cudaError_t noalloc_scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  ScratchEntry& e = g_noalloc[dev];
  const unsigned long long id = current_ctx_id();
  if (!e.ptr || (id != 0 && id != e.ctx_id)) {
    // set-up for this device (or its new context): not while capturing
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if ((err = cudaStreamIsCapturing(stream, &cs)) != cudaSuccess) return err;
    if (cs != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    void* p = nullptr;
    if ((err = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return err;
    e.ptr = p;
    e.ctx_id = current_ctx_id();  // the lookup made the context current if it was not
  }
  *out = e.ptr;
  return cudaSuccess;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

moe_status_t moe_forward_noalloc(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                                 const float* logit_bias, const void* gate_up_packed, const void* down_packed,
                                 uint16_t* out, cudaStream_t stream) {
  // every argument check comes before anything is enqueued
  moe_status_t st = check_forward_args(shape, x, T, router_w, logit_bias, gate_up_packed, down_packed, out);
  if (st != MOE_OK) return st;
  if (moe_workspace_bytes(shape, T) > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;  // batch too large
  if (T == 0) return MOE_OK;
  void* scratch = nullptr;
  if (noalloc_scratch_address(stream, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
  // the device counters after the status word must start at zero; the status
  // word itself keeps an earlier timeout until moe_noalloc_status reports it
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + sizeof(uint32_t), 0, kStatusBytes - sizeof(uint32_t),
                      stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_forward(shape, x, T, router_w, logit_bias, gate_up_packed, down_packed, scratch, kNoAllocScratchBytes,
                     out, nullptr, stream);
}

moe_status_t moe_noalloc_status(cudaStream_t stream) {
  void* scratch = nullptr;
  if (noalloc_scratch_address(stream, &scratch) != cudaSuccess) return MOE_ERR_CUDA;
  return moe_workspace_status(scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
