// Host-side launch helper: kernels of the forward pass are launched with
// programmatic stream serialization, so that a kernel's CTAs may be scheduled
// while its predecessor drains; each kernel waits (griddepcontrol.wait) before
// it reads anything the predecessor writes.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <utility>

namespace moe {

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Cooperative launch (every CTA resident at once, so CTAs may wait on one
// another), with programmatic stream serialization when the driver accepts
// both attributes together.
template <typename... KArgs, typename... Args>
cudaError_t launch_cooperative(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               Args&&... args) {
  static std::atomic<int> with_pdl{1};  // cleared once the driver refuses the combination
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = with_pdl.load() ? 2 : 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (err != cudaSuccess && cfg.numAttrs == 2) {
    (void)cudaGetLastError();
    with_pdl.store(0);
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  }
  return err;
}

}  // namespace moe
