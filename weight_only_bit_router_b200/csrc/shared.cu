// The dense shared expert beside the routed ones ("Tech2wild/Nex-N2.5-mini-
// Int4-Int8Mix", Recipe table: shared expert gate/up/down_proj and a
// shared_expert_gate; "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", What was
// quantized: shared experts stay bf16).  Its two products run on the tcgen05
// GEMM of gemm_sm100.cu (bf16 weights by TMA); this file holds the step
// between them: the SwiGLU of the gate_up product and the per-token sigmoid
// gate.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// One CTA per token: warp 0 takes the gate's dot product x_t . w_gate (fp32,
// lanes over strided elements, then a butterfly sum), every thread the
// SwiGLU of its features: a = bf16(silu(h_gate) * h_up).
__global__ void __launch_bounds__(256) shared_swiglu_gate_kernel(const uint16_t* __restrict__ x,
                                                                 const uint16_t* __restrict__ w_gate,
                                                                 const float* __restrict__ h, int H, int I,
                                                                 uint16_t* __restrict__ a, float* __restrict__ g) {
  const int t = blockIdx.x;
  const float* ht = h + size_t(t) * 2 * I;
  for (int i = threadIdx.x; i < I; i += blockDim.x)
    a[size_t(t) * I + i] = f32_to_bf16_rn(silu_mul(ht[i], ht[I + i]));
  if (threadIdx.x < 32) {
    const uint16_t* xt = x + size_t(t) * H;
    float z = 0.f;
    for (int k = threadIdx.x; k < H; k += 32) z = fmaf(bf16_to_f32(xt[k]), bf16_to_f32(w_gate[k]), z);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (threadIdx.x == 0) g[t] = 1.0f / (1.0f + expf(-z));
  }
}

}  // namespace

cudaError_t launch_shared_swiglu_gate(const uint16_t* x, const uint16_t* w_gate, const float* h, int T, int H,
                                      int I_s, uint16_t* a, float* g, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  shared_swiglu_gate_kernel<<<T, 256, 0, stream>>>(x, w_gate, h, H, I_s, a, g);
  return cudaGetLastError();
}

}  // namespace moe
