// The dense shared expert beside the routed ones ("Tech2wild/Nex-N2.5-mini-
// Int4-Int8Mix", Recipe table: shared expert gate/up/down_proj and a
// shared_expert_gate; "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", What was
// quantized: shared experts stay bf16).  For more than 32 tokens its two
// products run on the tcgen05 GEMM of gemm_sm100.cu (bf16 weights by TMA);
// for up to 32 tokens on the split-K mma.sync product below, which spreads
// the weight rows over a few hundred CTAs.  Between them: the SwiGLU of the
// gate_up product and the per-token sigmoid gate.
#include "common.cuh"
#include "decode_common.cuh"
#include "internal.h"
#include "launch.h"

namespace moe {

namespace {

// ---------------------------------------------------------------------------
// Small-batch product (T <= 32): part[s][t][n] = sum over k-split s of
// W[n][k] x[t][k], bf16 W [N][K] and x [T][K] (row stride K), fp32.  One CTA
// per (16 rows, 512 k); each of its four warps takes one 128-k block of the
// 16 rows with mma.sync m16n8k16 for every token tile of 8, and the four
// partial tiles are summed in warp order.  The weight rows are read once;
// the splits are summed (in order) by the consumer.
// ---------------------------------------------------------------------------
constexpr int kSgK = 512;  // k per CTA

// 16 words (32 bf16) at p, in the fragment k-permutation of decode_common.cuh.
MOE_DEV void bf16_slice_frags(const uint16_t* p, bool valid, uint32_t (&b)[8][2]) {
  uint32_t X[16];
  if (valid) {
    const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 u = __ldg(v + i);
      X[4 * i] = u.x; X[4 * i + 1] = u.y; X[4 * i + 2] = u.z; X[4 * i + 3] = u.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
  act_frags_from_raw(X, b);
}

template <int NT>
__global__ void __launch_bounds__(128) shared_gemv_kernel(const uint16_t* __restrict__ x,
                                                          const uint16_t* __restrict__ w, int T, int K, int N,
                                                          float* __restrict__ part) {
  __shared__ float red[4][NT][4][32];
  pdl_wait();  // the previous kernel on the stream may still read `part`
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int n0 = blockIdx.x * 16;
  const int k = blockIdx.y * kSgK + warp * 128 + 32 * q;  // this lane's 32-k slice
  const bool kin = k < K;                                  // K % 64 == 0: whole slices
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
  uint32_t alo[8][2], ahi[8][2];
  bf16_slice_frags(w + size_t(n0 + g) * K + k, kin, alo);
  bf16_slice_frags(w + size_t(n0 + g + 8) * K + k, kin, ahi);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int t = 8 * j + g;
    uint32_t bf[8][2];
    bf16_slice_frags(x + size_t(t < T ? t : 0) * K + k, kin && t < T, bf);
#pragma unroll
    for (int st = 0; st < 8; ++st) {
      const uint32_t a[4] = {alo[st][0], ahi[st][0], alo[st][1], ahi[st][1]};
      mma_bf16_16816(acc[j], a, bf[st][0], bf[st][1]);
    }
  }
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][j][c][lane] = acc[j][c];
  __syncthreads();
  for (int idx = threadIdx.x; idx < NT * 4 * 32; idx += blockDim.x) {
    const int j = idx / 128, c = (idx / 32) & 3, l = idx & 31;
    const float v = red[0][j][c][l] + red[1][j][c][l] + red[2][j][c][l] + red[3][j][c][l];
    // C fragment: c0, c1 row g, tokens 2q, 2q+1; c2, c3 row g + 8
    const int row = n0 + (l >> 2) + (c >> 1) * 8, tok = 8 * j + 2 * (l & 3) + (c & 1);
    if (tok < T) part[(size_t(blockIdx.y) * T + tok) * N + row] = v;
  }
}

// One CTA per token: warp 0 takes the gate's dot product x_t . w_gate (fp32,
// lanes over strided elements, then a butterfly sum), every thread the
// SwiGLU of its features: a = bf16(silu(h_gate) * h_up).
// h holds `splits` partial products [splits][T][2I] summed here in split order.
__global__ void __launch_bounds__(256) shared_swiglu_gate_kernel(const uint16_t* __restrict__ x,
                                                                 const uint16_t* __restrict__ w_gate,
                                                                 const float* __restrict__ h, int splits, int T,
                                                                 int H, int I, uint16_t* __restrict__ a,
                                                                 float* __restrict__ g) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < I; i += blockDim.x) {
    float hg = 0.f, hu = 0.f;
    for (int sp = 0; sp < splits; ++sp) {
      const float* ht = h + (size_t(sp) * T + t) * 2 * I;
      hg += ht[i];
      hu += ht[I + i];
    }
    a[size_t(t) * I + i] = f32_to_bf16_rn(silu_mul(hg, hu));
  }
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

int shared_gemv_splits(int K) { return (K + kSgK - 1) / kSgK; }

cudaError_t launch_shared_gemv(const uint16_t* x, const uint16_t* w, int T, int K, int N, float* part,
                               cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const dim3 grid(N / 16, shared_gemv_splits(K));
  if (T <= 8) return launch_pdl(shared_gemv_kernel<1>, grid, dim3(128), 0, stream, x, w, T, K, N, part);
  if (T <= 16) return launch_pdl(shared_gemv_kernel<2>, grid, dim3(128), 0, stream, x, w, T, K, N, part);
  return launch_pdl(shared_gemv_kernel<4>, grid, dim3(128), 0, stream, x, w, T, K, N, part);
}

cudaError_t launch_shared_swiglu_gate(const uint16_t* x, const uint16_t* w_gate, const float* h, int splits, int T,
                                      int H, int I_s, uint16_t* a, float* g, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  return launch_pdl(shared_swiglu_gate_kernel, dim3(T), dim3(256), 0, stream, x, w_gate, h, splits, T, H, I_s, a, g);
}

}  // namespace moe
