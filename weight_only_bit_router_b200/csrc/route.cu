// Router logits for small batches, top-k routing with renormalised softmax,
// and the stable token->expert permutation (histogram, scan, placement).
//
// Top-8 of 256 routed experts per token: "cbert33/Nex-N2.5-mini-FP8-Calibrated",
// Artifact summary.  The router weight stays bf16 ("Tech2wild/Nex-N2.5-mini-
// Int4-Int8Mix", Recipe table).  Softmax over the selected k and ties to the
// lower expert index are the readings this library takes.
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// ---------------------------------------------------------------------------
// logits[t][e] = sum_h x[t][h] * wr[e][h] for T <= 32 (fp32 accumulation).
// A CTA owns 2 experts; 4 warps split H for each expert; lanes read 16-byte
// chunks of the router row and of every token row.
// ---------------------------------------------------------------------------
constexpr int kRgExpertsPerCta = 2;
constexpr int kRgWarpsPerExpert = 4;

__global__ void __launch_bounds__(256) router_gemv_kernel(const uint16_t* __restrict__ x,
                                                          const uint16_t* __restrict__ wr, int T, int H, int E,
                                                          float* __restrict__ logits) {
  __shared__ float part[kRgExpertsPerCta][kRgWarpsPerExpert][kDecodeMaxT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int le = warp / kRgWarpsPerExpert, ks = warp % kRgWarpsPerExpert;
  const int e = blockIdx.x * kRgExpertsPerCta + le;
  float acc[kDecodeMaxT];
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) acc[t] = 0.f;
  if (e < E) {
    const int span = H / kRgWarpsPerExpert;  // multiple of 16
    const int c0 = ks * span;
    for (int c = c0 + lane * 8; c < c0 + span; c += 256) {
      const uint4 wv = *reinterpret_cast<const uint4*>(wr + size_t(e) * H + c);
      const float w8[8] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y),
                           bf16_lo(wv.z), bf16_hi(wv.z), bf16_lo(wv.w), bf16_hi(wv.w)};
#pragma unroll
      for (int t = 0; t < kDecodeMaxT; ++t) {
        if (t < T) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + size_t(t) * H + c));
          float s = acc[t];
          s = fmaf(w8[0], bf16_lo(xv.x), s); s = fmaf(w8[1], bf16_hi(xv.x), s);
          s = fmaf(w8[2], bf16_lo(xv.y), s); s = fmaf(w8[3], bf16_hi(xv.y), s);
          s = fmaf(w8[4], bf16_lo(xv.z), s); s = fmaf(w8[5], bf16_hi(xv.z), s);
          s = fmaf(w8[6], bf16_lo(xv.w), s); s = fmaf(w8[7], bf16_hi(xv.w), s);
          acc[t] = s;
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kDecodeMaxT; ++t) {
    if (t < T) {
      float s = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) part[le][ks][t] = s;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRgExpertsPerCta * T; i += blockDim.x) {
    const int l = i / T, t = i % T;
    const int ee = blockIdx.x * kRgExpertsPerCta + l;
    if (ee < E) {
      float s = 0.f;
      for (int w = 0; w < kRgWarpsPerExpert; ++w) s += part[l][w][t];
      logits[size_t(t) * E + ee] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// top-k: one warp per token.  Lane l holds experts l, l+32, ... (E <= 1024).
// Each round takes the largest remaining value, ties to the lower index.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                                   int T, int E, int k, int32_t* __restrict__ ids,
                                                   float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  float v[32];
  const int per = (E + 31) / 32;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int e = i * 32 + lane;
    float val = -FLT_MAX;
    if (i < per && e < E) {
      val = logits[size_t(t) * E + e];
      if (bias) val = val + bias[e];  // fp32 add
    }
    v[i] = val;
  }
  uint32_t taken = 0;
  float my_val = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    // local best among untaken entries (smallest index first on ties: i ascending)
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = i * 32 + lane;
      if (i < per && e < E && !((taken >> i) & 1u)) {
        if (v[i] > bv || (v[i] == bv && e < bi)) { bv = v[i]; bi = e; }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) { my_val = bv; my_id = bi; }
  }
  const float vmax = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - vmax) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[size_t(t) * k + lane] = my_id;
    wout[size_t(t) * k + lane] = ex / sum;
  }
}

// Exclusive scan of n <= 1024 ints held in smem by a 1024-thread block; the
// total is returned to every thread.
__device__ int block_exclusive_scan_1024(int* data, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int v = tid < n ? data[tid] : 0;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  if (tid < n) data[tid] = incl - v + warp_tot[warp];
  const int total = warp_tot[32];
  __syncthreads();
  return total;
}

// ---------------------------------------------------------------------------
// Small permutation: one 1024-thread CTA, R = T*k <= 1024 rows.
// Also writes the touched-expert list and the per-expert token-block prefix.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ sorted_rows,
                                                             int32_t* __restrict__ pos,
                                                             int32_t* __restrict__ touched,
                                                             int32_t* __restrict__ tile_base, int block_n) {
  __shared__ int s_ids[1024];
  __shared__ int s_cnt[kMaxExperts];
  __shared__ int s_off[kMaxExperts];
  __shared__ int s_aux[kMaxExperts];
  __shared__ int s_wt[33];
  const int tid = threadIdx.x;
  int my_e = -1;
  if (tid < R) {
    my_e = ids[tid];
    if (my_e < 0 || my_e >= E) my_e = -1;  // contract violation: row dropped
    s_ids[tid] = my_e;
  }
  if (tid < E) s_cnt[tid] = 0;
  __syncthreads();
  if (my_e >= 0) atomicAdd(&s_cnt[my_e], 1);
  __syncthreads();
  if (tid < E) {
    s_off[tid] = s_cnt[tid];
    s_aux[tid] = s_cnt[tid] > 0 ? 1 : 0;
  }
  __syncthreads();
  const int total = block_exclusive_scan_1024(s_off, E, s_wt);
  if (tid < E) offsets[tid] = s_off[tid];
  if (tid == 0) offsets[E] = total;
  // stable rank: rows of the same expert with a lower index
  if (my_e >= 0) {
    int rank = 0;
    for (int r = 0; r < tid; ++r) rank += (s_ids[r] == my_e);
    const int p = s_off[my_e] + rank;
    sorted_rows[p] = tid;
    pos[tid] = p;
  } else if (tid < R) {
    pos[tid] = -1;
  }
  // touched experts, ascending
  const int ntouched = block_exclusive_scan_1024(s_aux, E, s_wt);
  if (tid < E && s_cnt[tid] > 0) touched[1 + s_aux[tid]] = tid;
  if (tid == 0) touched[0] = ntouched;
  // token-block prefix for the grouped GEMMs
  if (tid < E) s_aux[tid] = (s_cnt[tid] + block_n - 1) / block_n;
  __syncthreads();
  const int nblocks = block_exclusive_scan_1024(s_aux, E, s_wt);
  if (tid < E) tile_base[tid] = s_aux[tid];
  if (tid == 0) tile_base[E] = nblocks;
}

// ---------------------------------------------------------------------------
// Large permutation, any R.  Blocks of 256 rows.
// K1: per-block histogram + stable rank of each row inside its block.
// K2: one CTA scans counts over experts and over blocks (bases per block).
// K3: placement.
// ---------------------------------------------------------------------------
constexpr int kPermRows = 256;

__global__ void __launch_bounds__(kPermRows) permute_hist_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                                 int32_t* __restrict__ block_hist,
                                                                 int32_t* __restrict__ row_rank) {
  extern __shared__ int warp_cnt[];  // [8][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = blockIdx.x * kPermRows + tid;
  for (int i = tid; i < 8 * E; i += kPermRows) warp_cnt[i] = 0;
  __syncthreads();
  int e = -1;
  if (r < R) {
    e = ids[r];
    if (e < 0 || e >= E) e = -1;
  }
  const uint32_t m = __match_any_sync(0xffffffffu, e);
  const int rank_w = __popc(m & ((1u << lane) - 1u));
  if (e >= 0 && rank_w == 0) warp_cnt[warp * E + e] = __popc(m);
  __syncthreads();
  if (e >= 0) {
    int rank = rank_w;
    for (int w = 0; w < warp; ++w) rank += warp_cnt[w * E + e];
    row_rank[r] = rank;
  } else if (r < R) {
    row_rank[r] = -1;
  }
  for (int ee = tid; ee < E; ee += kPermRows) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += warp_cnt[w * E + ee];
    block_hist[size_t(blockIdx.x) * E + ee] = s;
  }
}

// G threads per expert (G a power of two, G * E <= 1024) each own a
// contiguous range of row blocks.
__global__ void __launch_bounds__(1024) permute_scan_kernel(int nblk, int E, int G,
                                                            int32_t* __restrict__ block_hist,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ touched,
                                                            int32_t* __restrict__ tile_base, int block_n) {
  __shared__ int s_part[1024];
  __shared__ int s_tot[kMaxExperts];
  __shared__ int s_off[kMaxExperts];
  __shared__ int s_aux[kMaxExperts];
  __shared__ int s_wt[33];
  const int tid = threadIdx.x;
  const int e = tid / G, sub = tid % G;
  const int chunk = (nblk + G - 1) / G;
  const int b0 = min(nblk, sub * chunk), b1 = min(nblk, b0 + chunk);
  int part = 0;
  if (e < E) {
#pragma unroll 8
    for (int b = b0; b < b1; ++b) part += block_hist[size_t(b) * E + e];
  }
  s_part[tid] = part;
  __syncthreads();
  int sub_base = 0;
  if (e < E) {
    for (int s2 = 0; s2 < sub; ++s2) sub_base += s_part[e * G + s2];
  }
  if (tid < E) {
    int tot = 0;
    for (int s2 = 0; s2 < G; ++s2) tot += s_part[tid * G + s2];
    s_tot[tid] = tot;
    s_off[tid] = tot;
    s_aux[tid] = tot > 0 ? 1 : 0;
  }
  __syncthreads();
  const int total = block_exclusive_scan_1024(s_off, E, s_wt);
  if (tid == 0) offsets[E] = total;
  if (tid < E) offsets[tid] = s_off[tid];
  if (e < E) {
    int base = s_off[e] + sub_base;
    for (int b = b0; b < b1; b += 8) {
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = (b + u < b1) ? block_hist[size_t(b + u) * E + e] : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (b + u < b1) {
          block_hist[size_t(b + u) * E + e] = base;
          base += c[u];
        }
      }
    }
  }
  const int ntouched = block_exclusive_scan_1024(s_aux, E, s_wt);
  if (tid < E && s_tot[tid] > 0) touched[1 + s_aux[tid]] = tid;
  if (tid == 0) touched[0] = ntouched;
  if (tid < E) s_aux[tid] = (s_tot[tid] + block_n - 1) / block_n;
  __syncthreads();
  const int nblocks = block_exclusive_scan_1024(s_aux, E, s_wt);
  if (tid < E) tile_base[tid] = s_aux[tid];
  if (tid == 0) tile_base[E] = nblocks;
}

__global__ void __launch_bounds__(kPermRows) permute_place_kernel(const int32_t* __restrict__ ids, int R, int E,
                                                                  const int32_t* __restrict__ block_base,
                                                                  int32_t* __restrict__ sorted_rows,
                                                                  int32_t* __restrict__ pos) {
  const int r = blockIdx.x * kPermRows + threadIdx.x;
  if (r >= R) return;
  const int e = ids[r];
  const int rank = pos[r];  // the row rank K1 stored here
  if (e < 0 || e >= E || rank < 0) {
    pos[r] = -1;
    return;
  }
  const int p = block_base[size_t(blockIdx.x) * E + e] + rank;
  sorted_rows[p] = r;
  pos[r] = p;
}

}  // namespace

size_t permute_block_rows() { return kPermRows; }

size_t permute_large_hist_bytes(int T, int E, int k) {
  const size_t R = size_t(T) * k;
  const size_t nblk = (R + kPermRows - 1) / kPermRows;
  return nblk * size_t(E) * sizeof(int32_t);
}

cudaError_t launch_router_gemv(const uint16_t* x, const uint16_t* wr, int T, int H, int E, float* logits,
                               cudaStream_t stream) {
  const int grid = (E + kRgExpertsPerCta - 1) / kRgExpertsPerCta;
  router_gemv_kernel<<<grid, 32 * kRgExpertsPerCta * kRgWarpsPerExpert, 0, stream>>>(x, wr, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int warps_per_block = 8;
  const int grid = (T + warps_per_block - 1) / warps_per_block;
  topk_kernel<<<grid, 32 * warps_per_block, 0, stream>>>(logits, bias, T, E, k, ids, w);
  return cudaGetLastError();
}

cudaError_t launch_permute_small(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* sorted_rows,
                                 int32_t* pos, int32_t* touched, int32_t* tile_base, int block_n,
                                 cudaStream_t stream) {
  permute_small_kernel<<<1, 1024, 0, stream>>>(ids, T * k, E, offsets, sorted_rows, pos, touched, tile_base,
                                               block_n);
  return cudaGetLastError();
}

cudaError_t launch_permute_large(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* sorted_rows,
                                 int32_t* pos, int32_t* block_hist, int32_t* touched, int32_t* tile_base,
                                 int block_n, cudaStream_t stream) {
  const int R = T * k;
  const int nblk = (R + kPermRows - 1) / kPermRows;
  if (nblk == 0) return cudaSuccess;
  const size_t smem = size_t(8) * E * sizeof(int);
  permute_hist_kernel<<<nblk, kPermRows, smem, stream>>>(ids, R, E, block_hist, pos);
  int G = 1;
  while (G * 2 * E <= 1024) G *= 2;
  permute_scan_kernel<<<1, 1024, 0, stream>>>(nblk, E, G, block_hist, offsets, touched, tile_base, block_n);
  permute_place_kernel<<<nblk, kPermRows, 0, stream>>>(ids, R, E, block_hist, sorted_rows, pos);
  return cudaGetLastError();
}

}  // namespace moe
