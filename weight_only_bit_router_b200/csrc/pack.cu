// Packing of bf16 expert banks into the two 4-bit formats, and the debug
// dequantiser.  One warp quantises 128 consecutive K elements of one row
// (one INT4 group, or four MXFP4 blocks); each lane owns 4 elements.
//
// INT4: "Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe (symmetric, group 128,
//       round-to-nearest with min-max scales).
// MXFP4: "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Model summary and
//       Quantization method (E2M1 codes, E8M0 scale per 32 elements,
//       exponent floor(log2(amax / 6))).
#include <cuda_fp8.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// One warp per (row, 128-column chunk).  Lane l owns columns c0+4l .. c0+4l+3.
__global__ void __launch_bounds__(256) pack_int4_kernel(const uint16_t* __restrict__ w, long rows, int K,
                                                        uint8_t* __restrict__ codes, uint16_t* __restrict__ scales,
                                                        int32_t* nonfinite) {
  const int lane = threadIdx.x & 31;
  const int G = (K + 127) / 128;
  const long task = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (task >= rows * G) return;
  const long row = task / G;
  const int g = int(task % G);
  const int col = g * 128 + lane * 4;
  const bool active = col < K;  // K % 4 == 0: a lane is wholly in or out
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) {
    const uint2 raw = *reinterpret_cast<const uint2*>(w + row * K + col);
    v[0] = bf16_lo(raw.x); v[1] = bf16_hi(raw.x); v[2] = bf16_lo(raw.y); v[3] = bf16_hi(raw.y);
  }
  float amax = 0.f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bad |= !isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (bad && nonfinite) atomicAdd(nonfinite, 1);
  // s = bf16(fp32(amax) / 7): the group max maps to +-7
  const uint16_t s_bits = f32_to_bf16_rn(__fdiv_rn(amax, 7.0f));
  const float s = bf16_to_f32(s_bits);
  if (!active) return;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int q = 0;
    if (s != 0.f) q = max(-8, min(7, __float2int_rn(__fdiv_rn(v[i], s))));
    packed |= uint32_t(q + 8) << (4 * i);
  }
  *reinterpret_cast<uint16_t*>(codes + row * (K / 2) + col / 2) = uint16_t(packed);
  if (lane == 0) scales[row * G + g] = s_bits;
}

// E2M1 magnitude code of a non-negative fp32 v: nearest of {0,.5,1,1.5,2,3,4,6},
// ties to the even code, saturating at 6.
__device__ __forceinline__ uint32_t e2m1_code(float a) {
  if (a <= 0.25f) return 0;
  if (a < 0.75f) return 1;
  if (a <= 1.25f) return 2;
  if (a < 1.75f) return 3;
  if (a <= 2.5f) return 4;
  if (a < 3.5f) return 5;
  if (a <= 5.0f) return 6;
  return 7;
}

// floor(log2(amax / 6)) for amax > 0, computed exactly from the fp32 bits:
// amax = m * 2^E with m in [1, 2); 6 * 2^(E-2) <= amax iff m >= 1.5.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int bias = 0;
  if (amax < 1e-30f) { amax *= 18446744073709551616.0f; bias = 64; }  // 2^64, exact
  const uint32_t b = __float_as_uint(amax);
  const int E = int((b >> 23) & 0xFF) - 127 - bias;
  const int e = ((b & 0x7FFFFF) >= 0x400000u) ? E - 2 : E - 3;
  return max(-127, min(127, e));
}

// 2^p as fp32 for p in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2i(int p) {
  return p >= -126 ? __uint_as_float(uint32_t(p + 127) << 23) : __uint_as_float(0x00400000u);
}

// One warp per (row, 128 columns) = 4 MXFP4 blocks; lanes 8b..8b+7 own block b.
__global__ void __launch_bounds__(256) pack_mxfp4_kernel(const uint16_t* __restrict__ w, long rows, int K,
                                                         uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                         int32_t* nonfinite) {
  const int lane = threadIdx.x & 31;
  const int C = (K + 127) / 128;
  const long task = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (task >= rows * C) return;
  const long row = task / C;
  const int col = int(task % C) * 128 + lane * 4;
  const bool active = col < K;  // K % 32 == 0: a block of 8 lanes is wholly in or out
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) {
    const uint2 raw = *reinterpret_cast<const uint2*>(w + row * K + col);
    v[0] = bf16_lo(raw.x); v[1] = bf16_hi(raw.x); v[2] = bf16_lo(raw.y); v[3] = bf16_hi(raw.y);
  }
  float amax = 0.f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bad |= !isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (bad && nonfinite) atomicAdd(nonfinite, 1);
  if (!active) return;
  const int e = mx_exponent(amax);
  const float inv = exp2i(-e);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x = v[i] * inv;  // exact whenever it matters (|x| >= 2^-126)
    const uint32_t c = e2m1_code(fabsf(x));
    const uint32_t sgn = (v[i] < 0.f && c != 0) ? 8u : 0u;
    packed |= (sgn | c) << (4 * i);
  }
  *reinterpret_cast<uint16_t*>(codes + row * (K / 2) + col / 2) = uint16_t(packed);
  if ((lane & 7) == 0) scales[row * (K / 32) + col / 32] = uint8_t(e + 127);
}

// ---------------------------------------------------------------------------
// MXFP4 with a selectable exponent rule (the floor(log2(x / 6)) family of
// "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Quantization method).  One
// warp per block of 32; lane i owns element i.  The MSE rule evaluates its
// candidates in fp64 with explicitly rounded operations (no contraction), so
// that its integer decision is reproducible.
// ---------------------------------------------------------------------------

// ceil(log2(amax / 6)) for amax > 0: amax = m * 2^E, m in [1, 2);
// 6 * 2^(E-2) = 1.5 * 2^E >= amax iff m <= 1.5, else 6 * 2^(E-1) >= amax.
__device__ __forceinline__ int mx_exponent_ceil(float amax) {
  if (!(amax > 0.f)) return -127;
  int bias = 0;
  if (amax < 1e-30f) { amax *= 18446744073709551616.0f; bias = 64; }  // 2^64, exact
  const uint32_t b = __float_as_uint(amax);
  const int E = int((b >> 23) & 0xFF) - 127 - bias;
  const int e = ((b & 0x7FFFFF) <= 0x400000u) ? E - 2 : E - 1;
  return max(-127, min(127, e));
}

// floor(log2(amax)) - 2 for amax > 0.
__device__ __forceinline__ int mx_exponent_ocp(float amax) {
  if (!(amax > 0.f)) return -127;
  int bias = 0;
  if (amax < 1e-30f) { amax *= 18446744073709551616.0f; bias = 64; }
  const int E = int((__float_as_uint(amax) >> 23) & 0xFF) - 127 - bias;
  return max(-127, min(127, E - 2));
}

// Largest e with 6 * 2^e <= p for a normal fp64 p > 0: p = m * 2^E, m in
// [1, 2); 6 * 2^(E-2) <= p iff m >= 1.5.
__device__ __forceinline__ int mx_exponent_f64(double p) {
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(p));
  const int E = int((b >> 52) & 0x7FF) - 1023;
  return (b & (1ull << 51)) ? E - 2 : E - 3;
}

__device__ __forceinline__ double exp2i_f64(int p) {  // 2^p, p in [-1022, 1023]
  return __longlong_as_double(static_cast<long long>(p + 1023) << 52);
}

// E2M1 magnitude code of a non-negative fp64 a (same thresholds as e2m1_code).
__device__ __forceinline__ uint32_t e2m1_code_f64(double a) {
  if (a <= 0.25) return 0;
  if (a < 0.75) return 1;
  if (a <= 1.25) return 2;
  if (a < 1.75) return 3;
  if (a <= 2.5) return 4;
  if (a < 3.5) return 5;
  if (a <= 5.0) return 6;
  return 7;
}

__constant__ double kE2m1Grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// Sum over the warp of the squared error of quantising this lane's w with
// exponent e; pairwise in halving order, identical in every lane.
__device__ __forceinline__ double mx_block_sq_error(double w, int e) {
  const double a = fabs(w) * exp2i_f64(-e);  // exact power-of-two scaling
  const double mag = kE2m1Grid[e2m1_code_f64(a)] * exp2i_f64(e);
  const double d = __dsub_rn(w, w < 0.0 ? -mag : mag);  // exact
  double sq = __dmul_rn(d, d);                          // exact
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq = __dadd_rn(sq, __shfl_xor_sync(0xffffffffu, sq, o));
  return sq;
}

__global__ void __launch_bounds__(256) pack_mxfp4_rule_kernel(const uint16_t* __restrict__ w, long nblocks,
                                                              uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ scales, int32_t* nonfinite,
                                                              int rule) {
  const unsigned full = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const long blk = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (blk >= nblocks) return;
  const float v = bf16_to_f32(w[blk * 32 + lane]);
  if (!isfinite(v) && nonfinite) atomicAdd(nonfinite, 1);
  const float a = fabsf(v);
  // magnitudes are non-negative: their fp32 bit patterns order like the values
  const float amax = __uint_as_float(__reduce_max_sync(full, __float_as_uint(a)));
  int e;
  if (!(amax > 0.f)) {
    e = -127;
  } else if (rule == MOE_MX_EXP_CEIL) {
    e = mx_exponent_ceil(amax);
  } else if (rule == MOE_MX_EXP_OCP) {
    e = mx_exponent_ocp(amax);
  } else if (rule == MOE_MX_EXP_MSE) {
    // 99.5th percentile of the 32 magnitudes: v30 + 0.845 * (v31 - v30)
    const int n_max = __popc(__ballot_sync(full, a == amax));
    const float v30 = n_max >= 2 ? amax
                                 : __uint_as_float(__reduce_max_sync(full, a == amax ? 0u : __float_as_uint(a)));
    const double p = __dadd_rn(double(v30), __dmul_rn(__dsub_rn(double(amax), double(v30)), 0.845));
    const int e0 = mx_exponent_f64(p);
    const double wv = double(v);
    e = max(-127, min(127, e0 - 4));
    double best = mx_block_sq_error(wv, e);
    for (int d = -3; d <= 2; ++d) {  // e0 - 3 ... e0 + 1, then the no-clip exponent
      const int c = d <= 1 ? max(-127, min(127, e0 + d)) : mx_exponent_ceil(amax);
      const double err = mx_block_sq_error(wv, c);
      if (err < best) {
        best = err;
        e = c;
      }
    }
  } else {
    e = mx_exponent(amax);
  }
  const float x = v * exp2i(-e);  // exact whenever it matters (|x| >= 2^-126)
  const uint32_t c = e2m1_code(fabsf(x));
  const uint32_t nib = ((v < 0.f && c != 0) ? 8u : 0u) | c;
  const uint32_t hi = __shfl_down_sync(full, nib, 1);
  if ((lane & 1) == 0) codes[blk * 16 + lane / 2] = uint8_t(nib | (hi << 4));
  if (lane == 0) scales[blk] = uint8_t(e + 127);
}

// ---------------------------------------------------------------------------
// NVFP4 as W4A16 ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", What's
// quantized to what: group 16, one global scale per expert shared by gate and
// up, weights-only round-to-nearest).  Three steps: the maximum magnitude of
// every matrix (as fp32 bits, atomically, into the global-scale slots), the
// global scales g = fp32(amax / 2688) in place, then codes and E4M3 block
// scales (one warp per (row, 128 columns); four lanes per block of 16).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) nv_amax_kernel(const uint16_t* __restrict__ w, long per_matrix,
                                                      uint32_t* __restrict__ amax_bits) {
  const int e = blockIdx.y;
  const uint16_t* m = w + long(e) * per_matrix;
  uint32_t mx = 0;
  for (long i = long(blockIdx.x) * blockDim.x + threadIdx.x; i < per_matrix; i += long(gridDim.x) * blockDim.x) {
    const float v = fabsf(bf16_to_f32(m[i]));
    if (isfinite(v)) mx = max(mx, __float_as_uint(v));  // non-negative floats order like their bits
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if ((threadIdx.x & 31) == 0 && mx) atomicMax(&amax_bits[e], mx);
}

__global__ void nv_gscale_kernel(uint32_t* __restrict__ slots, int E) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) reinterpret_cast<float*>(slots)[e] = __fdiv_rn(__uint_as_float(slots[e]), 2688.0f);
}

__global__ void __launch_bounds__(256) pack_nvfp4_kernel(const uint16_t* __restrict__ w, long rows, int N, int K,
                                                         uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                         const float* __restrict__ gscale, int32_t* nonfinite) {
  const int lane = threadIdx.x & 31;
  const int C = (K + 127) / 128;
  const long task = (long(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (task >= rows * C) return;
  const long row = task / C;
  const int col = int(task % C) * 128 + lane * 4;
  const bool active = col < K;  // K % 32 == 0: a block of 4 lanes is wholly in or out
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) {
    const uint2 raw = *reinterpret_cast<const uint2*>(w + row * K + col);
    v[0] = bf16_lo(raw.x); v[1] = bf16_hi(raw.x); v[2] = bf16_lo(raw.y); v[3] = bf16_hi(raw.y);
  }
  float amax = 0.f;
  int bad = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bad |= !isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (bad && nonfinite) atomicAdd(nonfinite, 1);
  if (!active) return;
  const float g = gscale[row / N];
  const float six_g = __fmul_rn(6.0f, g);
  const float t = six_g == 0.f ? 0.f : __fdiv_rn(amax, six_g);
  // nearest E4M3, ties to even, saturating at 448
  const uint32_t code = uint32_t(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
  const float d = bf16_to_f32(uint16_t(nv_mult_bits(code, g)));
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c = d == 0.f ? 0u : e2m1_code(fabsf(__fdiv_rn(v[i], d)));
    const uint32_t sgn = (v[i] < 0.f && c != 0) ? 8u : 0u;
    packed |= (sgn | c) << (4 * i);
  }
  *reinterpret_cast<uint16_t*>(codes + row * (K / 2) + col / 2) = uint16_t(packed);
  if ((lane & 3) == 0) scales[row * (K / 16) + col / 16] = uint8_t(code);
}

// Debug dequantiser: one thread per code byte (two elements).
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const void* __restrict__ scales,
                               const float* __restrict__ gscale, int fmt, long rows, int N, int K,
                               uint16_t* __restrict__ out) {
  const long i = long(blockIdx.x) * blockDim.x + threadIdx.x;
  const long nbytes = rows * (K / 2);
  if (i >= nbytes) return;
  const long row = i / (K / 2);
  const int col = int(i % (K / 2)) * 2;
  const uint32_t byte = codes[i];
  uint16_t r[2];
  for (int h = 0; h < 2; ++h) {
    const uint32_t nib = (byte >> (4 * h)) & 15u;
    const int k = col + h;
    float val;
    if (fmt == MOE_FMT_INT4_G128) {
      const int G = (K + 127) / 128;
      const float s = bf16_to_f32(static_cast<const uint16_t*>(scales)[row * G + k / 128]);
      val = float(int(nib) - 8) * s;  // exact in fp32, rounded once below
    } else if (fmt == MOE_FMT_NVFP4_G16) {
      const uint32_t sbyte = static_cast<const uint8_t*>(scales)[row * (K / 16) + k / 16];
      const float d = bf16_to_f32(uint16_t(nv_mult_bits(sbyte, gscale[row / N])));
      const float mags[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
      val = mags[nib & 7u] * d;  // exact in fp32, rounded once below
      if (nib & 8u) val = -val;
    } else {
      const int e = int(static_cast<const uint8_t*>(scales)[row * (K / 32) + k / 32]) - 127;
      const float mags[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
      val = mags[nib & 7u] * exp2i(e);  // exact (subnormal products included)
      if (nib & 8u) val = -val;
    }
    r[h] = f32_to_bf16_rn(val);
  }
  *reinterpret_cast<uint32_t*>(out + row * K + col) = uint32_t(r[0]) | (uint32_t(r[1]) << 16);
}

}  // namespace

cudaError_t launch_pack(moe_format_t fmt, const uint16_t* w, int E, int N, int K, void* packed,
                        int32_t* nonfinite, cudaStream_t stream) {
  const long rows = long(E) * N;
  const long chunks = rows * ((K + 127) / 128);
  const long threads = chunks * 32;
  const int block = 256;
  const long grid = (threads + block - 1) / block;
  uint8_t* codes = static_cast<uint8_t*>(packed);
  void* scales = static_cast<uint8_t*>(packed) + bank_scale_offset(fmt, E, N, K);
  if (grid == 0) return cudaSuccess;
  if (fmt == MOE_FMT_NVFP4_G16) {
    uint32_t* slots = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(packed) + bank_gscale_offset(fmt, E, N, K));
    cudaError_t err = cudaMemsetAsync(slots, 0, size_t(E) * 4, stream);
    if (err != cudaSuccess) return err;
    const long per_matrix = long(N) * K;
    const int bx = int(std::min<long>(64, (per_matrix + 255) / 256));
    nv_amax_kernel<<<dim3(bx, E), 256, 0, stream>>>(w, per_matrix, slots);
    nv_gscale_kernel<<<(E + 255) / 256, 256, 0, stream>>>(slots, E);
    pack_nvfp4_kernel<<<dim3(unsigned(grid)), block, 0, stream>>>(w, rows, N, K, codes, static_cast<uint8_t*>(scales),
                                                                  reinterpret_cast<const float*>(slots), nonfinite);
    return cudaGetLastError();
  }
  if (fmt == MOE_FMT_INT4_G128)
    pack_int4_kernel<<<dim3(unsigned(grid)), block, 0, stream>>>(w, rows, K, codes, static_cast<uint16_t*>(scales),
                                                                 nonfinite);
  else
    pack_mxfp4_kernel<<<dim3(unsigned(grid)), block, 0, stream>>>(w, rows, K, codes, static_cast<uint8_t*>(scales),
                                                                  nonfinite);
  return cudaGetLastError();
}

cudaError_t launch_pack_mxfp4_rule(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                                   int rule, cudaStream_t stream) {
  if (rule == MOE_MX_EXP_FLOOR) return launch_pack(MOE_FMT_MXFP4_G32, w, E, N, K, packed, nonfinite, stream);
  const long nblocks = long(E) * N * (K / 32);
  if (nblocks == 0) return cudaSuccess;
  const int block = 256;
  const long grid = (nblocks * 32 + block - 1) / block;
  uint8_t* codes = static_cast<uint8_t*>(packed);
  uint8_t* scales = codes + bank_scale_offset(MOE_FMT_MXFP4_G32, E, N, K);
  pack_mxfp4_rule_kernel<<<dim3(unsigned(grid)), block, 0, stream>>>(w, nblocks, codes, scales, nonfinite, rule);
  return cudaGetLastError();
}

cudaError_t launch_dequant(moe_format_t fmt, const void* packed, int E, int N, int K, uint16_t* out,
                           cudaStream_t stream) {
  const long rows = long(E) * N;
  const long nbytes = rows * (K / 2);
  if (nbytes == 0) return cudaSuccess;
  const int block = 256;
  const long grid = (nbytes + block - 1) / block;
  const uint8_t* codes = static_cast<const uint8_t*>(packed);
  const void* scales = static_cast<const uint8_t*>(packed) + bank_scale_offset(fmt, E, N, K);
  const float* gscale = fmt == MOE_FMT_NVFP4_G16 ? reinterpret_cast<const float*>(
                                                       static_cast<const uint8_t*>(packed) + bank_gscale_offset(fmt, E, N, K))
                                                 : nullptr;
  dequant_kernel<<<dim3(unsigned(grid)), block, 0, stream>>>(codes, scales, gscale, int(fmt), rows, N, K, out);
  return cudaGetLastError();
}

}  // namespace moe
