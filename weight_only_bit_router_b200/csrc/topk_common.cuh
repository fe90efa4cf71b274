// Warp-level top-k of one token's router logits with the renormalised
// softmax over the selected experts (ties to the lower expert index).
#pragma once

#include <float.h>

#include "common.cuh"

namespace moe {

// Order-preserving map of a non-NaN fp32 value to uint32 (-0 and +0 equal).
MOE_DEV uint32_t orderable(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 + 0 = +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of orderable().
MOE_DEV float from_orderable(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Top-k of one token's logits by one warp.  Lane l holds experts l, l+32, ...
// (PER = ceil(E/32) of them) and first sorts them by (value descending, expert
// ascending) with a bitonic network in registers.  Each round then takes the
// largest head with two warp reductions (max of the value key, then min of the
// expert index among lanes whose head has that value: ties go to the lower
// expert) and the winning lane drops its head.  Logits are read through L2
// (they may come from other CTAs).
template <int PER>
MOE_DEV void warp_topk_t(const float* __restrict__ row, const float* __restrict__ bias, int E, int k,
                         int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  uint32_t key[PER];
  int slot[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = i * 32 + lane;
    slot[i] = i;
    key[i] = 0u;  // empty: below every real key
    if (e < E) {
      float val = __ldcg(row + e);
      if (bias) val = val + bias[e];  // fp32 add
      key[i] = orderable(val);
    }
  }
  // bitonic sort into ascending "worse" order: position 0 ends up the best
#pragma unroll
  for (int size = 2; size <= PER; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int l = i ^ stride;
        if (l > i) {
          // better(a, b): larger key, or equal key and lower slot
          const bool l_better = key[l] > key[i] || (key[l] == key[i] && slot[l] < slot[i]);
          const bool swap = ((i & size) == 0) ? l_better : !l_better;
          if (swap) {
            const uint32_t tk = key[i]; key[i] = key[l]; key[l] = tk;
            const int ts = slot[i]; slot[i] = slot[l]; slot[l] = ts;
          }
        }
      }
    }
  }
  float my_val = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, key[0]);
    const uint32_t cand = (key[0] != 0u && key[0] == kmax) ? uint32_t(slot[0] * 32 + lane) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if (int(win & 31) == lane) {
#pragma unroll
      for (int i = 0; i + 1 < PER; ++i) {
        key[i] = key[i + 1];
        slot[i] = slot[i + 1];
      }
      key[PER - 1] = 0u;
    }
    if (lane == j) {
      my_val = from_orderable(kmax);
      my_id = int(win);
    }
  }
  const float vmax = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - vmax) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[lane] = my_id;
    wout[lane] = ex / sum;
  }
}

MOE_DEV void warp_topk(const float* __restrict__ row, const float* __restrict__ bias, int E, int k,
                       int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int per = (E + 31) / 32;
  if (per <= 1) warp_topk_t<1>(row, bias, E, k, ids, wout);
  else if (per <= 2) warp_topk_t<2>(row, bias, E, k, ids, wout);
  else if (per <= 4) warp_topk_t<4>(row, bias, E, k, ids, wout);
  else if (per <= 8) warp_topk_t<8>(row, bias, E, k, ids, wout);
  else if (per <= 16) warp_topk_t<16>(row, bias, E, k, ids, wout);
  else warp_topk_t<32>(row, bias, E, k, ids, wout);
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// Top-k for k <= 8 of E <= 256 experts by one warp, without sequential
// selection rounds.  A candidate is one 64-bit code: the order-preserving
// key of its (biased) logit in the high word and the complement of its expert
// index in the low word, so a larger code is the better candidate (larger
// value, or equal value and lower index).  Each lane sorts its 8 codes
// (experts lane, lane+32, ...) with a bitonic network; five butterfly steps
// then merge every lane's list with its partner's (shfl_xor 1, 2, 4, 8, 16),
// keeping the larger 8 of the 16 as a sorted list, so that every lane ends
// with the warp's top 8.  Lane j < k then holds the j-th largest candidate.
// ---------------------------------------------------------------------------
MOE_DEV uint64_t max_u64(uint64_t a, uint64_t b) { return a > b ? a : b; }
MOE_DEV uint64_t min_u64(uint64_t a, uint64_t b) { return a > b ? b : a; }

// Sort 8 codes in descending order (bitonic network).
MOE_DEV void sort8_desc(uint64_t (&c)[8]) {
#pragma unroll
  for (int size = 2; size <= 8; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int l = i ^ stride;
        if (l > i) {
          const bool desc = (i & size) == 0;
          const uint64_t a = c[i], b = c[l];
          c[i] = desc ? max_u64(a, b) : min_u64(a, b);
          c[l] = desc ? min_u64(a, b) : max_u64(a, b);
        }
      }
    }
  }
}

// c: a descending list of 8; returns the descending top 8 of c and the
// partner lane's list (shfl_xor with `o`).
MOE_DEV void merge8_with_lane(uint64_t (&c)[8], int o) {
  uint64_t d[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // partner's element 7 - i (its list ascending from our point of view)
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, uint32_t(c[7 - i]), o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, uint32_t(c[7 - i] >> 32), o);
    d[i] = max_u64(c[i], (uint64_t(hi) << 32) | lo);  // the top 8 of 16, as a bitonic sequence
  }
#pragma unroll
  for (int stride = 4; stride > 0; stride >>= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int l = i ^ stride;
      if (l > i) {
        const uint64_t a = d[i], b = d[l];
        d[i] = max_u64(a, b);
        d[l] = min_u64(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = d[i];
}

// Top-k (k <= 8) of one token's logits row[0, E) (+ bias), E <= 256: writes
// ids[0, k) in descending order and the renormalised softmax weights over the
// selected (biased) logits.  `row` may point to shared or global memory.
MOE_DEV void warp_topk8(const float* row, const float* __restrict__ bias, int E, int k, int32_t* ids,
                        float* wout) {
  const int lane = threadIdx.x & 31;
  uint64_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = i * 32 + lane;
    c[i] = 0;  // empty: below every real candidate
    if (e < E) {
      float val = row[e];
      if (bias) val = val + bias[e];  // fp32 add
      c[i] = (uint64_t(orderable(val)) << 32) | uint32_t(0xFFFFFFFFu - uint32_t(e));
    }
  }
  sort8_desc(c);
  // one compact loop body: this code runs once per launch, from a cold
  // instruction cache, so its size matters more than its loop overhead
#pragma unroll 1
  for (int o = 1; o < 32; o <<= 1) merge8_with_lane(c, o);
  uint64_t mine = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane == i) mine = c[i];
  const float my_val = from_orderable(uint32_t(mine >> 32));
  const int my_id = int(0xFFFFFFFFu - uint32_t(mine));
  const float vmax = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - vmax) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane < k) {
    ids[lane] = my_id;
    wout[lane] = ex / sum;
  }
}

}  // namespace moe
