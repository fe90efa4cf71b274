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
// Top-k for k <= 8 of E <= 256 experts by one warp.  Lane l holds experts
// [8l, 8l + 8) and sorts them by (value descending, expert ascending) with a
// bitonic network.  Each of the k rounds then takes the largest head of the
// 32 lists with one redux.sync over the 32-bit value keys; among lanes whose
// head has that value the lowest lane wins, which is the lowest expert index
// because lanes own ascending blocks of experts (ties go to the lower expert),
// and the winning lane drops its head.
// ---------------------------------------------------------------------------

// Top-k (k <= 8) of one token's logits row[0, E) (+ bias), E <= 256: writes
// ids[0, k) in descending order and the renormalised softmax weights over the
// selected (biased) logits.  `row` may point to shared or global memory.
// Lane l holds experts 8l .. 8l + 7.  Each of the k rounds takes every lane's
// best remaining expert (larger key, ties to the lower expert), then the
// warp's best (max key; among lanes with it, the lowest lane: the lower
// expert), and the winning lane marks it taken.  Short code on purpose: it
// runs once per layer in a single CTA, often with a cold instruction cache.
MOE_DEV void warp_topk8(const float* row, const float* __restrict__ bias, int E, int k, int32_t* ids,
                        float* wout) {
  const unsigned full = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = 8 * lane + i;
    key[i] = 0u;  // empty: below every real key
    if (e < E) {
      float val = row[e];
      if (bias) val = val + bias[e];  // fp32 add
      key[i] = orderable(val);
    }
  }
  uint32_t taken = 0u;  // bit i: expert 8 lane + i already selected
  float my_val = 0.f;
  int my_id = 0;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      const uint32_t v = (taken >> i) & 1u ? 0u : key[i];
      if (v >= best) {  // from the top down: ties end on the lower index
        best = v;
        bi = i;
      }
    }
    const uint32_t kmax = __reduce_max_sync(full, best);
    const int wl = __ffs(__ballot_sync(full, best == kmax)) - 1;
    const int wi = __shfl_sync(full, bi, wl);
    if (lane == wl) taken |= 1u << wi;
    if (lane == j) {
      my_val = from_orderable(kmax);
      my_id = 8 * wl + wi;
    }
  }
  const float vmax = __shfl_sync(full, my_val, 0);
  const float ex = lane < k ? expf(my_val - vmax) : 0.f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(full, sum, o);
  if (lane < k) {
    ids[lane] = my_id;
    wout[lane] = ex / sum;
  }
}

}  // namespace moe
