// Decode path (small token counts, T <= 32): weight-streaming expert GEMVs.
//
// The time goes into streaming the touched experts' packed weights from HBM
// ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", Measured: at concurrency 32
// the bottleneck is weight bandwidth).  Both kernels are persistent: one
// producer warp per CTA starts 1-D bulk copies of 16-row weight tiles (one
// copy per row, at a padded shared-memory stride, plus their scales) into a
// ring of stages and keeps the next tiles' bytes in flight (and the tile after
// the ring into L2); consumer warps dequantise in registers
// (decode_common.cuh) and feed mma.sync m16n8k16 with up to 32 tokens.  The
// routing state (touched experts, per-expert row offsets, the rows' tokens) is
// read into shared memory once per CTA, and small token / activation sets are
// staged there once in MMA fragment order.
//
// gate_up: CTA c takes a contiguous run of the (touched expert, 8-feature)
// units; four warps split each unit's k-blocks and sum in shared memory.
// down: CTA c owns 16 output features of every token and runs over all
// touched experts, so the routing-weighted combine of a token's k expert
// outputs happens in the CTA (in slot order, deterministic) and the output is
// written once.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "decode_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kGroupWarps = 4;  // gate_up: consumer warps per work unit

// Build-time tuning knobs (the defaults are the measured best): gate_up
// consumer groups per CTA and its largest stage ring; down consumer warps per
// CTA and its largest stage ring.
#ifndef MOE_DEC_GROUPS
#define MOE_DEC_GROUPS 2
#endif
#ifndef MOE_DEC_STAGES
#define MOE_DEC_STAGES 8
#endif
#ifndef MOE_DEC_DN_WARPS
#define MOE_DEC_DN_WARPS 8
#endif
#ifndef MOE_DEC_DN_STAGES
#define MOE_DEC_DN_STAGES 32
#endif
constexpr int kGuGroups = MOE_DEC_GROUPS;
constexpr int kGuMaxStages = MOE_DEC_STAGES;
constexpr int kGuThreads = (kGuGroups * kGroupWarps + 1) * 32;
constexpr int kDnWarps = MOE_DEC_DN_WARPS;
constexpr int kDnMaxStages = MOE_DEC_DN_STAGES;
constexpr int kDnThreads = (kDnWarps + 1) * 32;
constexpr int kDnRows = 16;  // output features per down tile

// The routing state every CTA keeps in shared memory: the touched-expert list
// [n, e_0, e_1, ...] and the per-expert row offsets (E + 1 entries each).
MOE_DEV void load_routing(int* s_touched, int* s_off, const int32_t* touched, const int32_t* offsets, int E) {
  for (int i = threadIdx.x; i <= E; i += blockDim.x) {
    s_touched[i] = __ldcg(touched + i);
    s_off[i] = __ldcg(offsets + i);
  }
}

// The touched experts of the bank's range [e_lo, e_hi) are a contiguous slice
// [*t_lo, *t_hi) of the ascending touched list: counted by the whole CTA.
// Called by every thread after the routing state is in shared memory; ends
// with a block barrier.
MOE_DEV void local_slice(const int* s_touched, int e_lo, int e_hi, int E, int* s_cnt, int* t_lo, int* t_hi) {
  const int n = s_touched[0];
  if (e_lo == 0 && e_hi == E) {
    *t_lo = 0;
    *t_hi = n;
    return;
  }
  if (threadIdx.x < 2) s_cnt[threadIdx.x] = 0;
  __syncthreads();
  int below = 0, inside = 0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = s_touched[1 + i];
    below += e < e_lo;
    inside += e >= e_lo && e < e_hi;
  }
  if (below) atomicAdd(&s_cnt[0], below);
  if (inside) atomicAdd(&s_cnt[1], inside);
  __syncthreads();
  *t_lo = s_cnt[0];
  *t_hi = s_cnt[0] + s_cnt[1];
}

template <typename T>
MOE_DEV T* align8(void* p) {
  return reinterpret_cast<T*>((reinterpret_cast<uintptr_t>(p) + 7) & ~uintptr_t(7));
}

// Activation fragments of the gate_up kernel: token rows of x (staged in
// fragment order, or read through L1) for the token tiles of one unit.
template <int NT, bool X_SMEM>
struct XFrags {
  const uint16_t* x;      // global x [T, K]
  const uint8_t* x_s;     // staged rows (X_SMEM)
  int pstride, K, q;
  int tok[NT];            // token of column 8j + g
  MOE_DEV void load(int j, int b, bool in, uint32_t (&bf)[8][2]) const {
    if (X_SMEM) act_frags_staged(x_s + tok[j] * pstride + 256 * b, q, in, bf);
    else act_frags_global<1>(x + size_t(tok[j]) * K + 128 * b + 32 * q, in, bf);
  }
};

// Activation fragments of the down kernel: the expert's bf16 SwiGLU rows p
// (staged in fragment order, or read through L2: another kernel wrote them).
template <bool ACT_SMEM>
struct ActFrags {
  const uint16_t* act;    // global act [T*k, K]
  const uint8_t* act_s;   // staged rows (ACT_SMEM)
  int pstride, K, q, g, p0, n_e;
  MOE_DEV void load(int j, int b, bool in, uint32_t (&bf)[8][2]) const {
    const int c = 8 * j + g;
    const int p = p0 + (c < n_e ? c : 0);
    if (ACT_SMEM) act_frags_staged(act_s + size_t(p) * pstride + 256 * b, q, in, bf);
    else act_frags_global<2>(act + size_t(p) * K + 128 * b + 32 * q, in, bf);
  }
};

// Let the last bulk copies of this CTA's producer land before its shared
// memory is released (bounded: they complete unless the GPU is failing).
MOE_DEV void drain_stages(uint64_t* full, int issued, int S) {
  for (int i = max(0, issued - S); i < issued; ++i) mbar_wait_drain(&full[i % S], (i / S) & 1, kWaitLimitNs);
}

// Start the copies of one 16-row weight tile into `stage` (codes at the padded
// row stride, then scales): lanes 0-15 one code row each (source rows
// row_a + l for l < 8, row_b + l - 8 after), lanes 16 / 17 the scales of the
// two 8-row runs (16 contiguous rows when row_b = row_a + 8: lane 16 alone).
// Called by the whole producer warp after lane 0 announced the bytes.
template <int FMT>
MOE_DEV void stage_tile(const Bank& bk, long row_a, long row_b, uint8_t* stage, const StageLayout& L, uint64_t* bar,
                        uint64_t policy, int lane) {
  const int K = bk.K;
  const int srow = scale_row_bytes(FMT, K);
  const uint8_t* scales = static_cast<const uint8_t*>(bk.scales);
  if (lane < 16) {
    const long r = lane < 8 ? row_a + lane : row_b + lane - 8;
    bulk_g2s_hint(stage + lane * L.crow, bk.codes + r * (K / 2), uint32_t(K / 2), bar, policy);
  } else if (lane == 16) {
    const int n = row_b == row_a + 8 ? 16 : 8;
    bulk_g2s_hint(stage + L.cbytes, scales + row_a * srow, uint32_t(n * srow), bar, policy);
  } else if (lane == 17 && row_b != row_a + 8) {
    bulk_g2s_hint(stage + L.cbytes + 8 * srow, scales + row_b * srow, uint32_t(8 * srow), bar, policy);
  }
}

// ---------------------------------------------------------------------------
// gate_up + SwiGLU.  Work unit u = (touched slot u / (I/8), features
// f0 = 8 (u % (I/8)) .. f0 + 7): its 16 weight rows are the 8 gate rows f0..
// and the 8 matching up rows I + f0.., staged as one 16-row tile (gate rows
// 0-7, up rows 8-15), so the MMA's C fragment holds gate (c0, c1) and up
// (c2, c3) of the same feature and token: SwiGLU needs no shuffle.  CTA c
// takes units [c n / grid, (c + 1) n / grid); its i-th goes to stage i % S and
// consumer group i % G.  The group's four warps split K (128-k blocks w,
// w + 4, ...), and one of them (rotating) sums the four partial tiles in warp
// order and writes a = bf16(silu(gate) * up) to act[p][f] for the expert's
// sorted rows p.  With X_SMEM (small T) the consumers first stage the T token
// rows in fragment order.
// ---------------------------------------------------------------------------
template <int FMT, int NT, bool X_SMEM>
__global__ void __launch_bounds__(kGuThreads, 1) decode_gate_up_kernel(
    const uint16_t* __restrict__ x, int T, Bank gu, int I, int E, int top_k, int e_lo, int e_hi,
    const int32_t* __restrict__ touched, const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows,
    uint16_t* __restrict__ act, uint32_t* status, int S) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int G = kGuGroups;
  constexpr int CH = NT == 1 ? 4 : 2;  // accumulator chains per token tile
  const int K = gu.K, R = T * top_k;
  const StageLayout L = stage_layout(FMT, K, 16);
  const int srow = scale_row_bytes(FMT, K);
  const int pstride = staged_act_stride(K);
  uint8_t* ring = smem;                                                      // [S][stage]
  uint8_t* x_s = ring + size_t(S) * L.stage_bytes;                           // [T][pstride] (X_SMEM)
  float* red = reinterpret_cast<float*>(x_s + (X_SMEM ? size_t(T) * pstride : 0));  // [G][2][4][NT][4][32]
  int* s_touched = reinterpret_cast<int*>(red + G * 2 * kGroupWarps * NT * 128);
  int* s_off = s_touched + (E + 1);
  int* s_tok = s_off + (E + 1);                                              // [R] token of sorted row p
  uint64_t* full = align8<uint64_t>(s_tok + R);
  uint64_t* empty = full + S;
  __shared__ volatile int s_abort;  // raised by the first wait that gives up
  __shared__ int s_cnt[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kGroupWarps);
    }
    fence_mbar_init();
  }
  pdl_wait();
  pdl_trigger();
  load_routing(s_touched, s_off, touched, offsets, E);
  for (int p = threadIdx.x; p < R; p += blockDim.x) s_tok[p] = __ldcg(sorted_rows + p) / top_k;
  __syncthreads();
  int t_lo, t_hi;
  local_slice(s_touched, e_lo, e_hi, E, s_cnt, &t_lo, &t_hi);
  const int* s_local = s_touched + 1 + t_lo;  // the bank's touched experts (global ids)
  const int ftiles = I / 8;
  const int n_units = (t_hi - t_lo) * ftiles;
  const int u_begin = int(long(n_units) * blockIdx.x / gridDim.x);
  const int cnt = int(long(n_units) * (blockIdx.x + 1) / gridDim.x) - u_begin;
  if (cnt <= 0) return;

  if (warp == G * kGroupWarps) {
    // ---------------------------------------------------------------- producer
    const uint64_t policy = l2_policy_evict_first();
    const uint32_t tx = staged_bytes<FMT>(gu, 16);
    int slot = u_begin / ftiles, ft = u_begin - slot * ftiles;          // unit i
    int pslot = (u_begin + S) / ftiles, pft = (u_begin + S) - pslot * ftiles;  // unit i + S
    int i = 0, st = 0, ph = 0;  // unit i's stage and that stage's use count parity
    for (; i < cnt; ++i) {
      if (i >= S && !__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1, &s_abort, status))) break;
      const long row_g = long(s_local[slot] - e_lo) * gu.N + ft * 8;
      fence_proxy_async_smem();  // earlier generic-proxy reads of this stage before the refill
      if (lane == 0) mbar_arrive_expect_tx(&full[st], tx);
      __syncwarp();
      stage_tile<FMT>(gu, row_g, row_g + I, ring + size_t(st) * L.stage_bytes, L, &full[st], policy, lane);
      if (lane >= 18 && lane < 22 && i + S < cnt) {
        // the unit that will refill this stage, into L2 ahead of time
        const long rn = long(s_local[pslot] - e_lo) * gu.N + pft * 8 + ((lane & 1) ? I : 0);
        if (lane < 20) prefetch_codes<FMT>(gu, rn, 8);
        else prefetch_scales<FMT>(gu, rn, 8);
      }
      if (++st == S) st = 0, ph ^= 1;
      if (++ft == ftiles) ft = 0, ++slot;
      if (++pft == ftiles) pft = 0, ++pslot;
    }
    if (lane == 0) drain_stages(full, i, S);
    return;
  }

  // -------------------------------------------------------------------- consumers
  constexpr int kConsumers = G * kGroupWarps * 32;
  const int grp = warp / kGroupWarps, wj = warp % kGroupWarps;
  const int g = lane >> 2, q = lane & 3;
  if (X_SMEM) {
    stage_act_rows<1>(x_s, x, T, K, threadIdx.x, kConsumers);
    named_barrier_sync(1, kConsumers);
  }
  const int nfull = K / 128;  // blocks where every lane slice lies inside K
  const int my_full = wj < nfull ? (nfull - wj + kGroupWarps - 1) / kGroupWarps : 0;
  const int tail_b = ((K % 128) != 0 && nfull % kGroupWarps == wj) ? nfull : -1;
  int slot = (u_begin + grp) / ftiles, ft = (u_begin + grp) - slot * ftiles;
  int st = grp, ph = 0;
  for (int i = grp, n = 0; i < cnt; i += G, ++n) {
    // warp-uniform: the MMAs below run only if every lane saw the data land
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], ph, &s_abort, status));
    const int e = s_local[slot];
    const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
    const int f0 = ft * 8;
    const uint8_t* s_c = ring + size_t(st) * L.stage_bytes;
    const uint8_t* c_gate = s_c + g * L.crow + 16 * q;   // rows g (gate) and g + 8 (up), lane slice
    const uint8_t* c_up = c_gate + 8 * L.crow;
    const uint8_t* sc_gate = s_c + L.cbytes + g * srow;
    const uint8_t* sc_up = sc_gate + 8 * srow;
    const float gsc = FMT == MOE_FMT_NVFP4_G16 ? gu.gscale[e - e_lo] : 0.f;
    const int ntiles = min(NT, (n_e + 7) / 8);
    XFrags<NT, X_SMEM> xf;
    xf.x = x;
    xf.x_s = x_s;
    xf.pstride = pstride;
    xf.K = K;
    xf.q = q;
    // token of column 8j + g (a valid token's row for the padding columns)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int c = 8 * j + g;
      xf.tok[j] = s_tok[p0 + (c < n_e ? c : 0)];
    }
    float acc2[NT][CH][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int h = 0; h < CH; ++h)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc2[j][h][c] = 0.f;
    if (ok) warp_tile<FMT, NT, CH>(acc2, c_gate, c_up, sc_gate, sc_up, wj, kGroupWarps, my_full, tail_b, K, q, gsc,
                                   ntiles, xf);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
    // the group's partial tiles, double-buffered by unit parity
    float* red_u = red + size_t((grp * 2 + (n & 1)) * kGroupWarps) * NT * 128;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v = acc2[j][0][c];
#pragma unroll
        for (int h = 1; h < CH; ++h) v += acc2[j][h][c];
        red_u[((wj * NT + j) * 4 + c) * 32 + lane] = v;
      }
    named_barrier_sync(2 + grp, kGroupWarps * 32);
    if (ok && wj == n % kGroupWarps) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (j >= ntiles) break;
        float sum[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sum[c] = 0.f;
#pragma unroll
          for (int w = 0; w < kGroupWarps; ++w) sum[c] += red_u[((w * NT + j) * 4 + c) * 32 + lane];
        }
        // c0, c1: gate of feature f0+g at columns 2q, 2q+1; c2, c3: up of the same
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int col = 8 * j + 2 * q + hh;
          if (col < n_e) act[size_t(p0 + col) * I + f0 + g] = f32_to_bf16_rn(silu_mul(sum[hh], sum[2 + hh]));
        }
      }
    }
    st += G;
    if (st >= S) st -= S, ph ^= 1;
    ft += G;
    while (ft >= ftiles) ft -= ftiles, ++slot;
  }
}

// ---------------------------------------------------------------------------
// down projection and combine.  CTA c owns the 16 output features of tiles
// c, c + grid, ... (H / 16 tiles).  For a tile, work unit s = the tile's 16
// rows of the down matrix of touched expert s (all of K = I), taken by
// consumer warp s % W; its C fragment times the routing weight of each
// column's (token, slot) goes to ybuf[t k + j][f] in shared memory.  When the
// tile's units are done, each token's output is the sum of its k slots in
// slot order (plus the shared expert's gated output), rounded once to bf16,
// or the fp32 sum (an expert-parallel shard's partial: slots of other shards'
// experts stay zero).  The weights do not depend on the gate_up kernel that
// runs just before: the producer reads the routing state (written two
// launches back, and the kernel in between triggers its dependents only after
// its own wait) and starts the weight copies before the programmatic-launch
// wait; only the consumers wait.  With ACT_SMEM (small T) the consumers first
// stage the T*k activation rows in fragment order.
// ---------------------------------------------------------------------------
template <int FMT, int NT, bool ACT_SMEM>
__global__ void __launch_bounds__(kDnThreads, 1) decode_down_kernel(
    Bank dn, int T, int E, int top_k, int e_lo, int e_hi, const int32_t* __restrict__ touched,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows, const uint16_t* __restrict__ act,
    const float* __restrict__ topk_w, const float* __restrict__ sh_gate, const float* __restrict__ sh_y,
    uint16_t* __restrict__ out, float* __restrict__ partial_out, uint32_t* status, int S) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = kDnWarps;
  constexpr int CH = NT == 1 ? 4 : 2;
  const int H = dn.N, K = dn.K;  // K = I
  const int R = T * top_k;
  const StageLayout L = stage_layout(FMT, K, kDnRows);
  const int srow = scale_row_bytes(FMT, K);
  const int pstride = staged_act_stride(K);
  uint8_t* ring = smem;                                           // [S][stage]
  uint8_t* act_s = ring + size_t(S) * L.stage_bytes;              // [R][pstride] (ACT_SMEM)
  float* ybuf = reinterpret_cast<float*>(act_s + (ACT_SMEM ? size_t(R) * pstride : 0));  // [R][16]
  int* s_touched = reinterpret_cast<int*>(ybuf + R * kDnRows);
  int* s_off = s_touched + (E + 1);
  int* s_slot = s_off + (E + 1);                                  // [R] slot t k + j of sorted row p
  float* s_w = reinterpret_cast<float*>(s_slot + R);              // [R] its routing weight
  uint64_t* full = align8<uint64_t>(s_w + R);
  uint64_t* empty = full + S;
  __shared__ volatile int s_abort;
  __shared__ int s_cnt[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    fence_mbar_init();
  }
  // routing state: written two launches back (see above), read through L2
  load_routing(s_touched, s_off, touched, offsets, E);
  for (int p = threadIdx.x; p < R; p += blockDim.x) {
    const int r = __ldcg(sorted_rows + p);
    s_slot[p] = r;
    s_w[p] = __ldcg(topk_w + r);
  }
  for (int i = threadIdx.x; i < R * kDnRows; i += blockDim.x) ybuf[i] = 0.f;
  __syncthreads();
  int t_lo, t_hi;
  local_slice(s_touched, e_lo, e_hi, E, s_cnt, &t_lo, &t_hi);
  const int* s_local = s_touched + 1 + t_lo;  // the bank's touched experts (global ids)
  const int n_t = t_hi - t_lo;
  const int ntile = H / kDnRows;

  if (warp == W) {
    // ---------------------------------------------------------------- producer
    if (n_t > 0) {
      const uint64_t policy = l2_policy_evict_first();
      const uint32_t tx = staged_bytes<FMT>(dn, kDnRows);
      int ptile = blockIdx.x, ps = 0;  // unit i + S
      for (int a = 0; a < S; ++a)
        if (++ps == n_t) ps = 0, ptile += gridDim.x;
      int i = 0, st = 0, ph = 0;
      bool run = true;
      for (int tile = blockIdx.x; run && tile < ntile; tile += gridDim.x) {
        for (int s = 0; s < n_t; ++s, ++i) {
          if (i >= S && !__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1, &s_abort, status))) {
            run = false;
            break;
          }
          const long row0 = long(s_local[s] - e_lo) * H + tile * kDnRows;
          fence_proxy_async_smem();
          if (lane == 0) mbar_arrive_expect_tx(&full[st], tx);
          __syncwarp();
          stage_tile<FMT>(dn, row0, row0 + 8, ring + size_t(st) * L.stage_bytes, L, &full[st], policy, lane);
          if (lane >= 18 && lane < 20 && ptile < ntile) {
            // the unit that will refill this stage, into L2 ahead of time
            const long rn = long(s_local[ps] - e_lo) * H + ptile * kDnRows;
            if (lane == 18) prefetch_codes<FMT>(dn, rn, kDnRows);
            else prefetch_scales<FMT>(dn, rn, kDnRows);
          }
          if (++st == S) st = 0, ph ^= 1;
          if (++ps == n_t) ps = 0, ptile += gridDim.x;
        }
      }
      if (lane == 0) drain_stages(full, i, S);
    }
    pdl_wait();
    pdl_trigger();
    return;
  }

  // -------------------------------------------------------------------- consumers
  constexpr int kConsumers = W * 32;
  pdl_wait();  // the activations (and the previous readers of the output) of the kernels before
  pdl_trigger();
  const int g = lane >> 2, q = lane & 3;
  if (ACT_SMEM) stage_act_rows<2>(act_s, act, R, K, threadIdx.x, kConsumers);
  named_barrier_sync(1, kConsumers);
  const int nfull = K / 128;
  const int tail_b = (K % 128) != 0 ? nfull : -1;
  int ti = 0;
  for (int tile = blockIdx.x; tile < ntile; tile += gridDim.x, ++ti) {
    for (int s = warp; s < n_t; s += W) {
      const int idx = ti * n_t + s;  // the CTA's unit index
      const int st = idx % S;
      // warp-uniform: the MMAs below run only if every lane saw the data land
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (idx / S) & 1, &s_abort, status));
      const int e = s_local[s];
      const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
      const uint8_t* s_c = ring + size_t(st) * L.stage_bytes;
      const uint8_t* c_lo = s_c + g * L.crow + 16 * q;
      const uint8_t* c_hi = c_lo + 8 * L.crow;
      const uint8_t* sc_lo = s_c + L.cbytes + g * srow;
      const uint8_t* sc_hi = sc_lo + 8 * srow;
      const float gsc = FMT == MOE_FMT_NVFP4_G16 ? dn.gscale[e - e_lo] : 0.f;
      const int ntiles = min(NT, (n_e + 7) / 8);
      ActFrags<ACT_SMEM> af;
      af.act = act;
      af.act_s = act_s;
      af.pstride = pstride;
      af.K = K;
      af.q = q;
      af.g = g;
      af.p0 = p0;
      af.n_e = n_e;
      float acc2[NT][CH][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int h = 0; h < CH; ++h)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc2[j][h][c] = 0.f;
      if (ok) warp_tile<FMT, NT, CH>(acc2, c_lo, c_hi, sc_lo, sc_hi, 0, 1, nfull, tail_b, K, q, gsc, ntiles, af);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (!ok) continue;
      // c0, c1: feature g at columns 2q, 2q+1; c2, c3: feature g + 8
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (j >= ntiles) break;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = 8 * j + 2 * q + (c & 1);
          if (col < n_e) {
            float v = acc2[j][0][c];
#pragma unroll
            for (int h = 1; h < CH; ++h) v += acc2[j][h][c];
            ybuf[s_slot[p0 + col] * kDnRows + g + 8 * (c >> 1)] = s_w[p0 + col] * v;
          }
        }
      }
    }
    named_barrier_sync(1, kConsumers);
    // each token's k slots summed in slot order, two features per thread
    for (int o = threadIdx.x; o < T * (kDnRows / 2); o += kConsumers) {
      const int t = o / (kDnRows / 2), f = 2 * (o % (kDnRows / 2));
      float v0 = 0.f, v1 = 0.f;
      for (int j = 0; j < top_k; ++j) {
        float* yb = ybuf + (t * top_k + j) * kDnRows + f;
        v0 += yb[0];
        v1 += yb[1];
        yb[0] = 0.f;
        yb[1] = 0.f;
      }
      const size_t oi = size_t(t) * H + tile * kDnRows + f;
      if (partial_out) {
        *reinterpret_cast<float2*>(partial_out + oi) = make_float2(v0, v1);
      } else {
        if (sh_y) {
          const float gg = __ldcg(sh_gate + t);
          v0 += gg * __ldcg(sh_y + oi);
          v1 += gg * __ldcg(sh_y + oi + 1);
        }
        *reinterpret_cast<uint32_t*>(out + oi) = pack_bf16x2(v0, v1);
      }
    }
    named_barrier_sync(1, kConsumers);
  }
}

int max_touched(int T, int k, int E) { return (long(T) * k < E) ? T * k : E; }

constexpr size_t kMaxSmemPerCta = 226 * 1024;  // dynamic shared memory, leaving room for static
// Staged token rows (gate_up) and activation rows (down) up to these sizes.
constexpr size_t kMaxStagedX = 72 * 1024;
constexpr size_t kMaxStagedAct = 72 * 1024;

int nt_of(int T) { return T <= 8 ? 1 : T <= 16 ? 2 : 4; }

// gate_up: stages + staged token rows + the partial-tile buffers + routing
// state + barriers
size_t gate_up_smem(int fmt, int K, int NT, int E, int R, int x_rows, int S) {
  const StageLayout L = stage_layout(fmt, K, 16);
  return size_t(S) * L.stage_bytes + size_t(x_rows) * staged_act_stride(K) +
         size_t(kGuGroups) * 2 * kGroupWarps * NT * 128 * 4 + size_t(2 * (E + 1) + R) * 4 + 8 + 2 * size_t(S) * 8;
}

// down: stages + staged activation rows + the slot outputs + routing state +
// barriers
size_t down_smem(int fmt, int K, int E, int R, int act_rows, int S) {
  const StageLayout L = stage_layout(fmt, K, kDnRows);
  return size_t(S) * L.stage_bytes + size_t(act_rows) * staged_act_stride(K) + size_t(R) * kDnRows * 4 +
         size_t(2 * (E + 1) + 2 * R) * 4 + 8 + 2 * size_t(S) * 8;
}

struct GuPlan {
  bool x_smem;
  int S;
  size_t smem;
};
struct DnPlan {
  bool act_smem;
  int S;
  size_t smem;
};

// The largest stage ring (a multiple of the consumer groups, at least two
// stages per group) that fits beside the rest; S = 0 when none does.
GuPlan gate_up_plan(const moe_shape_t& s, int T) {
  const int R = T * s.top_k, NT = nt_of(T);
  GuPlan p;
  p.x_smem = size_t(T) * staged_act_stride(s.hidden) <= kMaxStagedX;
  p.S = 0;
  p.smem = 0;
  for (int S = kGuMaxStages / kGuGroups * kGuGroups; S >= 2 * kGuGroups; S -= kGuGroups) {
    const size_t b = gate_up_smem(s.fmt, s.hidden, NT, s.num_experts, R, p.x_smem ? T : 0, S);
    if (b <= kMaxSmemPerCta) {
      p.S = S;
      p.smem = b;
      break;
    }
  }
  return p;
}

DnPlan down_plan(const moe_shape_t& s, int T) {
  const int R = T * s.top_k;
  DnPlan p;
  p.act_smem = size_t(R) * staged_act_stride(s.inter) <= kMaxStagedAct;
  p.S = 0;
  p.smem = 0;
  for (int S = kDnMaxStages / kDnWarps * kDnWarps; S >= kDnWarps; S -= kDnWarps) {
    const size_t b = down_smem(s.fmt, s.inter, s.num_experts, R, p.act_smem ? R : 0, S);
    if (b <= kMaxSmemPerCta) {
      p.S = S;
      p.smem = b;
      break;
    }
  }
  return p;
}

int sm_count_cached() {
  static std::atomic<int> cached{0};
  int n = cached.load(std::memory_order_relaxed);
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached.store(n, std::memory_order_relaxed);
  }
  return n;
}

// Persistent grid: as many CTAs as fit on the GPU at once (at most `units`).
// The occupancy of each (kernel, shared-memory size) is computed once and kept
// in a small table (instantiations of one template share a function type, so
// the kernel's address is part of the key).
template <typename Kern>
int persistent_grid(Kern k, size_t smem, int units, int threads) {
  struct Entry {
    const void* fn;
    size_t smem;
    int per_sm;
  };
  static Entry cache[32] = {};
  static std::mutex mu;  // host threads may launch concurrently
  const int sms = sm_count_cached();
  std::lock_guard<std::mutex> lock(mu);
  const void* fn = reinterpret_cast<const void*>(k);
  int per_sm = 0;
  for (const Entry& e : cache)
    if (e.fn == fn && e.smem == smem) per_sm = e.per_sm;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, smem) != cudaSuccess || per_sm < 1)
      per_sm = 1;
    for (Entry& e : cache)
      if (e.fn == nullptr) {
        e = Entry{fn, smem, per_sm};
        break;
      }
  }
  return std::max(1, std::min(units, per_sm * sms));
}

template <typename Kern>
cudaError_t allow_smem(Kern k, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
}

template <int FMT, int NT>
cudaError_t gate_up_nt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const ExpertRange& er,
                       const Workspace& ws, int units, cudaStream_t stream) {
  const GuPlan p = gate_up_plan(s, T);
  if (p.S == 0) return cudaErrorInvalidConfiguration;
  auto k = p.x_smem ? decode_gate_up_kernel<FMT, NT, true> : decode_gate_up_kernel<FMT, NT, false>;
  cudaError_t err = allow_smem(k, p.smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, p.smem, units, kGuThreads);
  return launch_pdl(k, dim3(grid), dim3(kGuThreads), p.smem, stream, x, T, gu, s.inter, s.num_experts, s.top_k,
                    er.lo, er.hi, (const int32_t*)ws.touched, (const int32_t*)ws.offsets,
                    (const int32_t*)ws.sorted_rows, ws.act, ws.status, p.S);
}

template <int FMT>
cudaError_t gate_up_fmt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const ExpertRange& er,
                        const Workspace& ws, int units, cudaStream_t stream) {
  // token tiles of 8 held in registers: enough for the largest possible expert batch (T)
  if (T <= 8) return gate_up_nt<FMT, 1>(s, T, x, gu, er, ws, units, stream);
  if (T <= 16) return gate_up_nt<FMT, 2>(s, T, x, gu, er, ws, units, stream);
  return gate_up_nt<FMT, 4>(s, T, x, gu, er, ws, units, stream);
}

template <int FMT, int NT>
cudaError_t down_nt(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er, const Workspace& ws,
                    const float* sh_gate, const float* sh_y, uint16_t* out, float* partial_out, cudaStream_t stream) {
  const DnPlan p = down_plan(s, T);
  if (p.S == 0) return cudaErrorInvalidConfiguration;
  auto k = p.act_smem ? decode_down_kernel<FMT, NT, true> : decode_down_kernel<FMT, NT, false>;
  cudaError_t err = allow_smem(k, p.smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, p.smem, s.hidden / kDnRows, kDnThreads);
  return launch_pdl(k, dim3(grid), dim3(kDnThreads), p.smem, stream, dn, T, s.num_experts, s.top_k, er.lo, er.hi,
                    (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const int32_t*)ws.sorted_rows,
                    (const uint16_t*)ws.act, (const float*)ws.topk_w, sh_gate, sh_y, out, partial_out, ws.status,
                    p.S);
}

template <int FMT>
cudaError_t down_fmt(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er, const Workspace& ws,
                     const float* sh_gate, const float* sh_y, uint16_t* out, float* partial_out,
                     cudaStream_t stream) {
  if (T <= 8) return down_nt<FMT, 1>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
  if (T <= 16) return down_nt<FMT, 2>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
  return down_nt<FMT, 4>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
}

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
  if (T > kDecodeMaxT) return false;
  return gate_up_plan(s, T).S > 0 && down_plan(s, T).S > 0;
}

cudaError_t launch_decode_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu,
                                  const ExpertRange& er, const Workspace& ws, cudaStream_t stream) {
  const int units = std::min(max_touched(T, s.top_k, s.num_experts), er.hi - er.lo) * (s.inter / 8);
  if (units <= 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128) return gate_up_fmt<MOE_FMT_INT4_G128>(s, T, x, gu, er, ws, units, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return gate_up_fmt<MOE_FMT_NVFP4_G16>(s, T, x, gu, er, ws, units, stream);
  return gate_up_fmt<MOE_FMT_MXFP4_G32>(s, T, x, gu, er, ws, units, stream);
}

cudaError_t launch_decode_down(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er,
                               const Workspace& ws, const float* sh_gate, const float* sh_y, uint16_t* out,
                               float* partial_out, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128)
    return down_fmt<MOE_FMT_INT4_G128>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16)
    return down_fmt<MOE_FMT_NVFP4_G16>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
  return down_fmt<MOE_FMT_MXFP4_G32>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream);
}

}  // namespace moe
