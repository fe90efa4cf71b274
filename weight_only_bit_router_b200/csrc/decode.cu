// Decode path (small token counts, T <= 32): weight-streaming expert GEMVs.
//
// The time goes into streaming the touched experts' packed weights from HBM
// ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", Measured: at concurrency 32
// the bottleneck is weight bandwidth).  Both kernels are persistent streams of
// 16 KB-class work units: a unit's packed rows are one or two contiguous
// ranges of the canonical [E][N][K/2] layout, so one producer lane starts 1-D
// bulk copies of their codes and scales into a ring of shared-memory stages
// and every byte of several units is in flight at once.  Groups of four
// consumer warps dequantise in registers (decode_common.cuh) and feed
// mma.sync m16n8k16 with up to 32 tokens.  The routing state (touched
// experts, per-expert row offsets, the rows' tokens) is read into shared
// memory once per CTA.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "decode_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kGroupWarps = 4;  // consumer warps per work unit

// Number of consumer groups (units in flight through compute) per CTA,
// shared-memory stages per CTA, and CTAs per SM the register budget is sized
// for (build-time tuning knobs; the defaults are the measured best).
#ifndef MOE_DEC_GROUPS
#define MOE_DEC_GROUPS 2
#endif
#ifndef MOE_DEC_STAGES
#define MOE_DEC_STAGES 4
#endif
#ifndef MOE_DEC_MIN_CTAS
#define MOE_DEC_MIN_CTAS 2
#endif
// registers per thread that keep MOE_DEC_MIN_CTAS CTAs per SM (65536 per SM,
// allocated in multiples of 8 per thread); one CTA per SM above 8 tokens
constexpr int kDecRegs = (65536 / (MOE_DEC_MIN_CTAS * (MOE_DEC_GROUPS * 4 + 1) * 32)) / 8 * 8;
constexpr int kDecRegsWide = (65536 / ((MOE_DEC_GROUPS * 4 + 1) * 32)) / 8 * 8 > 255
                                 ? 248 : (65536 / ((MOE_DEC_GROUPS * 4 + 1) * 32)) / 8 * 8;
constexpr int kGroups = MOE_DEC_GROUPS;
constexpr int kStages = MOE_DEC_STAGES;
constexpr int kThreads = (kGroups * kGroupWarps + 1) * 32;

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

// Activation fragments of the gate_up kernel: token rows of x (staged in
// shared memory, or read through L1) for the token tiles of one unit.
template <int NT, bool X_SMEM>
struct XFrags {
  const uint16_t* x;      // global x [T, K]
  const uint8_t* x_s;     // staged rows (X_SMEM)
  int xstride, K, q;
  int tok[NT];            // token of column 8j + g
  MOE_DEV void load(int j, int b, bool in, uint32_t (&bf)[8][2]) const {
    if (X_SMEM) act_frags<0>(reinterpret_cast<const uint16_t*>(x_s + tok[j] * xstride) + 128 * b + 32 * q, in, bf);
    else act_frags<1>(x + size_t(tok[j]) * K + 128 * b + 32 * q, in, bf);
  }
};

// Activation fragments of the down kernel: the expert's bf16 SwiGLU rows p
// (staged in shared memory, or read through L2: another kernel wrote them).
template <bool ACT_SMEM>
struct ActFrags {
  const uint16_t* act;    // global act [T*k, K]
  const uint8_t* act_s;   // staged rows (ACT_SMEM)
  int astride, K, q, g, p0, n_e;
  MOE_DEV void load(int j, int b, bool in, uint32_t (&bf)[8][2]) const {
    const int c = 8 * j + g;
    const int p = p0 + (c < n_e ? c : 0);
    if (ACT_SMEM) act_frags<0>(reinterpret_cast<const uint16_t*>(act_s + p * astride) + 128 * b + 32 * q, in, bf);
    else act_frags<2>(act + size_t(p) * K + 128 * b + 32 * q, in, bf);
  }
};

// Let the last bulk copies of this CTA's producer land before its shared
// memory is released (bounded: they complete unless the GPU is failing).
MOE_DEV void drain_stages(uint64_t* full, int issued, int S) {
  for (int i = max(0, issued - S); i < issued; ++i) mbar_wait_drain(&full[i % S], (i / S) & 1, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// gate_up + SwiGLU.  Work unit u = (touched slot u / (I/8), features
// f0 = 8 (u % (I/8)) .. f0 + 7): its 16 weight rows are the 8 gate rows f0..
// and the 8 matching up rows I + f0.., staged as one 16-row tile (gate rows
// 0-7, up rows 8-15), so the MMA's C fragment holds gate (c0, c1) and up
// (c2, c3) of the same feature and token: SwiGLU needs no shuffle.  The CTA's
// i-th unit goes to stage i % S and consumer group i % G; the group's four
// warps split K (128-k blocks w, w + 4, ...), and one of them (rotating) sums
// the four partial tiles in warp order and writes a = bf16(silu(gate) * up) to
// act[p][f] for the expert's sorted rows p.
// With X_SMEM (small T) the producer warp first stages the T token rows in
// shared memory (one bulk copy per row, padded row stride).
// ---------------------------------------------------------------------------
template <int FMT, int NT, bool X_SMEM>
__global__ void __maxnreg__(NT >= 2 ? kDecRegsWide : kDecRegs) decode_gate_up_kernel(
    const uint16_t* __restrict__ x, int T, Bank gu, int I, int E, int top_k, int e_lo, int e_hi,
    const int32_t* __restrict__ touched, const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows,
    uint16_t* __restrict__ act, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int G = kGroups, S = kStages;
  const int K = gu.K, R = T * top_k;
  const UnitLayout L = unit_layout(FMT, K, 16);
  const int srow = scale_row_bytes(FMT, K);
  const int xstride = staged_row_stride(K);
  uint8_t* ring = smem;                                                  // [S][stage]
  uint8_t* x_s = ring + S * L.stage_bytes;                               // [T][xstride] (X_SMEM)
  float* red = reinterpret_cast<float*>(x_s + (X_SMEM ? T * xstride : 0));  // [G][2][4][NT][4][32]
  int* s_touched = reinterpret_cast<int*>(red + G * 2 * kGroupWarps * NT * 128);
  int* s_off = s_touched + (E + 1);
  int* s_tok = s_off + (E + 1);                                          // [R] token of sorted row p
  uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(s_tok + R) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + S;
  uint64_t* x_bar = empty + S;
  __shared__ volatile int s_abort;  // raised by the first wait that gives up
  __shared__ int s_cnt[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kGroupWarps);
    }
    mbar_init(x_bar, 1);
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
  if (int(blockIdx.x) >= n_units) return;

  if (warp == G * kGroupWarps) {
    // ---------------------------------------------------------------- producer
    if (X_SMEM) {
      if (lane == 0) mbar_arrive_expect_tx(x_bar, uint32_t(T) * uint32_t(2 * K));
      __syncwarp();
      stage_bf16_rows(x_s, x, T, K, x_bar);
    }
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      int i = 0;
      for (;; ++i) {
        const int u = blockIdx.x + i * gridDim.x;
        if (u >= n_units) break;
        const int st = i % S;
        if (i >= S && !mbar_wait(&empty[st], ((i / S) - 1) & 1, &s_abort, status)) break;
        const int e = s_local[u / ftiles];
        const long row_g = long(e - e_lo) * gu.N + (u % ftiles) * 8;
        uint8_t* stage = ring + st * L.stage_bytes;
        fence_proxy_async_smem();  // earlier generic-proxy reads of this stage before the refill
        mbar_arrive_expect_tx(&full[st], staged_bytes<FMT>(gu, 16));
        stage_rows<FMT>(gu, row_g, 8, stage, stage + L.cbytes, &full[st], policy);
        stage_rows<FMT>(gu, row_g + I, 8, stage + 8 * (K / 2), stage + L.cbytes + 8 * srow, &full[st], policy);
        // the unit that will refill this stage, into L2 ahead of time
        const int un = u + S * gridDim.x;
        if (un < n_units) {
          const long rn = long(s_local[un / ftiles] - e_lo) * gu.N + (un % ftiles) * 8;
          prefetch_rows<FMT>(gu, rn, 8);
          prefetch_rows<FMT>(gu, rn + I, 8);
        }
      }
      drain_stages(full, i, S);
    }
    return;
  }

  // -------------------------------------------------------------------- consumers
  const int grp = warp / kGroupWarps, wj = warp % kGroupWarps;
  const int g = lane >> 2, q = lane & 3;
  const int nblk_full = K / 128;              // blocks where every lane slice lies inside K
  const bool tail = (K % 128) != 0;           // a last block with slices past K
  const bool x_ok = !X_SMEM || mbar_wait(x_bar, 0, &s_abort, status);
  for (int i = grp, n = 0;; i += G, ++n) {
    const int u = blockIdx.x + i * gridDim.x;
    if (u >= n_units) break;
    const int st = i % S;
    // warp-uniform: the MMAs below run only if every lane saw the data land
    const bool ok = __all_sync(0xffffffffu, x_ok && mbar_wait(&full[st], (i / S) & 1, &s_abort, status));
    const int e = s_local[u / ftiles];
    const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
    const int f0 = (u % ftiles) * 8;
    const uint8_t* s_c = ring + st * L.stage_bytes;
    const uint8_t* c_gate = s_c + g * (K / 2) + 16 * q;   // rows g (gate) and g + 8 (up), lane slice
    const uint8_t* c_up = c_gate + 8 * (K / 2);
    const uint8_t* sc_gate = s_c + L.cbytes + g * srow;
    const uint8_t* sc_up = sc_gate + 8 * srow;
    const float gsc = FMT == MOE_FMT_NVFP4_G16 ? gu.gscale[e - e_lo] : 0.f;
    const int ntiles = min(NT, (n_e + 7) / 8);
    XFrags<NT, X_SMEM> xf;
    xf.x = x;
    xf.x_s = x_s;
    xf.xstride = xstride;
    xf.K = K;
    xf.q = q;
    // token of column 8j + g (a valid token's row for the padding columns)
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int c = 8 * j + g;
      xf.tok[j] = s_tok[p0 + (c < n_e ? c : 0)];
    }
    float acc2[NT][2][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc2[j][0][c] = acc2[j][1][c] = 0.f;
    if (ok)
      stream_kblocks<FMT, NT>(acc2, wj, kGroupWarps, nblk_full, (tail && nblk_full % kGroupWarps == wj) ? nblk_full : -1,
                              K, q, c_gate, c_up, sc_gate, sc_up, gsc, ntiles, xf);
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[j][c] = acc2[j][0][c] + acc2[j][1][c];
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
    // the group's partial tiles, double-buffered by unit parity
    float* red_u = red + size_t((grp * 2 + (n & 1)) * kGroupWarps) * NT * 128;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) red_u[((wj * NT + j) * 4 + c) * 32 + lane] = acc[j][c];
    named_barrier_sync(1 + grp, kGroupWarps * 32);
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
  }
}

// ---------------------------------------------------------------------------
// down projection.  Work unit u = (feature tile ft = u / n of 64 output
// features, touched slot u % n): the expert's 64 down rows (all of K = I).
// Consumer warp w of the unit's group takes rows 16 w .. 16 w + 15 over every
// k-block and writes w_tj * (Wd a) for each of the expert's sorted rows p
// (fp32, scaled by the row's routing weight) to ypart[p][f].  The combine
// kernel that follows sums each token's k rows in slot order (deterministic).
// The weights do not depend on the gate_up kernel that runs just before: the
// producer reads the routing state (written two launches back, and the kernel
// in between triggers its dependents only after its own wait) and starts the
// weight copies before the programmatic-launch wait; only the consumers wait.
// With ACT_SMEM (small T) one consumer warp stages the T*k activation rows.
// ---------------------------------------------------------------------------
constexpr int kDnRows = 64;  // output features per unit

template <int FMT, int NT, bool ACT_SMEM>
__global__ void __maxnreg__(NT >= 2 ? kDecRegsWide : kDecRegs) decode_down_kernel(
    Bank dn, int T, int E, int top_k, int e_lo, int e_hi, const int32_t* __restrict__ touched,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows, const uint16_t* __restrict__ act,
    const float* __restrict__ topk_w, float* __restrict__ ypart, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int G = kGroups, S = kStages;
  const int H = dn.N, K = dn.K;  // K = I
  const int R = T * top_k;
  const UnitLayout L = unit_layout(FMT, K, kDnRows);
  const int srow = scale_row_bytes(FMT, K);
  const int astride = staged_row_stride(K);
  uint8_t* ring = smem;                                  // [S][stage]
  uint8_t* act_s = ring + S * L.stage_bytes;             // [R][astride] (ACT_SMEM)
  int* s_touched = reinterpret_cast<int*>(act_s + (ACT_SMEM ? R * astride : 0));
  int* s_off = s_touched + (E + 1);
  float* s_wrow = reinterpret_cast<float*>(s_off + (E + 1));  // [R] routing weight of sorted row p
  uint64_t* full = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(s_wrow + R) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + S;
  uint64_t* act_bar = empty + S;
  __shared__ volatile int s_abort;
  __shared__ int s_cnt[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kGroupWarps);
    }
    mbar_init(act_bar, 1);
    fence_mbar_init();
  }
  // routing state: written two launches back (see above), read through L2
  load_routing(s_touched, s_off, touched, offsets, E);
  for (int p = threadIdx.x; p < R; p += blockDim.x) s_wrow[p] = __ldcg(topk_w + __ldcg(sorted_rows + p));
  __syncthreads();
  int t_lo, t_hi;
  local_slice(s_touched, e_lo, e_hi, E, s_cnt, &t_lo, &t_hi);
  const int* s_local = s_touched + 1 + t_lo;  // the bank's touched experts (global ids)
  const int n_t = t_hi - t_lo;
  const int ftiles = H / kDnRows;
  const int n_units = n_t * ftiles;
  if (int(blockIdx.x) >= n_units) {
    pdl_wait();
    pdl_trigger();
    return;
  }

  if (warp == G * kGroupWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      int i = 0;
      for (;; ++i) {
        const int u = blockIdx.x + i * gridDim.x;
        if (u >= n_units) break;
        const int st = i % S;
        if (i >= S && !mbar_wait(&empty[st], ((i / S) - 1) & 1, &s_abort, status)) break;
        const int e = s_local[u % n_t];
        const long row0 = long(e - e_lo) * H + (u / n_t) * kDnRows;
        uint8_t* stage = ring + st * L.stage_bytes;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[st], staged_bytes<FMT>(dn, kDnRows));
        stage_rows<FMT>(dn, row0, kDnRows, stage, stage + L.cbytes, &full[st], policy);
        // the unit that will refill this stage, into L2 ahead of time
        const int un = u + S * gridDim.x;
        if (un < n_units) prefetch_rows<FMT>(dn, long(s_local[un % n_t] - e_lo) * H + (un / n_t) * kDnRows, kDnRows);
      }
      drain_stages(full, i, S);
    }
    pdl_wait();
    pdl_trigger();
    return;
  }

  // -------------------------------------------------------------------- consumers
  pdl_wait();  // the activations (and the previous readers of ypart) of the kernels before
  pdl_trigger();
  const int grp = warp / kGroupWarps, wj = warp % kGroupWarps;
  const int g = lane >> 2, q = lane & 3;
  const int nblk_full = K / 128;
  const int tail = (K % 128) != 0 ? nblk_full : -1;
  if (ACT_SMEM && warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(act_bar, uint32_t(R) * uint32_t(2 * K));
    __syncwarp();
    stage_bf16_rows(act_s, act, R, K, act_bar);
  }
  const bool act_ok = !ACT_SMEM || mbar_wait(act_bar, 0, &s_abort, status);
  for (int i = grp;; i += G) {
    const int u = blockIdx.x + i * gridDim.x;
    if (u >= n_units) break;
    const int st = i % S;
    // warp-uniform: the MMAs below run only if every lane saw the data land
    const bool ok = __all_sync(0xffffffffu, act_ok && mbar_wait(&full[st], (i / S) & 1, &s_abort, status));
    const int e = s_local[u % n_t];
    const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
    const int f0 = (u / n_t) * kDnRows + 16 * wj;  // this warp's 16 output features
    const uint8_t* s_c = ring + st * L.stage_bytes;
    const uint8_t* c_lo = s_c + (16 * wj + g) * (K / 2) + 16 * q;
    const uint8_t* c_hi = c_lo + 8 * (K / 2);
    const uint8_t* sc_lo = s_c + L.cbytes + (16 * wj + g) * srow;
    const uint8_t* sc_hi = sc_lo + 8 * srow;
    const float gsc = FMT == MOE_FMT_NVFP4_G16 ? dn.gscale[e - e_lo] : 0.f;
    const int ntiles = min(NT, (n_e + 7) / 8);
    ActFrags<ACT_SMEM> af;
    af.act = act;
    af.act_s = act_s;
    af.astride = astride;
    af.K = K;
    af.q = q;
    af.g = g;
    af.p0 = p0;
    af.n_e = n_e;
    float acc2[NT][2][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc2[j][0][c] = acc2[j][1][c] = 0.f;
    if (ok) stream_kblocks<FMT, NT>(acc2, 0, 1, nblk_full, tail, K, q, c_lo, c_hi, sc_lo, sc_hi, gsc, ntiles, af);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    if (!ok) continue;
    // c0, c1: feature f0 + g at columns 2q, 2q+1; c2, c3: feature + 8
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j >= ntiles) break;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = 8 * j + 2 * q + (c & 1);
        if (col < n_e)
          ypart[size_t(p0 + col) * H + f0 + g + 8 * (c >> 1)] = s_wrow[p0 + col] * (acc2[j][0][c] + acc2[j][1][c]);
      }
    }
  }
}

int max_touched(int T, int k, int E) { return (long(T) * k < E) ? T * k : E; }

// stages + staged token rows + the partial-tile buffers + routing state + barriers
size_t gate_up_smem(int fmt, int K, int NT, int E, int R, int x_rows) {
  const UnitLayout L = unit_layout(fmt, K, 16);
  return size_t(kStages) * L.stage_bytes + size_t(x_rows) * staged_row_stride(K) +
         size_t(kGroups) * 2 * kGroupWarps * NT * 128 * 4 + size_t(2 * (E + 1) + R) * 4 + 8 +
         (2 * kStages + 1) * 8;
}

size_t down_smem(int fmt, int K, int E, int R, int act_rows) {
  const UnitLayout L = unit_layout(fmt, K, kDnRows);
  return size_t(kStages) * L.stage_bytes + size_t(act_rows) * staged_row_stride(K) + size_t(2 * (E + 1) + R) * 4 +
         8 + (2 * kStages + 1) * 8;
}

// Staged token rows (gate_up) and activation rows (down) up to these sizes.
constexpr size_t kMaxStagedX = 36 * 1024;
constexpr size_t kMaxStagedAct = 36 * 1024;
constexpr size_t kMaxSmemPerCta = 226 * 1024;  // dynamic shared memory, leaving room for static

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
  const int R = T * s.top_k;
  const bool x_smem = size_t(T) * staged_row_stride(s.hidden) <= kMaxStagedX;
  auto k = x_smem ? decode_gate_up_kernel<FMT, NT, true> : decode_gate_up_kernel<FMT, NT, false>;
  const size_t smem = gate_up_smem(FMT, s.hidden, NT, s.num_experts, R, x_smem ? T : 0);
  if (smem > kMaxSmemPerCta) return cudaErrorInvalidConfiguration;
  cudaError_t err = allow_smem(k, smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, smem, units, kThreads);
  return launch_pdl(k, dim3(grid), dim3(kThreads), smem, stream, x, T, gu, s.inter, s.num_experts, s.top_k, er.lo,
                    er.hi, (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const int32_t*)ws.sorted_rows,
                    ws.act, ws.status);
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
                    cudaStream_t stream) {
  const int R = T * s.top_k;
  const bool act_smem = size_t(R) * staged_row_stride(s.inter) <= kMaxStagedAct;
  auto k = act_smem ? decode_down_kernel<FMT, NT, true> : decode_down_kernel<FMT, NT, false>;
  const size_t smem = down_smem(FMT, s.inter, s.num_experts, R, act_smem ? R : 0);
  if (smem > kMaxSmemPerCta) return cudaErrorInvalidConfiguration;
  cudaError_t err = allow_smem(k, smem);
  if (err != cudaSuccess) return err;
  const int units = std::min(max_touched(T, s.top_k, s.num_experts), er.hi - er.lo) * (s.hidden / kDnRows);
  const int grid = persistent_grid(k, smem, std::max(units, 1), kThreads);
  return launch_pdl(k, dim3(grid), dim3(kThreads), smem, stream, dn, T, s.num_experts, s.top_k, er.lo, er.hi,
                    (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const int32_t*)ws.sorted_rows,
                    (const uint16_t*)ws.act, (const float*)ws.topk_w, ws.ypart, ws.status);
}

template <int FMT>
cudaError_t down_fmt(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er, const Workspace& ws,
                     cudaStream_t stream) {
  if (T <= 8) return down_nt<FMT, 1>(s, T, dn, er, ws, stream);
  if (T <= 16) return down_nt<FMT, 2>(s, T, dn, er, ws, stream);
  return down_nt<FMT, 4>(s, T, dn, er, ws, stream);
}

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
  if (T > kDecodeMaxT) return false;
  const int R = T * s.top_k;
  const int NT = T <= 8 ? 1 : T <= 16 ? 2 : 4;
  const bool x_smem = size_t(T) * staged_row_stride(s.hidden) <= kMaxStagedX;
  const bool act_smem = size_t(R) * staged_row_stride(s.inter) <= kMaxStagedAct;
  return gate_up_smem(s.fmt, s.hidden, NT, s.num_experts, R, x_smem ? T : 0) <= kMaxSmemPerCta &&
         down_smem(s.fmt, s.inter, s.num_experts, R, act_smem ? R : 0) <= kMaxSmemPerCta;
}

size_t decode_ypart_bytes(const moe_shape_t& s, int T) {
  return T <= kDecodeMaxT ? size_t(T) * s.top_k * s.hidden * 4 : 0;
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
                               const Workspace& ws, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128) return down_fmt<MOE_FMT_INT4_G128>(s, T, dn, er, ws, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return down_fmt<MOE_FMT_NVFP4_G16>(s, T, dn, er, ws, stream);
  return down_fmt<MOE_FMT_MXFP4_G32>(s, T, dn, er, ws, stream);
}

}  // namespace moe
