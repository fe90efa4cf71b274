// Decode path (small token counts, T <= 32): weight-streaming expert GEMVs.
//
// The time goes into streaming the touched experts' packed weights from HBM
// ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", Measured: at concurrency 32
// the bottleneck is weight bandwidth).  Consumer warps dequantise in
// registers (decode_common.cuh) and feed mma.sync m16n8k16 with up to 32
// tokens; small token sets are staged in shared memory once per CTA in MMA
// fragment order (the down kernel reads its activation rows through L2), and
// the routing state (touched experts, per-expert row offsets, the rows'
// tokens) is read into shared memory once per CTA.
//
// gate_up: persistent; CTA c takes the (touched expert, 8- or 16-feature)
// units c, c + grid, ....  One producer warp starts, per unit, two bulk
// copies (the unit's gate rows, its up rows: contiguous 8-16 KB ranges) and
// two of their scales into a ring of shared-memory stages, and prefetches the
// unit that will next refill the stage into L2; four consumer warps split
// each unit's k-blocks and sum in shared memory.  Few large copies: the
// bulk-copy engine's cost is per copy as much as per byte.
// down: CTA c owns 16 output features of every token and runs over all
// touched experts, so the routing-weighted combine of a token's k expert
// outputs happens in the CTA (in slot order, deterministic) and the output is
// written once.  Its 16-row weight tiles are small (16 rows x I/2 bytes), so
// each warp loads its tiles straight into registers (16 warps per CTA with
// one chunk each for INT4 and up to 8 tokens in every format; otherwise 8
// warps with the next chunk's loads in flight during the multiply), the
// first chunk's loads issued before the programmatic-launch wait; gate_up has
// requested the tiles into L2.
// Template parameter SH (both kernels): the bf16 shared expert rides along;
// gate_up turns the routing GEMV's split partials of its rows into its
// SwiGLU activation and gate, and down adds its gated down product to the
// combine.  Without SH neither kernel carries any of that code.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "decode_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kGroupWarps = 4;  // gate_up: consumer warps per work unit

// Build-time tuning knobs (the defaults are the measured best): gate_up
// consumer groups per CTA and its largest stage ring.
#ifndef MOE_DEC_GROUPS
#define MOE_DEC_GROUPS 2
#endif
#ifndef MOE_DEC_STAGES
#define MOE_DEC_STAGES 4
#endif
// gate_up unit size and CTAs per SM by token tiles (NT): with one token tile,
// 8-feature units (one 16-row MMA tile) and registers for two CTAs per SM,
// so twice the warps hide the latency (measured faster); more token tiles
// need the registers of one CTA per SM and share each activation fragment
// between two MMA tiles (16-feature units).
__host__ __device__ constexpr int gu_mt(int NT) { return NT == 1 ? 1 : 2; }
__host__ __device__ constexpr int gu_feat(int NT) { return 8 * gu_mt(NT); }
constexpr int gu_ctas(int NT) { return NT == 1 ? 2 : 1; }
constexpr int kGuGroups = MOE_DEC_GROUPS;
constexpr int kGuMaxStages = MOE_DEC_STAGES;
constexpr int kGuThreads = (kGuGroups * kGroupWarps + 1) * 32;
constexpr int kDnRows = 16;  // output features per down tile
// down warps per CTA: 16, each holding one register chunk (the other warps
// hide a chunk's loads; with one token tile measured 6 % faster than 8 warps
// with the next chunk's loads in flight, at 32 INT4 tokens 27 % faster);
// MXFP4 / NVFP4 with more token tiles need the registers of 8 warps, each
// with the next chunk in flight during the multiply.
constexpr int dn_warps(int NT, int FMT) { return NT == 1 || FMT == MOE_FMT_INT4_G128 ? 16 : 8; }
constexpr int dn_threads(int NT, int FMT) { return 32 * dn_warps(NT, FMT); }
constexpr int dn_regs(int NT, int FMT) {  // at most 65536 / threads, 8-aligned
  return dn_warps(NT, FMT) == 16 ? 128 : 224;
}
constexpr uint32_t kProducerSleepNs = 64;  // gate_up producer: sleep between tries for a free stage
constexpr int kDnPrefetchRows = 64;         // down-matrix rows per L2 prefetch issued by gate_up

// Offsets inside one gate_up stage: gate-row codes, 64 bytes of padding,
// up-row codes, then gate-row and up-row scales (see decode_common.cuh).
struct GuLayout {
  int cA, cB, sA, sB, stage_bytes;
};
__host__ __device__ inline GuLayout gu_layout(int fmt, int K, int feat) {
  const int run = feat * (K / 2), srun = feat * scale_row_bytes(fmt, K);
  GuLayout l;
  l.cA = 0;
  l.cB = run + 64;
  l.sA = 2 * run + 64;
  l.sB = l.sA + srun;
  l.stage_bytes = (l.sB + srun + 127) & ~127;
  return l;
}

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

// The shared expert's SwiGLU activation and sigmoid gate from the routing
// GEMV's split partials (summed in split order): a[t][i] = bf16(silu(h_gate)
// * h_up), g[t] = sigmoid(z_t).  The T * I_s features, then the T gates, are
// spread over the grid: thread `tid` of `nthreads` per CTA.
MOE_DEV void shared_activation(const SharedFold& sf, int T, int tid, int nthreads) {
  const int I = sf.inter, N2 = 2 * I + 1, n = T * I + T;
  for (int e = int(blockIdx.x) * nthreads + tid; e < n; e += int(gridDim.x) * nthreads) {
    if (e < T * I) {
      const int t = e / I, i = e - t * I;
      float hg = 0.f, hu = 0.f;
      for (int sp = 0; sp < sf.splits; ++sp) {
        const float* hs = sf.h + (size_t(sp) * T + t) * N2;
        hg += __ldcg(hs + i);
        hu += __ldcg(hs + I + i);
      }
      sf.a[size_t(t) * I + i] = f32_to_bf16_rn(silu_mul(hg, hu));
    } else {
      const int t = e - T * I;
      float z = 0.f;
      for (int sp = 0; sp < sf.splits; ++sp) z += __ldcg(sf.h + (size_t(sp) * T + t) * N2 + 2 * I);
      sf.g[t] = 1.0f / (1.0f + expf(-z));
    }
  }
}

// Sub-unit i of the shared expert's down product for one 16-feature tile: the
// tile's bf16 rows over k in [128 i, 128 i + 128) times the activation of
// every token, one warp; ys[t][f] (fp32, 16 features per token) gets the
// partial product.  The activation was written by the kernel before (read
// through L2); the rows are constant.
template <int NT>
MOE_DEV void shared_down_part(const SharedFold& sf, int T, int tile, int i, int g, int q, float* ys) {
  const int I = sf.inter;
  const int k = 128 * i + 32 * q;
  const bool kin = k < I;  // I % 64 == 0: a lane's 32-k slice is whole or past I
  const uint16_t* w = sf.w_down + size_t(tile * kDnRows + g) * I + k;
  uint32_t alo[8][2], ahi[8][2];
  act_frags_global<1>(w, kin, alo);
  act_frags_global<1>(w + size_t(8) * I, kin, ahi);
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    if (8 * j >= T) break;
    const int t = 8 * j + g;
    uint32_t bf[8][2];
    act_frags_global<2>(sf.a + size_t(t < T ? t : 0) * I + k, kin && t < T, bf);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int st = 0; st < 8; ++st) {
      const uint32_t a[4] = {alo[st][0], ahi[st][0], alo[st][1], ahi[st][1]};
      mma_bf16_16816(acc, a, bf[st][0], bf[st][1]);
    }
    // c0, c1: feature g at tokens 2q, 2q+1; c2, c3: feature g + 8
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = 8 * j + 2 * q + (c & 1);
      if (tok < T) ys[tok * kDnRows + g + 8 * (c >> 1)] = acc[c];
    }
  }
}

// Let the last bulk copies of this CTA's producer land before its shared
// memory is released (bounded: they complete unless the GPU is failing).
MOE_DEV void drain_stages(uint64_t* full, int issued, int S) {
  for (int i = max(0, issued - S); i < issued; ++i) mbar_wait_drain(&full[i % S], (i / S) & 1, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// gate_up + SwiGLU.  Work unit u = (touched slot u / (I/16), features
// f0 = 16 (u % (I/16)) .. f0 + 15): its 32 weight rows are the 16 gate rows
// f0.. and the 16 matching up rows I + f0.., staged as two runs.  Lane g of
// MMA tile t (features f0 + 8t ..) takes feature f0 + 8t + g's gate row and up
// row as its two MMA rows (low / high; swapped for odd g), so the C fragment
// holds gate and up of the same feature and token: SwiGLU needs no shuffle.
// CTA c takes units c, c + grid, ...; its i-th goes to stage i % S and
// consumer group i % G.  The group's four warps split K (128-k
// blocks w, w + 4, ...), and one of them (rotating) sums the four partial
// tiles in warp order and writes a = bf16(silu(gate) * up) to act[p][f] for
// the expert's sorted rows p.  With X_SMEM (small T) the consumers first
// stage the T token rows in fragment order, before the programmatic-launch
// wait.
// ---------------------------------------------------------------------------
template <int FMT, int NT, bool X_SMEM, bool SH>
__global__ void __launch_bounds__(kGuThreads, gu_ctas(NT)) decode_gate_up_kernel(
    const uint16_t* __restrict__ x, int T, Bank gu, int I, int E, int top_k, int e_lo, int e_hi,
    const int32_t* __restrict__ touched, const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows,
    uint16_t* __restrict__ act, uint32_t* status, int S, Bank dn, SharedFold sf) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int G = kGuGroups, MT = gu_mt(NT), FEAT = gu_feat(NT), CH = MT == 1 && NT == 1 ? 4 : 2;
  constexpr int kRed = kGroupWarps * NT * MT * 128;  // floats of one group's partial tiles
  const int K = gu.K, R = T * top_k;
  const GuLayout L = gu_layout(FMT, K, FEAT);
  const int srow = scale_row_bytes(FMT, K);
  const int pstride = staged_act_stride(K);
  uint8_t* ring = smem;                                                      // [S][stage]
  uint8_t* x_s = ring + size_t(S) * L.stage_bytes;                           // [T][pstride] (X_SMEM)
  float* red = reinterpret_cast<float*>(x_s + (X_SMEM ? size_t(T) * pstride : 0));  // [G][2][kRed]
  int* s_touched = reinterpret_cast<int*>(red + G * 2 * kRed);
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
  // The token rows do not depend on the kernel just before: every kernel of
  // the forward waits for its predecessor before it lets its dependents
  // launch, so x's producer finished before this kernel started.  Staged
  // before the wait (published by the block barrier below).
  if (X_SMEM && warp < G * kGroupWarps) stage_act_rows<1>(x_s, x, T, K, threadIdx.x, G * kGroupWarps * 32);
  pdl_wait();
  pdl_trigger();
  load_routing(s_touched, s_off, touched, offsets, E);
  for (int p = threadIdx.x; p < R; p += blockDim.x) s_tok[p] = __ldcg(sorted_rows + p) / top_k;
  __syncthreads();
  int t_lo, t_hi;
  local_slice(s_touched, e_lo, e_hi, E, s_cnt, &t_lo, &t_hi);
  const int* s_local = s_touched + 1 + t_lo;  // the bank's touched experts (global ids)
  const int ftiles = I / FEAT;
  const int n_units = (t_hi - t_lo) * ftiles;
  // CTA c takes units c, c + grid, ...: a popular expert's units spread over
  // many CTAs (its extra token tiles are work the CTAs share)
  const int grid = int(gridDim.x);
  const int cnt = n_units > int(blockIdx.x) ? (n_units - int(blockIdx.x) + grid - 1) / grid : 0;
  // SH: the shared expert's activation and gate, by the consumer threads
  // while the producer's first copies are in flight
  if (SH && warp < G * kGroupWarps) shared_activation(sf, T, threadIdx.x, G * kGroupWarps * 32);
  if (cnt <= 0) return;
  const int g_slot = grid / ftiles, g_ft = grid - g_slot * ftiles;  // a step of `grid` units
  auto advance = [&](int& sl, int& f, int steps) {  // (slot, feature tile) `steps` x grid units on
    for (int a = 0; a < steps; ++a) {
      sl += g_slot;
      f += g_ft;
      if (f >= ftiles) f -= ftiles, ++sl;
    }
  };

  if (warp == G * kGroupWarps) {
    // ---------------------------------------------------------------- producer
    const uint64_t policy = l2_policy_evict_first();
    const uint32_t run = uint32_t(FEAT * (K / 2)), srun = uint32_t(FEAT * srow);
    const uint8_t* scales = static_cast<const uint8_t*>(gu.scales);
    int slot = int(blockIdx.x) / ftiles, ft = int(blockIdx.x) - slot * ftiles;  // unit i
    int pslot = slot, pft = ft;                                                // unit i + S
    advance(pslot, pft, S);
    // This CTA's share of the touched experts' down matrices into L2 for the
    // down kernel that follows: pieces of kDnPrefetchRows rows, the CTA's
    // j-th piece is piece blockIdx.x + j * grid.
    const int dn_per_e = dn.codes ? dn.N / kDnPrefetchRows : 0;
    const int dn_pieces = (t_hi - t_lo) * dn_per_e;
    auto prefetch_down = [&](int j) {
      const int p = blockIdx.x + j * gridDim.x;
      if (p >= dn_pieces) return;
      const int ex = p / dn_per_e;
      const long row = long(s_local[ex] - e_lo) * dn.N + (p - ex * dn_per_e) * kDnPrefetchRows;
      prefetch_codes<FMT>(dn, row, kDnPrefetchRows);
      prefetch_scales<FMT>(dn, row, kDnPrefetchRows);
    };
    int pf_next = 0;  // the CTA's next piece
    int i = 0, st = 0, ph = 0;  // unit i's stage and that stage's use count parity
    for (; i < cnt; ++i) {
      if (i >= S &&
          !__all_sync(0xffffffffu, mbar_wait_backoff(&empty[st], ph ^ 1, &s_abort, status, kProducerSleepNs)))
        break;
      fence_proxy_async_smem();  // earlier generic-proxy reads of this stage before the refill
      if (lane == 0) mbar_arrive_expect_tx(&full[st], 2 * run + 2 * srun);
      __syncwarp();
      if (lane < 4) {
        // lane 0 / 1: gate / up codes; lane 2 / 3: their scales
        const long row = long(s_local[slot] - e_lo) * gu.N + ft * FEAT + ((lane & 1) ? I : 0);
        uint8_t* stage = ring + size_t(st) * L.stage_bytes;
        if (lane < 2) bulk_g2s_hint(stage + (lane ? L.cB : L.cA), gu.codes + row * (K / 2), run, &full[st], policy);
        else bulk_g2s_hint(stage + (lane & 1 ? L.sB : L.sA), scales + row * srow, srun, &full[st], policy);
      } else if (lane < 8) {
        if (i + S < cnt) {
          // the unit that will refill this stage, into L2 ahead of time
          const long row = long(s_local[pslot] - e_lo) * gu.N + pft * FEAT + ((lane & 1) ? I : 0);
          if (lane < 6) prefetch_codes<FMT>(gu, row, FEAT);
          else prefetch_scales<FMT>(gu, row, FEAT);
        }
      } else if (lane < 12 && i >= S) {
        prefetch_down(pf_next + lane - 8);  // once the ring is primed: four pieces per unit
      }
      if (i >= S) pf_next += 4;
      if (++st == S) st = 0, ph ^= 1;
      advance(slot, ft, 1);
      advance(pslot, pft, 1);
    }
    // the rest of the share, one piece per lane
    for (int j = pf_next + lane; blockIdx.x + j * int(gridDim.x) < dn_pieces; j += 32) prefetch_down(j);
    if (lane == 0) drain_stages(full, i, S);
    return;
  }

  // -------------------------------------------------------------------- consumers
  const int grp = warp / kGroupWarps, wj = warp % kGroupWarps;
  const int g = lane >> 2, q = lane & 3;
  const bool odd = (g & 1) != 0;  // this lane's low MMA row is the up row
  const int nfull = K / 128;  // blocks where every lane slice lies inside K
  const int my_full = wj < nfull ? (nfull - wj + kGroupWarps - 1) / kGroupWarps : 0;
  const int tail_b = ((K % 128) != 0 && nfull % kGroupWarps == wj) ? nfull : -1;
  const int lo_c = odd ? L.cB : L.cA, hi_c = odd ? L.cA : L.cB;
  const int lo_s = odd ? L.sB : L.sA, hi_s = odd ? L.sA : L.sB;
  int slot = int(blockIdx.x) / ftiles, ft = int(blockIdx.x) - slot * ftiles;
  advance(slot, ft, grp);
  int st = grp, ph = 0;
  for (int i = grp, n = 0; i < cnt; i += G, ++n) {
    // warp-uniform: the MMAs below run only if every lane saw the data land
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[st], ph, &s_abort, status));
    const int e = s_local[slot];
    const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
    const int f0 = ft * FEAT;
    const uint8_t* s_c = ring + size_t(st) * L.stage_bytes;
    const uint8_t* c_lo[MT];
    const uint8_t* c_hi[MT];
    const uint8_t* sc_lo[MT];
    const uint8_t* sc_hi[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int fi = 8 * t + g;
      c_lo[t] = s_c + lo_c + fi * (K / 2) + 16 * q;
      c_hi[t] = s_c + hi_c + fi * (K / 2) + 16 * q;
      sc_lo[t] = s_c + lo_s + fi * srow;
      sc_hi[t] = s_c + hi_s + fi * srow;
    }
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
    float acc[NT][MT][CH][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int h = 0; h < CH; ++h)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[j][t][h][c] = 0.f;
    // blocks four at a time (fewer with more token tiles: registers)
    constexpr int UNB = NT == 1 ? 4 : NT == 2 ? 2 : 1;
    if (ok)
      smem_unit<FMT, NT, MT, CH, UNB>(acc, c_lo, c_hi, sc_lo, sc_hi, wj, kGroupWarps, my_full, tail_b, K, q, gsc, ntiles,
                                      xf);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
    // the group's partial tiles, double-buffered by unit parity
    float* red_u = red + size_t(grp * 2 + (n & 1)) * kRed;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v = acc[j][t][0][c];
#pragma unroll
          for (int h = 1; h < CH; ++h) v += acc[j][t][h][c];
          red_u[(((wj * NT + j) * MT + t) * 4 + c) * 32 + lane] = v;
        }
    named_barrier_sync(2 + grp, kGroupWarps * 32);
    if (ok && wj == n % kGroupWarps) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (j >= ntiles) break;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          float sum[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            sum[c] = 0.f;
#pragma unroll
            for (int w = 0; w < kGroupWarps; ++w) sum[c] += red_u[(((w * NT + j) * MT + t) * 4 + c) * 32 + lane];
          }
          // c0, c1: low row at columns 2q, 2q+1; c2, c3: high row (gate low for even g)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = 8 * j + 2 * q + hh;
            const float gate = odd ? sum[2 + hh] : sum[hh], up = odd ? sum[hh] : sum[2 + hh];
            if (col < n_e) act[size_t(p0 + col) * I + f0 + 8 * t + g] = f32_to_bf16_rn(silu_mul(gate, up));
          }
        }
      }
    }
    st += G;
    if (st >= S) st -= S, ph ^= 1;
    advance(slot, ft, G);
  }
}

// ---------------------------------------------------------------------------
// down projection and combine.  CTA c owns the 16 output features of tiles
// c, c + grid, ... (H / 16 tiles).  For a tile, work unit s = the tile's 16
// rows of the down matrix of touched expert s (all of K = I), taken by warp
// s % W, in chunks of four 128-k blocks loaded into registers; the next
// chunk's loads are issued before the current chunk is multiplied.  The
// unit's C fragment times the routing weight of each column's (token, slot)
// goes to ybuf[t k + j][f] in shared memory.  When the tile's units are
// done, each token's output is the sum of its k slots in slot order (plus
// the shared expert's gated output), rounded once to bf16, or the fp32 sum
// (an expert-parallel shard's partial: slots of other shards' experts stay
// zero).  The weights do not depend on the gate_up kernel that runs just
// before: the routing state was written two launches back (and the kernel in
// between triggers its dependents only after its own wait), so every warp
// requests its tiles into L2 and loads its first chunk before the
// programmatic-launch wait.  With ACT_SMEM (a build with a non-zero staging
// threshold, small T) the warps then stage the T*k activation rows in
// fragment order; otherwise the fragments are read through L2.
// ---------------------------------------------------------------------------
template <int FMT, int NT, bool ACT_SMEM, bool SH>
__global__ void __maxnreg__(dn_regs(NT, FMT)) decode_down_kernel(
    Bank dn, int T, int E, int top_k, int e_lo, int e_hi, const int32_t* __restrict__ touched,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows, const uint16_t* __restrict__ act,
    const float* __restrict__ topk_w, const float* __restrict__ sh_gate, const float* __restrict__ sh_y,
    uint16_t* __restrict__ out, float* __restrict__ partial_out, SharedFold sf) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int W = dn_warps(NT, FMT), kThreads = dn_threads(NT, FMT);
  constexpr bool kOneChunk = W > 8;
  constexpr int CH = NT == 1 ? 4 : 2;
  const int H = dn.N, K = dn.K;  // K = I
  const int R = T * top_k;
  const int srow = scale_row_bytes(FMT, K);
  const int pstride = staged_act_stride(K);
  uint8_t* act_s = smem;                                          // [R][pstride] (ACT_SMEM)
  float* ybuf = reinterpret_cast<float*>(act_s + (ACT_SMEM ? size_t(R) * pstride : 0));  // [R][16]
  int* s_touched = reinterpret_cast<int*>(ybuf + R * kDnRows);
  int* s_off = s_touched + (E + 1);
  int* s_slot = s_off + (E + 1);                                  // [R] slot t k + j of sorted row p
  float* s_w = reinterpret_cast<float*>(s_slot + R);              // [R] its routing weight
  float* s_sh = s_w + R;  // [nsu][T][16] the shared expert's down sub-unit products (with sf)
  const int nsu = SH ? (sf.inter + 127) / 128 : 0;
  __shared__ int s_cnt[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
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
  const int nblk = kblocks(K), nch = (nblk + 3) / 4;  // k-blocks and chunks of four per unit
  const uint8_t* scales = static_cast<const uint8_t*>(dn.scales);
  const int my_units = warp < n_t ? (n_t - warp + W - 1) / W : 0;  // per tile
  const int nk = my_units * nch;                                   // chunks per tile
  // the tile's outputs: each token's k slots summed in slot order, two
  // features per thread (block barriers before and after: ybuf is complete,
  // then cleared for the next tile)
  auto finish_tile = [&](int tile) {
    __syncthreads();
    for (int o = threadIdx.x; o < T * (kDnRows / 2); o += kThreads) {
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
        if (SH) {
          // the shared expert: its sub-units summed in k order, times the gate
          const float* ys = s_sh + t * kDnRows + f;
          float y0 = ys[0], y1 = ys[1];
          for (int i = 1; i < nsu; ++i) {
            y0 += ys[i * T * kDnRows];
            y1 += ys[i * T * kDnRows + 1];
          }
          const float gg = __ldcg(sf.g + t);
          v0 += gg * y0;
          v1 += gg * y1;
        }
        *reinterpret_cast<uint32_t*>(out + oi) = pack_bf16x2(v0, v1);
      }
    }
    __syncthreads();
  };
  if (lane < my_units && blockIdx.x < ntile) {
    // all of this warp's tiles of the CTA's first tile into L2
    const long r0 = long(s_local[warp + W * lane] - e_lo) * H + blockIdx.x * kDnRows;
    prefetch_codes<FMT>(dn, r0, kDnRows);
    prefetch_scales<FMT>(dn, r0, kDnRows);
  }
  if (SH && threadIdx.x == 0 && blockIdx.x < ntile)  // the shared expert's rows of the first tile
    bulk_prefetch_l2(sf.w_down + size_t(blockIdx.x) * kDnRows * sf.inter, uint32_t(kDnRows * sf.inter * 2));
  // The tile loop; FULL (every chunk is four whole k-blocks) drops the
  // bounds checks of the chunk loads and multiplies.
  auto run = [&](auto full_tag) {
    constexpr bool FULL = decltype(full_tag)::value;
    // chunk k of this warp's units: unit m = k / nch, chunk k % nch
    auto load = [&](RegChunk& c, int tile, int k) {
      const int m = nch == 1 ? k : k / nch, ch = k - m * nch;
      const long r = long(s_local[warp + W * m] - e_lo) * H + tile * kDnRows + g;
      const uint8_t* c_lo = dn.codes + r * (K / 2) + 16 * q;
      const uint8_t* s_lo = scales + r * srow;
      load_chunk<FMT, FULL>(c, c_lo, c_lo + 8 * (K / 2), s_lo, s_lo + 8 * srow, 4 * ch, nblk, K, q);
    };
    RegChunk cA, cB;
    if (nk > 0 && blockIdx.x < ntile) load(cA, blockIdx.x, 0);

    pdl_wait();  // the activations (and the previous readers of the output) of the kernels before
    pdl_trigger();
    if (ACT_SMEM) {
      stage_act_rows<2>(act_s, act, R, K, threadIdx.x, kThreads);
      __syncthreads();
    }
    for (int tile = blockIdx.x; tile < ntile; tile += gridDim.x) {
      if (tile != int(blockIdx.x) && nk > 0) load(cA, tile, 0);
      float acc[NT][CH][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int h = 0; h < CH; ++h)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[j][h][c] = 0.f;
      // multiply chunk k (in `cur`); after a unit's last chunk, its weighted
      // outputs go to ybuf and the accumulators restart
      auto step = [&](const RegChunk& cur, int k) {
        const int m = nch == 1 ? k : k / nch, ch = k - m * nch;
        const int e = s_local[warp + W * m];
        const int p0 = s_off[e], n_e = s_off[e + 1] - p0;
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
        chunk_mma<FMT, NT, CH, FULL>(acc, cur, 4 * ch, nblk, K, q, gsc, ntiles, af);
        if (ch != nch - 1) return;
        // c0, c1: feature g at columns 2q, 2q+1; c2, c3: feature g + 8
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (j < ntiles) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = 8 * j + 2 * q + (c & 1);
              float v = acc[j][0][c];
#pragma unroll
              for (int h = 1; h < CH; ++h) v += acc[j][h][c];
              if (col < n_e) ybuf[s_slot[p0 + col] * kDnRows + g + 8 * (c >> 1)] = s_w[p0 + col] * v;
            }
          }
#pragma unroll
          for (int h = 0; h < CH; ++h)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[j][h][c] = 0.f;
        }
      };
      if (kOneChunk) {
        for (int k = 0; k < nk; ++k) {
          if (k > 0) load(cA, tile, k);
          step(cA, k);
        }
      } else {
        for (int k = 0; k < nk;) {
          if (k + 1 < nk) load(cB, tile, k + 1);
          step(cA, k);
          if (++k >= nk) break;
          if (k + 1 < nk) load(cA, tile, k + 1);
          step(cB, k);
          ++k;
        }
      }
      // the shared expert's sub-units: the warps after the last routed unit's
      if (SH)
        for (int i = 0; i < nsu; ++i)
          if (warp == (n_t + i) % W) shared_down_part<NT>(sf, T, tile, i, g, q, s_sh + i * T * kDnRows);
      finish_tile(tile);
    }
  };
  if (K % 512 == 0) run(std::true_type{});
  else run(std::false_type{});
}

int max_touched(int T, int k, int E) { return (long(T) * k < E) ? T * k : E; }

constexpr size_t kMaxSmemPerCta = 226 * 1024;  // dynamic shared memory, leaving room for static
constexpr size_t kSmemPerSm = 228 * 1024;       // shared memory of one SM
constexpr size_t kSmemReservedPerCta = 2 * 1024;  // the system's share per CTA and the kernels' static arrays
// Staged token rows (gate_up) and activation rows (down) up to these sizes.
// The down kernel reads the activation rows through L2 by default: staging
// them costs a block barrier before the first multiply, which measured
// slower (4 tokens: down stage 14.6 us without staging, 15.5 us with).
#ifndef MOE_DEC_MAX_STAGED_ACT_KB
#define MOE_DEC_MAX_STAGED_ACT_KB 0
#endif
constexpr size_t kMaxStagedX = 72 * 1024;
constexpr size_t kMaxStagedAct = size_t(MOE_DEC_MAX_STAGED_ACT_KB) * 1024;

int nt_of(int T) { return T <= 8 ? 1 : T <= 16 ? 2 : 4; }

// gate_up: stages + staged token rows + the partial-tile buffers + routing
// state + barriers
size_t gate_up_smem(int fmt, int K, int NT, int E, int R, int x_rows, int S) {
  return size_t(S) * gu_layout(fmt, K, gu_feat(NT)).stage_bytes + size_t(x_rows) * staged_act_stride(K) +
         size_t(kGuGroups) * 2 * kGroupWarps * NT * gu_mt(NT) * 128 * 4 + size_t(2 * (E + 1) + R) * 4 + 8 +
         2 * size_t(S) * 8;
}

// down: staged activation rows + the slot outputs + routing state (+ the
// shared expert's sub-unit products)
size_t down_smem(int E, int R, int K, int act_rows, int T, bool shared) {
  return size_t(act_rows) * staged_act_stride(K) + size_t(R) * kDnRows * 4 + size_t(2 * (E + 1) + 2 * R) * 4 +
         (shared ? size_t(kSharedFoldMaxInter / 128) * T * kDnRows * 4 : 0);
}

struct GuPlan {
  bool x_smem;
  int S;
  size_t smem;
};
struct DnPlan {
  bool act_smem;
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
  // the largest ring that leaves room for gu_ctas(NT) CTAs per SM, else the
  // largest that fits one CTA
  const size_t shared_budget = kSmemPerSm / gu_ctas(NT) - kSmemReservedPerCta;
  for (size_t budget : {std::min(shared_budget, kMaxSmemPerCta), kMaxSmemPerCta}) {
    for (int S = kGuMaxStages / kGuGroups * kGuGroups; S >= 2 * kGuGroups; S -= kGuGroups) {
      const size_t b = gate_up_smem(s.fmt, s.hidden, NT, s.num_experts, R, p.x_smem ? T : 0, S);
      if (b <= budget) {
        p.S = S;
        p.smem = b;
        return p;
      }
    }
  }
  return p;
}

DnPlan down_plan(const moe_shape_t& s, int T, bool shared = false) {
  const int R = T * s.top_k;
  DnPlan p;
  p.act_smem = size_t(R) * staged_act_stride(s.inter) <= kMaxStagedAct;
  p.smem = down_smem(s.num_experts, R, s.inter, p.act_smem ? R : 0, T, shared);
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
cudaError_t gate_up_nt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Bank& dn,
                       const ExpertRange& er, const Workspace& ws, int units, const SharedFold& sf,
                       cudaStream_t stream) {
  const GuPlan p = gate_up_plan(s, T);
  if (p.S == 0) return cudaErrorInvalidConfiguration;
  const bool sh = sf.h != nullptr;
  auto k = p.x_smem ? (sh ? decode_gate_up_kernel<FMT, NT, true, true> : decode_gate_up_kernel<FMT, NT, true, false>)
                    : (sh ? decode_gate_up_kernel<FMT, NT, false, true> : decode_gate_up_kernel<FMT, NT, false, false>);
  cudaError_t err = allow_smem(k, p.smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, p.smem, units, kGuThreads);
  return launch_pdl(k, dim3(grid), dim3(kGuThreads), p.smem, stream, x, T, gu, s.inter, s.num_experts, s.top_k,
                    er.lo, er.hi, (const int32_t*)ws.touched, (const int32_t*)ws.offsets,
                    (const int32_t*)ws.sorted_rows, ws.act, ws.status, p.S, dn, sf);
}

template <int FMT>
cudaError_t gate_up_fmt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Bank& dn,
                        const ExpertRange& er, const Workspace& ws, int units, const SharedFold& sf,
                        cudaStream_t stream) {
  // token tiles of 8 held in registers: enough for the largest possible expert batch (T)
  if (T <= 8) return gate_up_nt<FMT, 1>(s, T, x, gu, dn, er, ws, units, sf, stream);
  if (T <= 16) return gate_up_nt<FMT, 2>(s, T, x, gu, dn, er, ws, units, sf, stream);
  return gate_up_nt<FMT, 4>(s, T, x, gu, dn, er, ws, units, sf, stream);
}

// The down kernel's instantiation: staged activations only when the build
// allows staging at all (MOE_DEC_MAX_STAGED_ACT_KB > 0).
template <int FMT, int NT>
auto down_kernel_for(bool act_smem, bool sh) {
  if constexpr (kMaxStagedAct > 0) {
    if (act_smem) return sh ? decode_down_kernel<FMT, NT, true, true> : decode_down_kernel<FMT, NT, true, false>;
  }
  (void)act_smem;
  return sh ? decode_down_kernel<FMT, NT, false, true> : decode_down_kernel<FMT, NT, false, false>;
}

template <int FMT, int NT>
cudaError_t down_nt(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er, const Workspace& ws,
                    const float* sh_gate, const float* sh_y, uint16_t* out, float* partial_out,
                    const SharedFold& sf, cudaStream_t stream) {
  const DnPlan p = down_plan(s, T, sf.w_down != nullptr);
  if (p.smem > kMaxSmemPerCta) return cudaErrorInvalidConfiguration;
  auto k = down_kernel_for<FMT, NT>(p.act_smem, sf.w_down != nullptr);
  cudaError_t err = allow_smem(k, p.smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, p.smem, s.hidden / kDnRows, dn_threads(NT, FMT));
  return launch_pdl(k, dim3(grid), dim3(dn_threads(NT, FMT)), p.smem, stream, dn, T, s.num_experts, s.top_k, er.lo, er.hi,
                    (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const int32_t*)ws.sorted_rows,
                    (const uint16_t*)ws.act, (const float*)ws.topk_w, sh_gate, sh_y, out, partial_out, sf);
}

template <int FMT>
cudaError_t down_fmt(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er, const Workspace& ws,
                     const float* sh_gate, const float* sh_y, uint16_t* out, float* partial_out,
                     const SharedFold& sf, cudaStream_t stream) {
  if (T <= 8) return down_nt<FMT, 1>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, sf, stream);
  if (T <= 16) return down_nt<FMT, 2>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, sf, stream);
  return down_nt<FMT, 4>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, sf, stream);
}

}  // namespace

bool decode_supported(const moe_shape_t& s, int T) {
  if (T > kDecodeMaxT) return false;
  return gate_up_plan(s, T).S > 0 && down_plan(s, T).smem <= kMaxSmemPerCta;
}

bool decode_shared_fits(const moe_shape_t& s, int T) {
  return decode_supported(s, T) && down_plan(s, T, true).smem <= kMaxSmemPerCta;
}

cudaError_t launch_decode_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Bank& dn,
                                  const ExpertRange& er, const Workspace& ws, cudaStream_t stream,
                                  const SharedFold* sf) {
  const SharedFold shf = sf ? *sf : SharedFold{};
  int units = std::min(max_touched(T, s.top_k, s.num_experts), er.hi - er.lo) * (s.inter / gu_feat(nt_of(T)));
  if (units <= 0) {
    if (!sf || T == 0) return cudaSuccess;
    units = 1;  // no routed unit, but the shared expert's activation is due
  }
  Bank pf = dn;
  if (s.hidden % kDnPrefetchRows) pf.codes = nullptr;  // whole pieces only
  if (s.fmt == MOE_FMT_INT4_G128) return gate_up_fmt<MOE_FMT_INT4_G128>(s, T, x, gu, pf, er, ws, units, shf, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return gate_up_fmt<MOE_FMT_NVFP4_G16>(s, T, x, gu, pf, er, ws, units, shf, stream);
  return gate_up_fmt<MOE_FMT_MXFP4_G32>(s, T, x, gu, pf, er, ws, units, shf, stream);
}

cudaError_t launch_decode_down(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er,
                               const Workspace& ws, const float* sh_gate, const float* sh_y, uint16_t* out,
                               float* partial_out, cudaStream_t stream, const SharedFold* sf) {
  if (T == 0) return cudaSuccess;
  if (sf && partial_out) return cudaErrorInvalidValue;  // the shared term belongs to the bf16 output only
  const SharedFold shf = sf ? *sf : SharedFold{};
  if (s.fmt == MOE_FMT_INT4_G128)
    return down_fmt<MOE_FMT_INT4_G128>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, shf, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16)
    return down_fmt<MOE_FMT_NVFP4_G16>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, shf, stream);
  return down_fmt<MOE_FMT_MXFP4_G32>(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, shf, stream);
}

}  // namespace moe
