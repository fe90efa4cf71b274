// The whole layer for a decode batch (T <= 8 tokens) in ONE persistent
// cooperative kernel: router logits, top-k with the renormalised softmax, the
// stable token->expert permutation, gate_up + SwiGLU, down and the
// routing-weighted combine.
//
// Why one kernel.  A decode step of this layer is bound by streaming the
// touched experts' packed weights from HBM ("primitive-ai/Nex-N2.5-mini-
// mixed-NVFP4-FP8", Measured: the bottleneck at concurrency 32 is weight
// bandwidth, and 4-bit moves half the bytes).  With separate kernels every
// dependent step (routing -> gate_up -> down) drains the weight stream and
// pays a launch.  Here each CTA (one per SM) keeps its own stream of packed
// weight tiles going from the moment the routing is known until its last down
// tile, and the steps that depend on other CTAs synchronise through device
// counters instead of kernel boundaries:
//
//  1. Router.  CTA c computes the logits of experts [c*Ec, (c+1)*Ec) for all
//     tokens (fp32 accumulation of bf16 x bf16) and stores them; a device-wide
//     counter then tells every CTA that all logits are written.
//  2. Routing metadata, redundantly in every CTA: top-k of each token (one
//     warp per token), the stable counting sort of the T*k (token, expert)
//     rows, the touched-expert list and, per (touched expert, token), the row
//     of that pair.  CTA 0 also stores them in the workspace.
//  3. Work items, in one global order: first every gate_up item (touched slot,
//     8 features: its 8 gate rows and 8 up rows), then every down item
//     (touched slot, 64 output features).  CTA c takes items c, c + G, ...
//     A producer warp copies each item's packed rows (codes + scales) into a
//     ring of shared-memory stages with 1-D bulk copies; sixteen compute
//     warps each own one 128-wide k-block of the item, dequantise it in
//     registers and run mma.sync m16n8k16 with the T <= 8 tokens as the 8 MMA
//     columns; an epilogue warp sums the sixteen partial tiles in warp order
//     and finishes the item.
//  4. gate_up epilogue: a = bf16(silu(gate) * up) for the tokens routed to
//     the expert, stored at the pair's sorted row; a per-expert device
//     counter counts the expert's finished gate_up items.  A down item of an
//     expert may start once that counter is complete: a poller warp watches
//     the counters of the CTA's down items in order and releases them to the
//     compute warps, so a CTA moves on to down items without waiting for the
//     other experts.  Gate_up items never wait on other CTAs, so this cannot
//     deadlock; the producer keeps filling the ring with down weights, which
//     depend on nothing.
//  5. down epilogue: y rows (unweighted, fp32) of the routed pairs; the CTA
//     that completes the last expert of a 64-feature range then forms
//     out[t] = bf16(sum_j w[t][j] * y[t][j]) over j in ascending order, so
//     the combine is deterministic.
//  6. The last CTA to finish resets the device counters for the next launch.
//
// Every wait is bounded (kWaitLimitNs): on expiry the CTA raises the timeout
// bit in the status word, the other CTAs see it and stop, and copies still in
// flight are drained before a CTA exits.  The workspace must then be
// re-initialised.
#include <algorithm>

#include "common.cuh"
#include "decode_common.cuh"
#include "internal.h"
#include "launch.h"
#include "topk_common.cuh"

#include <mutex>

namespace moe {

namespace {

constexpr int kFuWarps = 16;                 // compute warps: one 128-k block each
constexpr int kFuProducer = kFuWarps;        // warp index of the bulk-copy producer
constexpr int kFuEpilogue = kFuWarps + 1;    // warp index of the epilogue warp
constexpr int kFuSync = kFuWarps + 2;        // warp index of the publisher / dependency poller
constexpr int kFuThreads = (kFuWarps + 3) * 32;
constexpr int kFuCompute = kFuWarps * 32;    // compute threads
constexpr int kFuMaxT = 8;                   // tokens = MMA columns
constexpr int kFuMaxR = kFuMaxT * kMaxTopK;  // (token, expert) rows
constexpr int kFuGuRows = 16;                // gate_up item: 8 gate + 8 up rows
constexpr int kFuGuFeatures = 8;
constexpr int kFuDnRows = 64;                // down item: 64 output features = 4 M-tiles
constexpr int kFuGroups = 2;                 // compute groups, taking alternate items
constexpr int kFuGroupWarps = kFuWarps / kFuGroups;
constexpr int kFuGuBlocks = 2;               // gate_up k-blocks per warp (H <= 16 * 128)
constexpr int kFuDnKBlocks = 4;              // down k-blocks of 128 (I <= 512), one per warp
constexpr int kFuRedBufs = 2 * kFuGroups;    // partial-tile buffers (double-buffered per group)
constexpr int kFuMaxStages = 12;
constexpr int kFuRedFloats = kFuGroupWarps * 2 * 4 * 32;  // two partial tiles per warp of a group

// device counters, as uint32 indices into the workspace status block
constexpr int kCtrRoute = 8;    // CTAs whose logits are stored
constexpr int kCtrDone = 10;    // CTAs finished
constexpr int kCtrHr = 64;      // per 64-feature output range: down items finished (H <= 4096)
constexpr int kCtrSlot = 128;   // per touched slot: gate_up items finished (<= kFuMaxR slots)

struct FusedArgs {
  const uint16_t* x;       // [T][H]
  const uint16_t* wr;      // router weight [E][H]; null when the routing is given
  const float* bias;       // optional fp32 logit bias [E]
  const int32_t* ids_in;   // given routing [T][k] (ids, weights), or null
  const float* w_in;
  Bank gu, dn;
  int T, H, I, E, k;
  int stages;
  int stage_bytes;
  float* logits;           // [T][E]
  int32_t* topk_ids;       // [T][k]
  float* topk_w;           // [T][k]
  int32_t* offsets;        // [E+1]
  int32_t* sorted_rows;    // [T*k]
  int32_t* pos;            // [T*k]
  int32_t* touched;        // [1 + E]
  uint16_t* act;           // [T*k][I] bf16, sorted rows
  float* ypart;            // [T*k][H] fp32, sorted rows
  uint16_t* out;           // [T][H]
  uint32_t* status;        // status block: word 0 = status, counters at kCtr*
};

struct FusedSmem {
  int ids[kFuMaxR];
  float w[kFuMaxR];
  int pos[kFuMaxR];
  int rank[kFuMaxR];
  int sorted[kFuMaxR];
  int cnt[kMaxExperts];        // count per expert, then its first sorted position
  int slot[kMaxExperts];       // touched slot of each expert (-1: not touched)
  int touched[kFuMaxR];        // slot -> expert
  int16_t rmap[kFuMaxR][kFuMaxT];  // (slot, token) -> row t*k + j, or -1
  float lred[kFuWarps][kFuMaxT];
  int n_touched, n_valid;
  int abort;
  int ready;                   // down items of this CTA released by the sync warp
  int epi_done;                // items of this CTA whose epilogue stores are issued
  uint64_t full[kFuMaxStages], empty[kFuMaxStages];
  uint64_t red_full[kFuRedBufs], red_empty[kFuRedBufs];
};

// Stable counting sort of the R rows by expert with one warp (rows whose id
// lies outside [0, E) are dropped), the touched list (ascending expert id)
// and each expert's slot.
MOE_DEV void fused_route_meta(FusedSmem& m, int R, int E) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  for (int e = lane; e < E; e += 32) {
    m.cnt[e] = 0;
    m.slot[e] = -1;
  }
  __syncwarp();
  for (int r0 = 0; r0 < R; r0 += 32) {
    const int r = r0 + lane;
    int e = r < R ? m.ids[r] : -1;
    if (e >= E) e = -1;
    const unsigned mm = __match_any_sync(full, e);
    const int before = __popc(mm & ((1u << lane) - 1u));
    const int base = e >= 0 ? m.cnt[e] : 0;
    __syncwarp();
    if (e >= 0 && before == 0) m.cnt[e] = base + __popc(mm);
    if (r < R) m.rank[r] = e >= 0 ? base + before : -1;
    __syncwarp();
  }
  const int per = (E + 31) / 32;
  const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
  int csum = 0, nz = 0;
  for (int e = e0; e < e1; ++e) {
    csum += m.cnt[e];
    nz += m.cnt[e] > 0;
  }
  int c_incl = csum, nz_incl = nz;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(full, c_incl, o), b = __shfl_up_sync(full, nz_incl, o);
    if (lane >= o) {
      c_incl += a;
      nz_incl += b;
    }
  }
  int run = c_incl - csum, tpos = nz_incl - nz;
  for (int e = e0; e < e1; ++e) {
    const int c = m.cnt[e];
    m.cnt[e] = run;
    if (c > 0) {
      m.slot[e] = tpos;
      m.touched[tpos++] = e;
    }
    run += c;
  }
  if (lane == 31) {
    m.n_touched = nz_incl;
    m.n_valid = c_incl;
  }
  __syncwarp();
  for (int r = lane; r < R; r += 32) {
    const int e = m.ids[r];
    if (e < 0 || e >= E) {
      m.pos[r] = -1;
      continue;
    }
    const int p = m.cnt[e] + m.rank[r];
    m.sorted[p] = r;
    m.pos[r] = p;
  }
}

// bf16 pairs of a 16-byte chunk -> 8 floats
MOE_DEV void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Router logits of this CTA's experts for all tokens, by the compute warps:
// two experts at a time, one per half of the compute threads; a thread owns
// 8 consecutive k of its expert row and of every token.
MOE_DEV void fused_router(const FusedArgs& a, FusedSmem& m) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int kHalf = kFuCompute / 2;
  const int half = tid / kHalf, ht = tid % kHalf;
  const int G = gridDim.x;
  const int Ec = (a.E + G - 1) / G;
  const int eb = blockIdx.x * Ec, ee = min(a.E, eb + Ec);
  const int H = a.H, T = a.T;
  for (int e0 = eb; e0 < ee; e0 += 2) {
    const int e = e0 + half;
    float acc[kFuMaxT];
#pragma unroll
    for (int t = 0; t < kFuMaxT; ++t) acc[t] = 0.f;
    if (e < ee) {
      for (int kc = ht; kc < H / 8; kc += kHalf) {
        float w[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.wr + size_t(e) * H) + kc), w);
#pragma unroll
        for (int t = 0; t < kFuMaxT; ++t) {
          if (t < T) {
            float xv[8];
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + size_t(t) * H) + kc), xv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[t] = fmaf(w[i], xv[i], acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kFuMaxT; ++t) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) m.lred[warp][t] = v;
    }
    named_barrier_sync(1, kFuCompute);
    if (tid < 2 * kFuMaxT) {
      const int hh = tid / kFuMaxT, t = tid % kFuMaxT;
      if (e0 + hh < ee && t < T) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kFuWarps / 2; ++w) sum += m.lred[hh * (kFuWarps / 2) + w][t];
        a.logits[size_t(t) * a.E + e0 + hh] = sum;
      }
    }
    named_barrier_sync(1, kFuCompute);
  }
}

// Lane 0 waits until the poller has released more than `n` down items; the
// result is broadcast to the warp.  Bounded like every other wait.
MOE_DEV bool wait_released(FusedSmem& m, int n, volatile int* abort, uint32_t* gstatus) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    volatile int* ready = &m.ready;
    if (*ready <= n) {
      const uint64_t t0 = globaltimer_ns();
      while (*ready <= n) {
        if (*abort) { ok = 0; break; }
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          *abort = 1;
          atomicOr(gstatus, kStatusTimeout);
          ok = 0;
          break;
        }
        __nanosleep(20);
      }
    }
    __threadfence_block();
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Non-blocking: has the poller released more than `n` down items?
MOE_DEV bool is_released(FusedSmem& m, int n) {
  int r = 0;
  if ((threadIdx.x & 31) == 0) {
    r = *reinterpret_cast<volatile int*>(&m.ready) > n;
    __threadfence_block();
  }
  return __shfl_sync(0xffffffffu, r, 0) != 0;
}

template <int FMT>
__global__ void __launch_bounds__(kFuThreads, 1) decode_fused_kernel(const FusedArgs a) {
  extern __shared__ __align__(128) uint8_t dsmem[];
  __shared__ FusedSmem m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int G = gridDim.x;
  const int T = a.T, H = a.H, I = a.I, E = a.E, k = a.k;
  const int R = T * k;
  const int S = a.stages;
  uint32_t* const ctr = a.status;
  uint8_t* const ring = dsmem;
  float* const red = reinterpret_cast<float*>(dsmem + size_t(S) * a.stage_bytes);  // [kFuRedBufs][kFuRedFloats]
  volatile int* const abort_flag = &m.abort;

  pdl_wait();
  pdl_trigger();
  if (threadIdx.x == 0) {
    m.abort = 0;
    m.ready = 0;
    m.epi_done = 0;
    for (int st = 0; st < S; ++st) {
      mbar_init(&m.full[st], 1);
      mbar_init(&m.empty[st], kFuGroupWarps);  // one arrival per warp of the item's group
    }
    for (int b = 0; b < kFuRedBufs; ++b) {
      mbar_init(&m.red_full[b], kFuGroupWarps);
      mbar_init(&m.red_empty[b], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ 1. router
  const bool routed = a.ids_in != nullptr;
  if (!routed) {
    if (warp < kFuWarps) {
      fused_router(a, m);
      __threadfence();
      named_barrier_sync(1, kFuCompute);
      if (threadIdx.x == 0) {
        atomicAdd(&ctr[kCtrRoute], 1u);
        spin_until_geq(&ctr[kCtrRoute], uint32_t(G), abort_flag, a.status);
      }
    }
    __syncthreads();
    if (m.abort) return;
  }
  // gate_up activation fragments of the warp's k-block: token g of the lane
  // (read-only input: loaded once, held in registers)
  uint32_t xb[kFuGuBlocks][8][2];
  if (warp < kFuWarps) {
#pragma unroll
    for (int x = 0; x < kFuGuBlocks; ++x)
      load_act_frags(a.x + size_t(g < T ? g : 0) * H, H, 128 * (kFuGuBlocks * (warp % kFuGroupWarps) + x), q, g < T,
                     xb[x]);
  }
  // ------------------------------------------------------------ 2. routing metadata
  if (!routed) {
    for (int t = warp; t < T; t += kFuThreads / 32)
      warp_topk(a.logits + size_t(t) * E, a.bias, E, k, m.ids + t * k, m.w + t * k);
  } else {
    for (int r = threadIdx.x; r < R; r += kFuThreads) {
      m.ids[r] = a.ids_in[r];
      m.w[r] = a.w_in[r];
    }
  }
  __syncthreads();
  if (warp == 0) fused_route_meta(m, R, E);
  __syncthreads();
  const int n_touched = m.n_touched;
  for (int i = threadIdx.x; i < n_touched * kFuMaxT; i += kFuThreads) m.rmap[i / kFuMaxT][i % kFuMaxT] = -1;
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += kFuThreads)
    if (m.pos[r] >= 0) m.rmap[m.slot[m.ids[r]]][r / k] = int16_t(r);
  if (blockIdx.x == 0) {
    // the routing, for the caller's debug outputs and the workspace
    for (int r = threadIdx.x; r < R; r += kFuThreads) {
      if (!routed) {
        a.topk_ids[r] = m.ids[r];
        a.topk_w[r] = m.w[r];
      }
      a.pos[r] = m.pos[r];
      if (r < m.n_valid) a.sorted_rows[r] = m.sorted[r];
    }
    for (int e = threadIdx.x; e < E; e += kFuThreads) a.offsets[e] = m.cnt[e];
    for (int s = threadIdx.x; s < n_touched; s += kFuThreads) a.touched[1 + s] = m.touched[s];
    if (threadIdx.x == 0) {
      a.offsets[E] = m.n_valid;
      a.touched[0] = n_touched;
    }
  }
  __syncthreads();

  const int ftiles = I / kFuGuFeatures;
  const int hr_n = H / kFuDnRows;
  const int n_gu = n_touched * ftiles;
  const int n_items = n_gu + n_touched * hr_n;
  // this CTA's first down item and its position in the CTA's item sequence
  const int j_down = int(blockIdx.x) >= n_gu ? 0 : (n_gu - int(blockIdx.x) + G - 1) / G;
  const int i_down = int(blockIdx.x) + j_down * G;
  if (n_touched == 0) {
    // no row has a valid expert: the layer output is zero
    for (size_t idx = size_t(blockIdx.x) * kFuThreads + threadIdx.x; idx < size_t(T) * H;
         idx += size_t(G) * kFuThreads)
      a.out[idx] = 0;
  }
  const UnitLayout Lg = unit_layout(FMT, H, kFuGuRows, 1);
  const UnitLayout Ld = unit_layout(FMT, I, kFuDnRows, 1);

  if (warp == kFuProducer) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const int sbh = scale_row_bytes(FMT, H);
      int j = 0;
      for (int i = blockIdx.x; i < n_items; i += G, ++j) {
        const int st = j % S;
        if (!mbar_wait(&m.empty[st], ((j / S) & 1) ^ 1, abort_flag, a.status)) break;
        fence_proxy_async_smem();  // the consumers' reads of this stage before the refill
        uint8_t* stg = ring + size_t(st) * a.stage_bytes;
        if (i < n_gu) {
          const int e = m.touched[i / ftiles];
          const long row_g = long(e) * (2 * I) + (i % ftiles) * kFuGuFeatures;
          mbar_arrive_expect_tx(&m.full[st], staged_bytes<FMT>(a.gu, kFuGuRows));
          stage_rows<FMT>(a.gu, row_g, kFuGuFeatures, stg, stg + Lg.cbytes, &m.full[st]);
          stage_rows<FMT>(a.gu, row_g + I, kFuGuFeatures, stg + kFuGuFeatures * (H / 2),
                          stg + Lg.cbytes + kFuGuFeatures * sbh, &m.full[st]);
        } else {
          const int d = i - n_gu;
          const int e = m.touched[d / hr_n];
          mbar_arrive_expect_tx(&m.full[st], staged_bytes<FMT>(a.dn, kFuDnRows));
          stage_rows<FMT>(a.dn, long(e) * H + (d % hr_n) * kFuDnRows, kFuDnRows, stg, stg + Ld.cbytes,
                          &m.full[st]);
        }
      }
      if (m.abort) {
        // let the copies still in flight land before the CTA exits
        for (int jj = max(0, j - S); jj < j; ++jj) mbar_wait_drain(&m.full[jj % S], (jj / S) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == kFuSync) {
    // ---------------------------------------------------------- sync warp
    // (a) publishes the items whose epilogue stores are issued: one device
    //     fence covers all of them, then a counter per item (the expert's
    //     gate_up count, or the output range's down count, whose last arrival
    //     runs the combine of that range);
    // (b) releases this CTA's down items, in order, once their expert's
    //     gate_up items (on any CTA) are all published.
    // It never blocks on one of the two while the other could progress, so
    // publishing cannot wait on another CTA.
    const int my_items = int(blockIdx.x) < n_items ? (n_items - int(blockIdx.x) + G - 1) / G : 0;
    const int my_down = i_down < n_items ? (n_items - i_down + G - 1) / G : 0;
    int pub = 0, rel = 0;
    uint64_t t_last = globaltimer_ns();
    while (pub < my_items || rel < my_down) {
      bool progress = false;
      int done = 0;
      if (lane == 0) {
        done = *reinterpret_cast<volatile int*>(&m.epi_done);
        __threadfence_block();
      }
      __syncwarp();
      done = __shfl_sync(0xffffffffu, done, 0);
      if (done > pub) {
        __threadfence();  // the epilogue's stores of items [pub, done) before the counters
        while (pub < done) {
          const int nb = min(done - pub, 32);
          const int i = int(blockIdx.x) + (pub + lane) * G;
          int last = 0;
          if (lane < nb) {
            if (i < n_gu) red_add_u32(&ctr[kCtrSlot + i / ftiles], 1u);
            else last = atomicAdd(&ctr[kCtrHr + (i - n_gu) % hr_n], 1u) == uint32_t(n_touched - 1);
          }
          unsigned lm = __ballot_sync(0xffffffffu, last);
          while (lm) {
            // every expert's y rows of this 64-feature range are stored: combine.
            // Lane: 4 consecutive features (16 lanes span the range), tokens of
            // one parity; a token's k loads are in flight at once.
            const int l = __ffs(lm) - 1;
            lm &= lm - 1;
            const int h0 = ((int(blockIdx.x) + (pub + l) * G - n_gu) % hr_n) * kFuDnRows;
            __threadfence();
            const int hq = h0 + 4 * (lane & 15);
            for (int t = lane >> 4; t < T; t += 2) {
              float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int j0 = 0; j0 < k; j0 += 8) {
                float4 v[8];
                float wv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const int jj = j0 + u;
                  const int p = jj < k ? m.pos[t * k + jj] : -1;
                  wv[u] = p >= 0 ? m.w[t * k + jj] : 0.f;
                  v[u] = p >= 0 ? __ldcg(reinterpret_cast<const float4*>(a.ypart + size_t(p) * H + hq))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  acc.x = fmaf(wv[u], v[u].x, acc.x);
                  acc.y = fmaf(wv[u], v[u].y, acc.y);
                  acc.z = fmaf(wv[u], v[u].z, acc.z);
                  acc.w = fmaf(wv[u], v[u].w, acc.w);
                }
              }
              uint2 o2;
              o2.x = pack_bf16x2(acc.x, acc.y);
              o2.y = pack_bf16x2(acc.z, acc.w);
              *reinterpret_cast<uint2*>(a.out + size_t(t) * H + hq) = o2;
            }
          }
          pub += nb;
        }
        progress = true;
      }
      if (rel < my_down) {
        const int slot = (i_down + rel * G - n_gu) / hr_n;
        int ok = 0;
        if (lane == 0 && ld_acquire_gpu(&ctr[kCtrSlot + slot]) >= uint32_t(ftiles)) {
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&m.ready) = rel + 1;
          ok = 1;
        }
        if (__shfl_sync(0xffffffffu, ok, 0)) {
          ++rel;
          progress = true;
        }
      }
      const uint64_t now = globaltimer_ns();
      if (progress) {
        t_last = now;
      } else {
        int stop = 0;
        if (lane == 0) {
          if (*abort_flag || (ld_relaxed_gpu(a.status) & kStatusTimeout)) {
            *abort_flag = 1;
            stop = 1;
          } else if (now - t_last > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(a.status, kStatusTimeout);
            stop = 1;
          }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) break;
        __nanosleep(32);
      }
    }
  } else if (warp == kFuEpilogue) {
    // ---------------------------------------------------------- epilogue
    int j = 0;
    for (int i = blockIdx.x; i < n_items; i += G, ++j) {
      const int rb = j % kFuRedBufs;
      if (!mbar_wait(&m.red_full[rb], (j / kFuRedBufs) & 1, abort_flag, a.status)) break;
      const float* rbuf = red + rb * kFuRedFloats;
      if (i < n_gu) {
        float s[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          s[c] = 0.f;
#pragma unroll
          for (int w = 0; w < kFuGroupWarps; ++w) s[c] += rbuf[(w * 8 + c) * 32 + lane];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&m.red_empty[rb]);
        // c0, c1: gate of feature f at tokens 2q, 2q+1; c2, c3: up of the same
        const int slot = i / ftiles, f = (i % ftiles) * kFuGuFeatures + g;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = 2 * q + h;
          const int r = t < T ? m.rmap[slot][t] : -1;
          if (r >= 0) a.act[size_t(m.pos[r]) * I + f] = f32_to_bf16_rn(silu_mul(s[h], s[2 + h]));
        }
      } else {
        const int d = i - n_gu, slot = d / hr_n, hr = d % hr_n, h0 = hr * kFuDnRows;
        // group warp w: k-block w & 3, M-tiles (w >> 2) and (w >> 2) + 2 as
        // partial tiles 0 and 1: sum the k-blocks of each M-tile in order
        float y[4][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float v = 0.f;
#pragma unroll
            for (int kb = 0; kb < kFuDnKBlocks; ++kb)
              v += rbuf[(((kb + 4 * (mt & 1)) * 2 + (mt >> 1)) * 4 + c) * 32 + lane];
            y[mt][c] = v;
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(&m.red_empty[rb]);
        // c0, c1: feature 16mt+g at tokens 2q, 2q+1; c2, c3: feature 16mt+g+8
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int t = 2 * q + h;
          const int r = t < T ? m.rmap[slot][t] : -1;
          if (r >= 0) {
            float* yrow = a.ypart + size_t(m.pos[r]) * H + h0 + g;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
              yrow[16 * mt] = y[mt][h];
              yrow[16 * mt + 8] = y[mt][2 + h];
            }
          }
        }
      }
      // hand the item to the sync warp (CTA-scope release of the stores above)
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&m.epi_done) = j + 1;
      }
    }
  } else {
    // ---------------------------------------------------------- compute warps
    // Two groups of eight warps take alternate items of the CTA's sequence,
    // so the groups run out of phase and their waits and pipe bursts overlap.
    // Gate_up item: warp wg owns k-blocks 2wg, 2wg+1 of the 16-row tile.
    // Down item: warp wg owns k-block wg & 3 of M-tiles (wg >> 2) and
    // (wg >> 2) + 2 (rows 16mt .. 16mt+15), which share its activations.
    // The codes and scales of the group's NEXT item are loaded into
    // registers at the top of each iteration and the stage is released right
    // away, so the shared-memory load latency overlaps this item's work.
    const int grp = warp / kFuGroupWarps, wg = warp % kFuGroupWarps;
    const int nblk_h = (H + 127) / 128, nblk_i = (I + 127) / 128;
    const int kbd = wg & 3, mt0 = wg >> 2;
    auto fetch = [&](int item, int jt, RowChunk (&c)[4]) -> bool {
      const int st = jt % S;
      if (!mbar_wait(&m.full[st], (jt / S) & 1, abort_flag, a.status)) return false;
      const uint8_t* s_c = ring + size_t(st) * a.stage_bytes;
      if (item < n_gu) {
#pragma unroll
        for (int x = 0; x < kFuGuBlocks; ++x) {
          const int b = kFuGuBlocks * wg + x;
          if (b < nblk_h) {
            c[2 * x] = smem_row_chunk<FMT>(s_c, s_c + Lg.cbytes, g, H, 128 * b, q);
            c[2 * x + 1] = smem_row_chunk<FMT>(s_c, s_c + Lg.cbytes, g + 8, H, 128 * b, q);
          }
        }
      } else if (kbd < nblk_i) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int mt = mt0 + 2 * x;
          c[2 * x] = smem_row_chunk<FMT>(s_c, s_c + Ld.cbytes, 16 * mt + g, I, 128 * kbd, q);
          c[2 * x + 1] = smem_row_chunk<FMT>(s_c, s_c + Ld.cbytes, 16 * mt + g + 8, I, 128 * kbd, q);
        }
      }
      // the stage's contents are in registers: hand it back to the producer
      // (__syncwarp orders every lane's reads before lane 0's releasing arrival)
      __syncwarp();
      if (lane == 0) mbar_arrive(&m.empty[st]);
      return true;
    };
    // partial tiles of item jt to its reduction buffer, then tell the epilogue
    auto publish = [&](int jt, const float (&acc)[2][4]) {
      float* rw = red + (jt % kFuRedBufs) * kFuRedFloats + wg * 256;
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
        for (int c = 0; c < 4; ++c) rw[(t2 * 4 + c) * 32 + lane] = acc[t2][c];
      __syncwarp();
      if (lane == 0) mbar_arrive(&m.red_full[jt % kFuRedBufs]);
    };
    auto wait_red = [&](int jt) {
      return mbar_wait(&m.red_empty[jt % kFuRedBufs], ((jt / kFuRedBufs) & 1) ^ 1, abort_flag, a.status);
    };
    bool ok = true;
    RowChunk cur[4] = {};
    // the group's items: CTA-local indices j = grp, grp + 2, ...
    int i = int(blockIdx.x) + grp * G, j = grp;
    if (i < n_items) ok = fetch(i, j, cur);
    constexpr int kStep = kFuGroups;
    for (; ok && i < n_gu; i += kStep * G, j += kStep) {
      RowChunk nxt[4] = {};
      if (i + kStep * G < n_items && !(ok = fetch(i + kStep * G, j + kStep, nxt))) break;
      if (!(ok = wait_red(j))) break;
      float acc[2][4] = {};
#pragma unroll
      for (int x = 0; x < kFuGuBlocks; ++x)
        if (kFuGuBlocks * wg + x < nblk_h) mma_block<FMT>(acc[x], cur[2 * x], cur[2 * x + 1], xb[x]);
      // one tile: gate/up rows of 8 features; the two k-blocks summed in order
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[0][c] += acc[1][c];
        acc[1][c] = 0.f;
      }
      publish(j, acc);
#pragma unroll
      for (int x = 0; x < 4; ++x) cur[x] = nxt[x];
    }
    // down items (i is the group's first down item unless a wait gave up);
    // jj counts the CTA's down items, releases are in that order
    uint32_t raw[16];
    auto load_raw = [&](int item) {
      const int slot = (item - n_gu) / hr_n;
      const int r = g < T ? m.rmap[slot][g] : -1;
      load_act_raw_cg(a.act + size_t(r >= 0 ? m.pos[r] : 0) * I, I, 128 * kbd, q, r >= 0, raw);
    };
    bool have = false;  // raw holds the activations of item i
    for (; ok && i < n_items; i += kStep * G, j += kStep) {
      const int jj = j - j_down;
      if (!have) {
        if (!(ok = wait_released(m, jj, abort_flag, a.status))) break;
        load_raw(i);
      }
      uint32_t bfr[8][2];
      act_frags_from_raw(raw, bfr);
      RowChunk nxt[4] = {};
      if (i + kStep * G < n_items && !(ok = fetch(i + kStep * G, j + kStep, nxt))) break;
      // the next item's activations, in flight during this one if already released
      have = i + kStep * G < n_items && is_released(m, jj + kStep);
      if (have) load_raw(i + kStep * G);
      if (!(ok = wait_red(j))) break;
      float acc[2][4] = {};
      if (kbd < nblk_i) {
        mma_block<FMT>(acc[0], cur[0], cur[1], bfr);
        mma_block<FMT>(acc[1], cur[2], cur[3], bfr);
      }
      publish(j, acc);
#pragma unroll
      for (int x = 0; x < 4; ++x) cur[x] = nxt[x];
    }
  }

  // ------------------------------------------------------------ 6. reset
  __syncthreads();
  if (threadIdx.x == 0 && !m.abort) {
    __threadfence();
    if (atomicAdd(&ctr[kCtrDone], 1u) == uint32_t(G - 1)) {
      // every CTA is past every wait of this launch
      ctr[kCtrRoute] = 0;
      for (int h = 0; h < hr_n; ++h) ctr[kCtrHr + h] = 0;
      for (int s = 0; s < n_touched; ++s) ctr[kCtrSlot + s] = 0;
      ctr[kCtrDone] = 0;
    }
  }
}

size_t fused_stage_bytes(int fmt, int H, int I) {
  const auto layout = [&](int K, int rows) {
    const size_t cb = size_t(rows) * (K / 2);
    const size_t sb = size_t(rows) * (fmt == MOE_FMT_INT4_G128 ? int4_groups(K) * 2 : K / 32);
    return cb + ((sb + 15) & ~size_t(15));
  };
  return align_up(std::max(layout(H, kFuGuRows), layout(I, kFuDnRows)), 128);
}

struct FusedPlan {
  int grid = 0, stages = 0;
  size_t smem = 0;
};

template <int FMT>
cudaError_t fused_launch(const FusedArgs& args, cudaStream_t stream) {
  auto kern = decode_fused_kernel<FMT>;
  static FusedPlan plan;
  static int plan_stage_bytes = -1;
  static int plan_dev = -1;
  static std::mutex mu;  // host threads may launch concurrently
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::unique_lock<std::mutex> lock(mu);
  if (plan_stage_bytes != args.stage_bytes || plan_dev != dev) {
    int sms = 0, max_optin = 0;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return err;
    cudaFuncAttributes fa;
    if ((err = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return err;
    const size_t red_bytes = size_t(kFuRedBufs) * kFuRedFloats * sizeof(float);
    const size_t avail = size_t(max_optin) - fa.sharedSizeBytes - red_bytes;
    int stages = int(std::min<size_t>(kFuMaxStages, avail / size_t(args.stage_bytes)));
    if (stages < 2) return cudaErrorInvalidConfiguration;
    FusedPlan p;
    p.stages = stages;
    p.smem = size_t(stages) * args.stage_bytes + red_bytes;
    if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(p.smem))) != cudaSuccess)
      return err;
    int per_sm = 0;
    if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFuThreads, p.smem)) != cudaSuccess)
      return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    p.grid = per_sm * sms;
    plan = p;
    plan_stage_bytes = args.stage_bytes;
    plan_dev = dev;
  }
  const FusedPlan use = plan;
  lock.unlock();
  FusedArgs a = args;
  a.stages = use.stages;
  return launch_cooperative(kern, dim3(use.grid), dim3(kFuThreads), use.smem, stream, a);
}

}  // namespace

bool decode_fused_supported(const moe_shape_t& s, int T) {
  // gate_up: two 128-k blocks per warp of a group (H <= 2048); down: one (I <= 512);
  // INT4 and MXFP4 banks (NVFP4 runs on the three-kernel decode path)
  return s.fmt != MOE_FMT_NVFP4_G16 && T >= 1 && T <= kFuMaxT && s.hidden <= 128 * kFuGuBlocks * kFuGroupWarps && s.inter <= 128 * kFuDnKBlocks &&
         s.hidden % kFuDnRows == 0 && s.inter % kFuGuFeatures == 0 && kCtrHr + s.hidden / kFuDnRows <= kCtrSlot &&
         kCtrSlot + kFuMaxR <= int(kStatusBytes / 4) && s.num_experts <= kMaxExperts && s.top_k <= kMaxTopK;
}

size_t decode_fused_ypart_bytes(const moe_shape_t& s, int T) {
  return T <= kFuMaxT ? size_t(T) * s.top_k * s.hidden * sizeof(float) : 0;
}

cudaError_t launch_decode_fused(const moe_shape_t& s, int T, const uint16_t* x, const uint16_t* router_w,
                                const float* bias, const int32_t* ids_in, const float* w_in, const Bank& gu,
                                const Bank& dn, const Workspace& ws, uint16_t* out, cudaStream_t stream) {
  FusedArgs a{};
  a.x = x;
  a.wr = router_w;
  a.bias = bias;
  a.ids_in = ids_in;
  a.w_in = w_in;
  a.gu = gu;
  a.dn = dn;
  a.T = T;
  a.H = s.hidden;
  a.I = s.inter;
  a.E = s.num_experts;
  a.k = s.top_k;
  a.stage_bytes = int(fused_stage_bytes(s.fmt, s.hidden, s.inter));
  a.logits = ws.logits;
  a.topk_ids = ws.topk_ids;
  a.topk_w = ws.topk_w;
  a.offsets = ws.offsets;
  a.sorted_rows = ws.sorted_rows;
  a.pos = ws.pos;
  a.touched = ws.touched;
  a.act = ws.act;
  a.ypart = ws.ypart;
  a.out = out;
  a.status = ws.status;
  if (s.fmt == MOE_FMT_INT4_G128) return fused_launch<MOE_FMT_INT4_G128>(a, stream);
  return fused_launch<MOE_FMT_MXFP4_G32>(a, stream);
}

}  // namespace moe
