// Decode path (small token counts): weight-streaming expert GEMVs.
//
// The time goes into streaming the touched experts' packed weights from HBM
// ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", Measured: at concurrency 32
// the bottleneck is weight bandwidth).  A CTA owns one work unit, (touched
// expert, a tile of output features): the unit's packed rows are one
// contiguous range of the canonical [E][N][K/2] layout, so a single thread
// starts 1-D bulk copies of the codes and scales into shared memory and every
// byte of the unit is in flight at once.  Warps then dequantise in registers
// (bf16(q*s) for INT4, e2m1*2^e for MXFP4) and feed mma.sync m16n8k16 with up
// to 8 tokens per tile.
// (The fragment k-permutation is described in decode_common.cuh.)
#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "decode_common.cuh"
#include "launch.h"

namespace moe {

namespace {

// ---------------------------------------------------------------------------
// gate_up + SwiGLU, persistent, warp-specialised.  Work unit u = (touched slot
// u / (I/8), features f0 = 8*(u % (I/8)) .. f0+7).  Its 16 weight rows are the
// 8 gate rows f0.. and the 8 matching up rows I+f0.., staged as one 16-row
// tile (gate rows 0-7, up rows 8-15), so the MMA's C fragment holds gate
// (c0, c1) and up (c2, c3) of the same feature and token: SwiGLU needs no
// shuffle.  A producer warp walks the CTA's units u = blockIdx.x + i*gridDim.x:
// it writes each unit's routing metadata (expert, first sorted row, row count,
// token of each row) into a header in shared memory and starts the bulk
// copies of its codes and scales, two stages ahead.  Eight compute warps split
// K, sum their partial tiles in shared memory and write a = bf16(silu(gate) *
// up) to act[p][f] for the expert's sorted rows p.
// ---------------------------------------------------------------------------
constexpr int kGuFeatures = kDecRows / 2;  // features per gate_up unit
constexpr int kGuWarps = 8;                // compute warps (split K)
constexpr int kGuThreads = (kGuWarps + 1) * 32;
constexpr int kGuStages = 2;
constexpr int kHdrTokens = 32;             // token rows carried in a unit header

struct UnitHeader {
  int e, p0, n_e, pad;
  int tok[kHdrTokens];  // token of sorted row p0 + i (i < min(n_e, 32))
};

// With X_SMEM (small T), the producer warp first stages the T token rows of x
// into shared memory (one bulk copy per row, padded row stride), and the
// compute warps read their activation fragments from there.
template <int FMT, int NT, bool X_SMEM>
__global__ void __launch_bounds__(kGuThreads, NT == 1 ? 4 : 1) decode_gate_up_kernel(
    const uint16_t* __restrict__ x, int T, Bank gu, int I, int top_k, const int32_t* __restrict__ touched,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows, uint16_t* __restrict__ act,
    uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = gu.K;
  // stage layout: [16 rows of codes: gate 0-7, up 8-15][16 rows of scales]
  const UnitLayout L = unit_layout(FMT, K, kDecRows, 1);
  UnitHeader* hdr = reinterpret_cast<UnitHeader*>(smem + kGuStages * L.stage_bytes);
  float* red = reinterpret_cast<float*>(hdr + kGuStages);  // [warp][tile][4][lane]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + kGuWarps * NT * 4 * 32);
  uint64_t* empty = full + kGuStages;
  uint64_t* x_bar = empty + kGuStages;
  uint8_t* x_s = reinterpret_cast<uint8_t*>(x_bar + 2);  // [T][staged_row_stride(K)]
  const int xstride = staged_row_stride(K);
  __shared__ int s_units;
  __shared__ volatile int s_abort;  // raised by the first wait that gives up

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ftiles = I / kGuFeatures;
  if (threadIdx.x == 0) {
    s_abort = 0;
    s_units = touched[0] * ftiles;
    for (int st = 0; st < kGuStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kGuWarps);
    }
    if (X_SMEM) mbar_init(x_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_units = s_units;
  if (int(blockIdx.x) >= n_units) return;

  if (warp == kGuWarps) {
    // ---------------------------------------------------------------- producer
    if (X_SMEM) {
      if (lane == 0) mbar_arrive_expect_tx(x_bar, uint32_t(T) * uint32_t(2 * K));
      __syncwarp();
      stage_act_rows(x_s, x, T, K, x_bar);
    }
    int i = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
      const int st = i % kGuStages;
      if (!mbar_wait(&empty[st], ((i / kGuStages) & 1) ^ 1, &s_abort, status)) break;
      const int e = touched[1 + u / ftiles];
      const int p0 = offsets[e], n_e = offsets[e + 1] - p0;
      UnitHeader& h = hdr[st];
      if (lane < n_e) h.tok[lane] = sorted_rows[p0 + lane] / top_k;
      if (lane == 0) {
        h.e = e;
        h.p0 = p0;
        h.n_e = n_e;
      }
      __syncwarp();
      if (lane == 0) {
        fence_proxy_async_smem();  // earlier generic-proxy reads of this stage before the refill
        const long row_g = long(e) * gu.N + (u % ftiles) * kGuFeatures;
        const int sb = scale_row_bytes(FMT, K);
        uint8_t* stage = smem + st * L.stage_bytes;
        mbar_arrive_expect_tx(&full[st], staged_bytes<FMT>(gu, kDecRows));
        stage_rows<FMT>(gu, row_g, kGuFeatures, stage, stage + L.cbytes, &full[st]);
        stage_rows<FMT>(gu, row_g + I, kGuFeatures, stage + kGuFeatures * (K / 2), stage + L.cbytes + kGuFeatures * sb,
                        &full[st]);
      }
      __syncwarp();
    }
    return;
  }

  // -------------------------------------------------------------------- compute
  const int g = lane >> 2, q = lane & 3;
  const int nblk = (K + 127) / 128;
  const bool x_ok = !X_SMEM || mbar_wait(x_bar, 0, &s_abort, status);
  const int srow = scale_row_bytes(FMT, K);
  const int nb_q = lane_kblocks(K, q);
  int i = 0;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++i) {
    const int st = i % kGuStages;
    const bool ok = mbar_wait(&full[st], (i / kGuStages) & 1, &s_abort, status) && x_ok;
    const uint8_t* s_c = smem + st * L.stage_bytes;
    const uint8_t* s_s = s_c + L.cbytes;
    const UnitHeader& h = hdr[st];
    const int p0 = h.p0, n_e = h.n_e;
    const float gsc = FMT == MOE_FMT_NVFP4_G16 ? gu.gscale[h.e] : 0.f;
    const int f0 = (u % ftiles) * kGuFeatures;
    const int ntiles = (n_e + 7) / 8;
    for (int nt0 = 0; nt0 < ntiles; nt0 += NT) {
      float acc[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
      int xtok[NT];
      bool xval[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        const int c = (nt0 + j) * 8 + g;
        xval[j] = c < n_e;
        xtok[j] = !xval[j] ? 0 : (c < kHdrTokens ? h.tok[c] : sorted_rows[p0 + c] / top_k);
      }
      if (ok) {
        // the lane's rows g (gate) and g + 8 (up) at its k-slice, and their scales
        const uint8_t* c_gate = s_c + g * (K / 2) + 16 * q;
        const uint8_t* c_up = c_gate + 8 * (K / 2);
        const uint8_t* sc_gate = s_s + g * srow;
        const uint8_t* sc_up = sc_gate + 8 * srow;
        for (int b = warp; b < nblk; b += kGuWarps) {
          const bool in = b < nb_q;
          const RowChunk gate = row_chunk_at<FMT>(c_gate, sc_gate, b, q, in, gsc);
          const RowChunk up = row_chunk_at<FMT>(c_up, sc_up, b, q, in, gsc);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            if (nt0 + j >= ntiles) break;
            uint32_t bf[8][2];
            if (X_SMEM) load_act_frags_smem(x_s + xtok[j] * xstride + 256 * b + 64 * q, in && xval[j], bf);
            else load_act_frags(x + size_t(xtok[j]) * K, K, b * 128, q, xval[j], bf);
            mma_block<FMT>(acc[j], gate, up, bf);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) red[((warp * NT + j) * 4 + c) * 32 + lane] = acc[j][c];
      named_barrier_sync(1, kGuWarps * 32);
      // warp w < NT finishes token tile nt0 + w
      const int j = warp;
      if (ok && j < NT && nt0 + j < ntiles) {
        float sum[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sum[c] = 0.f;
#pragma unroll
          for (int w = 0; w < kGuWarps; ++w) sum[c] += red[((w * NT + j) * 4 + c) * 32 + lane];
        }
        // c0, c1: gate of feature f0+g at tokens 2q, 2q+1; c2, c3: up of the same
        const int f = f0 + g;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int col = (nt0 + j) * 8 + 2 * q + hh;
          if (col < n_e) act[size_t(p0 + col) * I + f] = f32_to_bf16_rn(silu_mul(sum[hh], sum[2 + hh]));
        }
      }
      named_barrier_sync(1, kGuWarps * 32);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
  }
}

// ---------------------------------------------------------------------------
// down projection + deterministic combine.  One CTA per 16-feature tile of
// the output; its 16 warps own the touched experts (warp w takes slots w,
// w+16, ...), each streaming its experts' 16 down rows (all of K = I) through
// its own two-stage ring of bulk copies.  A warp multiplies the expert's rows
// with the activations of the expert's tokens and adds w_tj * y into its own
// shared-memory accumulator [token][feature]; the 16 accumulators are then
// summed in warp order and written as bf16.  The summation order is fixed, so
// the output is deterministic.  Tokens are processed in chunks of 32 (one
// chunk for T <= 32).
// ---------------------------------------------------------------------------
constexpr int kDnWarps = 16;
constexpr int kDnStages = 2;
constexpr int kDnTokens = 32;  // token chunk per pass

// First sorted row in [p0, p1) whose token is >= t (rows ascend with the
// token index), found 32 rows at a time with a warp ballot.
MOE_DEV int chunk_bound(const int32_t* __restrict__ sorted_rows, int p0, int p1, int top_k, int t) {
  const int lane = threadIdx.x & 31;
  for (int p = p0; p < p1; p += 32) {
    const bool below = p + lane < p1 && sorted_rows[p + lane] / top_k < t;
    const unsigned m = __ballot_sync(0xffffffffu, below);
    if (m != 0xffffffffu) return p + __popc(m);
  }
  return p1;
}

template <int FMT>
MOE_DEV void issue_down_rows(const Bank& dn, int e, int f0, uint8_t* stage, const UnitLayout& L, uint64_t* bar) {
  mbar_arrive_expect_tx(bar, staged_bytes<FMT>(dn, kDecRows));
  stage_rows<FMT>(dn, long(e) * dn.N + f0, kDecRows, stage, stage + L.cbytes, bar);
}

// With ACT_SMEM (T <= kDnTokens and the rows fit), one warp first stages all
// T*k activation rows into shared memory with one bulk copy per row, so the
// fragment loads of the expert loop read shared memory instead of waiting on
// L2 once per k-block.
template <int FMT, int NT, bool ACT_SMEM>
__global__ void __launch_bounds__(kDnWarps * 32) decode_down_kernel(
    Bank dn, int T, int top_k, const int32_t* __restrict__ touched, const int32_t* __restrict__ offsets,
    const uint16_t* __restrict__ act, const float* __restrict__ topk_w, const int32_t* __restrict__ sorted_rows,
    uint16_t* __restrict__ out, const float* __restrict__ sh_gate, const float* __restrict__ sh_y, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int H = dn.N, K = dn.K;  // K = I
  const UnitLayout L = unit_layout(FMT, K, kDecRows, 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int tchunk = min(T, kDnTokens);  // tokens per pass
  const int srow = scale_row_bytes(FMT, K);
  const int nb_q = lane_kblocks(K, q);
  uint8_t* ring = smem + warp * kDnStages * L.stage_bytes;
  float* accs = reinterpret_cast<float*>(smem + kDnWarps * kDnStages * L.stage_bytes);  // [warp][token][16]
  float* acc_w = accs + warp * tchunk * kDecRows;
  uint64_t* all_bars = reinterpret_cast<uint64_t*>(accs + kDnWarps * tchunk * kDecRows);
  uint64_t* bars = all_bars + warp * kDnStages;
  uint64_t* act_bar = all_bars + kDnWarps * kDnStages;
  uint8_t* act_s = reinterpret_cast<uint8_t*>(act_bar + 2);  // [T*k][staged_row_stride(K)]
  const int astride = staged_row_stride(K);

  __shared__ volatile int s_abort;
  pdl_wait();
  pdl_trigger();
  const int f0 = blockIdx.x * kDecRows;
  const int n_touched = touched[0];
  const int nblk = (K + 127) / 128;
  if (threadIdx.x == 0) {
    s_abort = 0;
    if (ACT_SMEM) mbar_init(act_bar, 1);
  }
  if (lane == 0) {
    for (int st = 0; st < kDnStages; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (ACT_SMEM && warp == 0) {
    const int R = T * top_k;
    if (lane == 0) mbar_arrive_expect_tx(act_bar, uint32_t(R) * uint32_t(2 * K));
    __syncwarp();
    stage_act_rows(act_s, act, R, K, act_bar);
  }
  int uses = 0;  // ring slots consumed so far by this warp (over all chunks)
  for (int t0 = 0; t0 < T; t0 += kDnTokens) {
    const int t1 = min(T, t0 + kDnTokens);
    for (int i = lane; i < tchunk * kDecRows; i += 32) acc_w[i] = 0.f;
    // prologue: first experts of this warp into the ring
    if (lane == 0) {
      for (int st = 0; st < kDnStages; ++st) {
        const int slot = warp + st * kDnWarps;
        if (slot < n_touched) {
          fence_proxy_async_smem();
          issue_down_rows<FMT>(dn, touched[1 + slot], f0, ring + ((uses + st) % kDnStages) * L.stage_bytes, L,
                               &bars[(uses + st) % kDnStages]);
        }
      }
    }
    __syncwarp();
    // the staged activation rows (one chunk: T <= kDnTokens)
    const bool act_ok = !ACT_SMEM || n_touched <= warp || mbar_wait(act_bar, 0, &s_abort, status);
    for (int slot = warp, n = 0; slot < n_touched; slot += kDnWarps, ++n) {
      const int st = (uses + n) % kDnStages;
      const uint32_t parity = ((uses + n) / kDnStages) & 1;
      const uint8_t* s_c = ring + st * L.stage_bytes;
      const uint8_t* s_s = s_c + L.cbytes;
      const int e = touched[1 + slot];
      // rows of expert e whose token lies in [t0, t1): a contiguous sub-range
      // (sorted rows ascend with the token index); one chunk when T <= 32
      int p0 = offsets[e], pe = offsets[e + 1];
      if (T > kDnTokens) {
        pe = chunk_bound(sorted_rows, p0, pe, top_k, t1);
        p0 = chunk_bound(sorted_rows, p0, pe, top_k, t0);
      }
      const int n_e = pe - p0;
      const float gsc = FMT == MOE_FMT_NVFP4_G16 ? dn.gscale[e] : 0.f;
      const bool ok = mbar_wait(&bars[st], parity, &s_abort, status) && act_ok;
      const int ntiles = (n_e + 7) / 8;
      for (int nt0 = 0; ok && nt0 < ntiles; nt0 += NT) {
        // routing of the next 32 rows: lane l holds row nt0*8 + l
        const int rl = nt0 * 8 + lane;
        int my_tok = 0;
        float my_w = 0.f;
        if (rl < n_e) {
          const int r = sorted_rows[p0 + rl];
          my_tok = r / top_k - t0;
          my_w = topk_w[r];
        }
        float acc[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
        const uint8_t* c_lo = s_c + g * (K / 2) + 16 * q;
        const uint8_t* c_hi = c_lo + 8 * (K / 2);
        const uint8_t* sc_lo = s_s + g * srow;
        const uint8_t* sc_hi = sc_lo + 8 * srow;
        for (int b = 0; b < nblk; ++b) {
          const bool in = b < nb_q;
          const RowChunk c0 = row_chunk_at<FMT>(c_lo, sc_lo, b, q, in, gsc);
          const RowChunk c1 = row_chunk_at<FMT>(c_hi, sc_hi, b, q, in, gsc);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            if (nt0 + j >= ntiles) break;
            const int col = (nt0 + j) * 8 + g;
            const int prow = p0 + (col < n_e ? col : 0);
            uint32_t bf[8][2];
            if (ACT_SMEM) load_act_frags_smem(act_s + prow * astride + 256 * b + 64 * q, in && col < n_e, bf);
            else load_act_frags(act + size_t(prow) * K, K, b * 128, q, col < n_e, bf);
            mma_block<FMT>(acc[j], c0, c1, bf);
          }
        }
        // c0,c1: feature g, rows 2q, 2q+1 of the tile; c2,c3: feature g+8
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int lr = j * 8 + 2 * q + h;  // row within this group of 32
            const int t = __shfl_sync(0xffffffffu, my_tok, lr);
            const float w = __shfl_sync(0xffffffffu, my_w, lr);
            if (nt0 + j < ntiles && (nt0 + j) * 8 + 2 * q + h < n_e) {
              acc_w[t * kDecRows + g] += w * acc[j][h];
              acc_w[t * kDecRows + g + 8] += w * acc[j][2 + h];
            }
          }
        }
      }
      __syncwarp();  // ring slot st consumed by every lane
      if (lane == 0) {
        const int next = slot + kDnStages * kDnWarps;
        if (next < n_touched) {
          fence_proxy_async_smem();
          issue_down_rows<FMT>(dn, touched[1 + next], f0, ring + st * L.stage_bytes, L, &bars[st]);
        }
      }
      __syncwarp();
    }
    // every warp's ring slots used in this chunk
    uses += (n_touched > warp) ? (n_touched - warp + kDnWarps - 1) / kDnWarps : 0;
    __syncthreads();
    // sum the warps' accumulators in a fixed order
    for (int idx = threadIdx.x; idx < (t1 - t0) * kDecRows; idx += blockDim.x) {
      float sum = 0.f;
#pragma unroll 4
      for (int w = 0; w < kDnWarps; ++w) sum += accs[w * tchunk * kDecRows + idx];
      const int t = t0 + idx / kDecRows, f = f0 + idx % kDecRows;
      if (sh_y) sum += sh_gate[t] * sh_y[size_t(t) * H + f];  // the shared expert, before the one rounding
      out[size_t(t) * H + f] = f32_to_bf16_rn(sum);
    }
    __syncthreads();
  }
  if (ACT_SMEM && warp == 0 && n_touched <= 0) {
    // nothing waited on the staged rows: let the copies land before exiting
    mbar_wait_drain(act_bar, 0, kWaitLimitNs);
  }
}

int max_touched(int T, int k, int E) { return (long(T) * k < E) ? T * k : E; }

size_t unit_stage_bytes(int fmt, int K, int rows, int mats) {
  const int cbytes = rows * (K / 2);
  const int sbytes = rows * scale_row_bytes(fmt, K);
  return size_t(mats) * (cbytes + ((sbytes + 15) & ~15));
}

// stages + unit headers + the cross-warp reduction buffer + barriers + the
// token rows' barrier (16 bytes) and, with x_rows > 0, those rows
size_t gate_up_smem(int fmt, int K, int nt, int x_rows) {
  return kGuStages * unit_stage_bytes(fmt, K, kDecRows, 1) + kGuStages * sizeof(UnitHeader) +
         size_t(kGuWarps) * nt * 4 * 32 * 4 + 2 * kGuStages * 8 + 16 + size_t(x_rows) * staged_row_stride(K);
}

// Token rows staged in shared memory by the gate_up kernel up to this many
// bytes: 4 rows of hidden 2048 keep four CTAs resident per SM.
constexpr size_t kGuMaxStagedX = 4 * (2 * 2048 + 16);

// per-warp rings + per-warp accumulators + per-warp barriers + the staged
// activation rows' barrier (16 bytes) and, with act_rows > 0, those rows
size_t down_smem(int fmt, int K, int T, int act_rows) {
  const int tchunk = std::min(T, kDnTokens);
  return size_t(kDnWarps) * kDnStages * unit_stage_bytes(fmt, K, kDecRows, 1) +
         size_t(kDnWarps) * tchunk * kDecRows * 4 + size_t(kDnWarps) * kDnStages * 8 + 16 +
         size_t(act_rows) * staged_row_stride(K);
}

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
  static Entry cache[16] = {};
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

}  // namespace

namespace {

template <int FMT, int NT>
cudaError_t gate_up_nt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Workspace& ws,
                       int units, cudaStream_t stream) {
  const bool x_smem = size_t(T) * staged_row_stride(s.hidden) <= kGuMaxStagedX;
  auto k = x_smem ? decode_gate_up_kernel<FMT, NT, true> : decode_gate_up_kernel<FMT, NT, false>;
  const size_t smem = gate_up_smem(FMT, s.hidden, NT, x_smem ? T : 0);
  cudaError_t err = allow_smem(k, smem);
  if (err != cudaSuccess) return err;
  const int grid = persistent_grid(k, smem, units, kGuThreads);
  return launch_pdl(k, dim3(grid), dim3(kGuThreads), smem, stream, x, T, gu, s.inter, s.top_k,
                    (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const int32_t*)ws.sorted_rows, ws.act,
                    ws.status);
}

template <int FMT>
cudaError_t gate_up_fmt(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Workspace& ws,
                        int units, cudaStream_t stream) {
  // token tiles of 8 held in registers: enough for the largest possible expert batch (T)
  if (T <= 8) return gate_up_nt<FMT, 1>(s, T, x, gu, ws, units, stream);
  if (T <= 16) return gate_up_nt<FMT, 2>(s, T, x, gu, ws, units, stream);
  return gate_up_nt<FMT, kDecNT>(s, T, x, gu, ws, units, stream);
}

template <int FMT, int NT>
cudaError_t down_nt(const moe_shape_t& s, int T, const Bank& dn, const Workspace& ws, uint16_t* out,
                    const float* sh_gate, const float* sh_y, cudaStream_t stream) {
  // stage all T*k activation rows in shared memory when they fit
  const int R = T * s.top_k;
  const bool act_smem = T <= kDnTokens && down_smem(FMT, s.inter, T, R) <= kMaxSmemPerCta;
  auto k = act_smem ? decode_down_kernel<FMT, NT, true> : decode_down_kernel<FMT, NT, false>;
  const size_t smem = down_smem(FMT, s.inter, T, act_smem ? R : 0);
  cudaError_t err = allow_smem(k, smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(k, dim3(s.hidden / kDecRows), dim3(kDnWarps * 32), smem, stream, dn, T, s.top_k,
                    (const int32_t*)ws.touched, (const int32_t*)ws.offsets, (const uint16_t*)ws.act,
                    (const float*)ws.topk_w, (const int32_t*)ws.sorted_rows, out, sh_gate, sh_y, ws.status);
}

template <int FMT>
cudaError_t down_fmt(const moe_shape_t& s, int T, const Bank& dn, const Workspace& ws, uint16_t* out,
                     const float* sh_gate, const float* sh_y, cudaStream_t stream) {
  if (T <= 8) return down_nt<FMT, 1>(s, T, dn, ws, out, sh_gate, sh_y, stream);
  if (T <= 16) return down_nt<FMT, 2>(s, T, dn, ws, out, sh_gate, sh_y, stream);
  return down_nt<FMT, kDecNT>(s, T, dn, ws, out, sh_gate, sh_y, stream);
}

}  // namespace

cudaError_t launch_decode_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu,
                                  const Workspace& ws, cudaStream_t stream) {
  const int units = max_touched(T, s.top_k, s.num_experts) * (s.inter / kGuFeatures);
  if (units == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128) return gate_up_fmt<MOE_FMT_INT4_G128>(s, T, x, gu, ws, units, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return gate_up_fmt<MOE_FMT_NVFP4_G16>(s, T, x, gu, ws, units, stream);
  return gate_up_fmt<MOE_FMT_MXFP4_G32>(s, T, x, gu, ws, units, stream);
}

cudaError_t launch_decode_down_combine(const moe_shape_t& s, int T, const Bank& dn, const Workspace& ws,
                                       uint16_t* out, const float* sh_gate, const float* sh_y,
                                       cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128) return down_fmt<MOE_FMT_INT4_G128>(s, T, dn, ws, out, sh_gate, sh_y, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return down_fmt<MOE_FMT_NVFP4_G16>(s, T, dn, ws, out, sh_gate, sh_y, stream);
  return down_fmt<MOE_FMT_MXFP4_G32>(s, T, dn, ws, out, sh_gate, sh_y, stream);
}

}  // namespace moe
