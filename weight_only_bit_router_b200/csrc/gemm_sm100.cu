// Grouped GEMMs of the prefill path on the 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory).
//
// One persistent, warp-specialised kernel serves three products, all computed
// "weights x tokens^T" so that a 128-row weight tile is the MMA's M side and
// the tokens of one expert are its N side (N = the expert's token count
// rounded up to 16, at most 128 per tile):
//
//   ROUTER   logits[t][e]   = Wr[e, :] . x[t, :]                (bf16 A by TMA)
//   GATE_UP  act[p][f]      = bf16(silu(g_f . x_t) * (u_f . x_t)), two
//                             accumulators (gate rows f, up rows I+f)
//   DOWN     out_acc[t][f] += w_tj * (Wd[e, f, :] . act[p, :])
//
// The expert weights ("Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe: fused
// banks gate_up [E, 2I, H], down [E, H, I]) arrive as packed 4-bit codes by
// TMA, are dequantised to bf16 by a warpgroup straight into the 128-byte
// swizzled K-major layout the MMA reads (W4A16: 4-bit weights, bf16
// activations, "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Model summary),
// and the token rows of each expert are gathered by cp.async.
//
// Warp roles (512 threads):
//   warp 0       TMA producer: code tiles (or router weight tiles), and once
//                per tile a bulk copy of the tile's scale rows
//   warp 1       TMEM allocation + single-thread tcgen05.mma issue
//   warps 2-3    token-row gather (cp.async, 16 B per thread per copy)
//   warps 4-11   dequantisation, two threads per weight row (32 k each)
//   warps 12-15  epilogue, one TMEM lane (weight row) per thread; the down
//                product's weighted tile goes through shared memory and is
//                added into the fp32 output with one bulk reduction per token
// Every wait is bounded; an expired wait raises the workspace status word and
// the CTA unwinds, frees its tensor memory and exits.
#include <stdio.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "launch.h"

namespace moe {

namespace {

enum GemmMode { kRouter = 0, kGateUp = 1, kDown = 2 };

constexpr int BM = 128;        // weight rows per tile (MMA M)
constexpr int BN = kGemmBN;    // token columns per tile (max MMA N)
constexpr int BK = 64;         // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int SA_DEFAULT = 3;  // bf16 weight-operand stages (dequantised, or router weights by TMA)
constexpr int SB_DEFAULT = 4;  // gathered token-operand stages (copies signal their own arrival)
constexpr int SC = 3;          // code stages
constexpr int kThreads = 512;
constexpr int kDqThreads = 256;           // dequantisation threads (warps 4-11)
constexpr int kEpiWarp0 = 12;             // first epilogue warp
// scale bytes staged per weight row: K <= 2048 for INT4 and MXFP4; NVFP4 keeps
// one E4M3 byte per 16 k and, to make room, one bf16 operand stage less
constexpr int kMaxScaleRow = 64;
constexpr int kMaxScaleRowNv = 128;
constexpr int kMaxScaleRowInt4 = 32;  // INT4: K <= 2048
constexpr int kTileBytes = BM * BK * 2;   // 16 KB bf16 operand tile
constexpr int kCodeBytes = BM * BK / 2;   // 4 KB code tile

struct GemmArgs {
  int mode, fmt;
  int K;                // reduction length
  int M_total;          // rows of the weight side: E (router), I (gate_up), H (down)
  int n_ftiles;         // weight-row tiles of 128
  int T, top_k, I, H, E;
  int e_lo, e_hi;              // grouped modes: the bank holds experts [e_lo, e_hi)
  const uint16_t* bsrc;        // token operand: x [T, H] (router, gate_up) or act [T*k, I] (down)
  const int32_t* offsets;      // [E+1]
  const int32_t* sorted_rows;  // [T*k]
  const int32_t* tile_base;    // [E+1] token-block prefix
  const float* topk_w;         // [T*k]
  const void* scales;          // scale plane of the packed bank
  const float* gscale;         // NVFP4: per-expert global scales (null otherwise)
  int scale_row_stride;        // scale elements per weight row
  float* logits;
  uint16_t* act;
  float* out_acc;
  float* ypart;                // down: per-row outputs [T*k][H] instead of out_acc (deterministic combine)
  uint32_t* status;
};

template <int MODE, int FMT>
struct Cfg {
  static constexpr bool NV_WIDE = FMT == MOE_FMT_NVFP4_G16 && MODE == kGateUp;
  // Four weight-operand stages where shared memory allows (INT4 gate_up,
  // down), one token stage less: the dequantisation of a stage waits for the
  // tensor core to release the stage SA back, so SA covers the MMAs' latency.
  static constexpr bool DEEP = MODE == kDown || (MODE == kGateUp && FMT == MOE_FMT_INT4_G128);
  static constexpr int SA = NV_WIDE ? SA_DEFAULT - 1 : DEEP ? SA_DEFAULT + 1 : SA_DEFAULT;
  static constexpr int SB = DEEP ? SB_DEFAULT - 1 : SB_DEFAULT;
  static constexpr int SROW = FMT == MOE_FMT_NVFP4_G16 ? kMaxScaleRowNv
                              : FMT == MOE_FMT_INT4_G128 ? kMaxScaleRowInt4 : kMaxScaleRow;
  static constexpr int NACC = MODE == kGateUp ? 2 : 1;                 // accumulators per tile
  static constexpr uint32_t TMEM_COLS = MODE == kGateUp ? 512 : 256;   // 2 buffers x NACC x BN
  static constexpr int SMEM_A = SA * NACC * kTileBytes;
  static constexpr int SMEM_B = SB * kTileBytes;
  static constexpr int SMEM_C = SC * NACC * kCodeBytes;
  static constexpr int SMEM_S = MODE == kRouter ? 0 : 2 * NACC * BM * SROW;  // two tiles of scale rows
  static constexpr int SMEM_D = MODE == kDown ? BN * BM * 4 : 0;                     // down: [token][row] fp32
  static constexpr int SMEM = SMEM_A + SMEM_B + SMEM_C + SMEM_S + SMEM_D + 1024 /*barriers*/ + 1024 /*align*/ +
                             (kMaxExperts + 1) * 4;
  static_assert(SMEM <= 232448, "shared memory of one CTA");
};

struct Tile {
  int e;        // expert (grouped modes)
  int eb;       // its index in the bank (e - e_lo)
  int fb;       // weight-row tile
  int p_begin;  // first sorted row (grouped) or first token (router)
  int n;        // valid token columns (1..BN)
};

MOE_DEV Tile decode_tile(const GemmArgs& a, int tile, const int* s_tile_base) {
  Tile t;
  t.fb = tile % a.n_ftiles;
  const int blk = tile / a.n_ftiles;
  if (a.mode == kRouter) {
    t.e = 0;
    t.eb = 0;
    t.p_begin = blk * BN;
    t.n = min(BN, a.T - t.p_begin);
    return t;
  }
  // expert e with tile_base[e] <= blk' < tile_base[e+1] (skip empty experts),
  // blk' counted from the bank's first expert
  const int gblk = blk + s_tile_base[a.e_lo];
  int lo = a.e_lo, hi = a.e_hi;  // invariant: tile_base[lo] <= gblk < tile_base[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_tile_base[mid] <= gblk) lo = mid; else hi = mid;
  }
  t.e = lo;
  t.eb = lo - a.e_lo;
  const int tb = gblk - s_tile_base[lo];
  const int p0 = a.offsets[lo];
  const int n_e = a.offsets[lo + 1] - p0;
  t.p_begin = p0 + tb * BN;
  t.n = min(BN, n_e - tb * BN);
  return t;
}

MOE_DEV int num_tiles(const GemmArgs& a, const int* s_tile_base) {
  if (a.mode == kRouter) return a.n_ftiles * ((a.T + BN - 1) / BN);
  return (s_tile_base[a.e_hi] - s_tile_base[a.e_lo]) * a.n_ftiles;
}

// byte offset of 16-byte chunk c of row r inside a 128B-swizzled K-major tile
MOE_DEV uint32_t sw128_offset(int r, int c) {
  return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

MOE_DEV void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Prefetch the box at (x, y, z) of a 3-D tensor map into L2.
MOE_DEV void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z)
               : "memory");
}

// Sleep between tries of the waits off the critical path: the producers
// (code tiles, scale rows, token rows) run ahead of the dequantisation warps,
// and the epilogue waits for a whole tile's main loop.
constexpr uint32_t kProducerSleepNs = 64;
constexpr uint32_t kEpilogueSleepNs = 256;
// The MMA issuer waits on the dequantisation warps most of the time; a short
// sleep between its tries keeps its polls from taking their issue slots.
constexpr uint32_t kMmaSleepNs = 32;
// The dequantisation warps' waits (code tiles landed, weight stage free):
// a build-time tuning knob, 0 = plain tries with the suspend hint.
#ifndef MOE_GEMM_DQ_SLEEP_NS
#define MOE_GEMM_DQ_SLEEP_NS 0
#endif
MOE_DEV bool dq_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* gstatus) {
  return MOE_GEMM_DQ_SLEEP_NS > 0 ? mbar_wait_backoff(bar, parity, abort, gstatus, MOE_GEMM_DQ_SLEEP_NS)
                                  : mbar_wait(bar, parity, abort, gstatus);
}

// Code tiles this many k-stages ahead of the producer are prefetched into L2.
constexpr int kCodePrefetch = 8;

// bf16x2 with both halves = 2^e (e in [-127, 127]).
MOE_DEV uint32_t pow2x2(int e) {
  const uint32_t b = e >= -126 ? uint32_t(e + 127) << 7 : 0x0040u;
  return b | (b << 16);
}

// Dequantise 32 codes (one 16-byte chunk, k = 32*half .. +31 of the stage) of
// one row and store them as four 16-byte bf16 chunks in swizzled layout.
// Code words 0-1 use `mult`, words 2-3 `mult2` (the two 16-element NVFP4
// blocks of the chunk; equal for the other formats).
//
// INT4 with a scale s in [2^-126, 2^-5): byte c of a code word holds the
// adjacent elements 2c (low nibble u0) and 2c + 1 (high nibble u1).  The byte
// copied into both halves of a word and masked with 0x00F0000F gives the bf16
// values u0 * 2^-133 (low half) and u1 * 2^-129 (high half): bit patterns
// below 256 are linear in value.  One bf16 fused multiply-add with the
// multipliers (s * 2^133, s * 2^129) and -8 s in both halves yields
// (bf16((u0 - 8) s), bf16((u1 - 8) s)), exact before its single rounding, in
// the order the swizzled K-major tile wants.  Other scales take the two-step
// path (the exact integer q, then one multiply).
template <int FMT>
MOE_DEV void dequant_store32(uint4 codes, uint32_t mult, uint32_t mult2, uint32_t two, uint8_t* tile, int r,
                             int half) {
  const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
  if (FMT == MOE_FMT_INT4_G128) {
    const uint32_t sv = mult & 0xFFFFu;
    if (sv - 0x0080u < 0x3D00u - 0x0080u) {
      const uint32_t m = (sv + 0x4280u) | ((sv + 0x4080u) << 16);  // (s 2^133, s 2^129)
      const uint32_t bias = mult + 0x81808180u;                     // -8 s in both halves
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          o[c] = bf16x2_fma(prmt(w[j], 0u, 0x4040u | uint32_t(c) | (uint32_t(c) << 8)) & 0x00F0000Fu, m, bias);
        *reinterpret_cast<uint4*>(tile + sw128_offset(r, half * 4 + j)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      return;
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t P[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t v;
      if (FMT == MOE_FMT_INT4_G128) {
        v = int4_pair(w[j], i);
      } else {
        // E2M1 codes as value * 2^-126; the multipliers carry 2^126 unless `two`
        v = e2m1_pair_scaled(w[j], i);
        if (two) v = bf16x2_mul(v, kBf16x2Pow126);
      }
      P[i] = bf16x2_mul(v, j < 2 ? mult : mult2);  // (k+i, k+i+4)
    }
    uint4 o;
    o.x = prmt(P[0], P[1], 0x5410u);  // k0 k1
    o.y = prmt(P[2], P[3], 0x5410u);  // k2 k3
    o.z = prmt(P[0], P[1], 0x7632u);  // k4 k5
    o.w = prmt(P[2], P[3], 0x7632u);  // k6 k7
    const int c = half * 4 + j;
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = o;
  }
}

template <int MODE, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                        const GemmArgs args) {
  using C = Cfg<MODE, FMT>;
  constexpr int SA = C::SA;
  constexpr int SB = C::SB;
  constexpr int kSrow = C::SROW;
  constexpr int NACC = C::NACC;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment by an offset into the shared array (not by integer
  // arithmetic on its address), so every access below stays a shared-memory
  // access instead of a generic one
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;                          // [SA][NACC][16 KB]
  uint8_t* sB = sA + C::SMEM_A;                // [SB][16 KB]
  uint8_t* sC = sB + C::SMEM_B;                // [SC][NACC][4 KB]
  uint8_t* sS = sC + C::SMEM_C;                // [2][NACC][BM rows][scale row bytes]
  float* sD = reinterpret_cast<float*>(sS + C::SMEM_S);  // down: [BN tokens][BM rows]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sS + C::SMEM_S + C::SMEM_D);
  uint64_t* codes_full = bars;                 // [SC]
  uint64_t* codes_empty = codes_full + SC;     // [SC]
  uint64_t* opA_full = codes_empty + SC;       // [SA]
  uint64_t* opA_empty = opA_full + SA;         // [SA]
  uint64_t* opB_full = opA_empty + SA;         // [SB]
  uint64_t* opB_empty = opB_full + SB;         // [SB]
  uint64_t* acc_full = opB_empty + SB;         // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* drain = acc_empty + 2;             // [1]
  uint64_t* sc_full = drain + 1;               // [2] scale rows of a tile
  uint64_t* sc_empty = sc_full + 2;            // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sc_empty + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tile_base = reinterpret_cast<int*>(bars + 64);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GemmArgs& a = args;
  // scale bytes per weight row (INT4: bf16 per 128 k; MXFP4: one byte per 32 k)
  const int sb = FMT == MOE_FMT_INT4_G128 ? 2 * a.scale_row_stride : a.scale_row_stride;  // bytes

  if (threadIdx.x == 0) {
    for (int i = 0; i < SC; ++i) {
      mbar_init(&codes_full[i], 1);
      mbar_init(&codes_empty[i], kDqThreads / 32);
    }
    for (int i = 0; i < SA; ++i) {
      mbar_init(&opA_full[i], MODE == kRouter ? 1 : kDqThreads / 32);
      mbar_init(&opA_empty[i], 1);
    }
    for (int i = 0; i < SB; ++i) {
      mbar_init(&opB_full[i], MODE == kDown ? 1 : 64);
      mbar_init(&opB_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
      mbar_init(&sc_full[i], 1);
      mbar_init(&sc_empty[i], kDqThreads / 32);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (MODE != kRouter)
    for (int i = threadIdx.x; i <= a.E; i += kThreads) s_tile_base[i] = a.tile_base[i];
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_a);
    if (MODE == kDown) tma_prefetch_desc(&tmap_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = num_tiles(a, s_tile_base);
  const int KS = a.K / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const Tile t = decode_tile(a, tile, s_tile_base);
        // the CTA's next tile, for the L2 prefetch of code tiles ahead of the ring
        const bool has_next = tile + int(gridDim.x) < ntiles;
        const Tile tn = has_next ? decode_tile(a, tile + gridDim.x, s_tile_base) : t;
        if (MODE != kRouter) {
          // the tile's scale rows: contiguous rows of the scale plane, once per tile
          const int slot = it & 1;
          if (!(ok = mbar_wait_backoff(&sc_empty[slot], ((it >> 1) & 1) ^ 1, abort, a.status, kProducerSleepNs)))
            break;
          const int f0 = t.fb * BM;
          const int rows = min(BM, a.M_total - f0);
          const uint32_t bytes = uint32_t(rows * sb);
          mbar_arrive_expect_tx(&sc_full[slot], NACC * bytes);
          const uint8_t* sp = static_cast<const uint8_t*>(a.scales);
#pragma unroll
          for (int c = 0; c < NACC; ++c) {
            long row0;
            if (MODE == kGateUp) row0 = long(t.eb) * 2 * a.I + (c ? a.I : 0) + f0;
            else row0 = long(t.eb) * a.H + f0;
            bulk_g2s(sS + (slot * NACC + c) * BM * kSrow, sp + row0 * sb, bytes, &sc_full[slot]);
          }
        }
        for (int ks = 0; ks < KS; ++ks, ++g) {
          if (MODE == kRouter) {
            const int s = g % SA;
            if (!(ok = mbar_wait(&opA_empty[s], ((g / SA) & 1) ^ 1, abort, a.status))) break;
            mbar_arrive_expect_tx(&opA_full[s], kTileBytes);
            tma_load_2d(sA + s * NACC * kTileBytes, &tmap_a, &opA_full[s], ks * BK, t.fb * BM);
          } else {
            const int s = g % SC;
            if (!(ok = mbar_wait_backoff(&codes_empty[s], ((g / SC) & 1) ^ 1, abort, a.status, kProducerSleepNs)))
              break;
            mbar_arrive_expect_tx(&codes_full[s], NACC * kCodeBytes);
            uint8_t* dst = sC + s * NACC * kCodeBytes;
            if (MODE == kGateUp) {
              tma_load_3d(dst, &tmap_a, &codes_full[s], ks * (BK / 2), t.fb * BM, 2 * t.eb);
              tma_load_3d(dst + kCodeBytes, &tmap_a, &codes_full[s], ks * (BK / 2), t.fb * BM, 2 * t.eb + 1);
            } else {
              tma_load_3d(dst, &tmap_a, &codes_full[s], ks * (BK / 2), t.fb * BM, t.eb);
            }
            // the code tile kCodePrefetch stages ahead, into L2
            const int kp = ks + kCodePrefetch;
            if (kp < KS || has_next) {
              const Tile& tp = kp < KS ? t : tn;
              const int kq = kp < KS ? kp : kp - KS;
              if (kq < KS) {
                if (MODE == kGateUp) {
                  tma_prefetch_3d(&tmap_a, kq * (BK / 2), tp.fb * BM, 2 * tp.eb);
                  tma_prefetch_3d(&tmap_a, kq * (BK / 2), tp.fb * BM, 2 * tp.eb + 1);
                } else {
                  tma_prefetch_3d(&tmap_a, kq * (BK / 2), tp.fb * BM, tp.eb);
                }
              }
            }
          }
        }
      }
      if (!ok) {
        // let copies already in flight land before the CTA unwinds
        volatile int never = 0;
        for (uint32_t i = 0; i < (MODE == kRouter ? SA : SC) && i < g; ++i) {
          const uint32_t gg = g - 1 - i;
          if (MODE == kRouter)
            mbar_wait(&opA_full[gg % SA], (gg / SA) & 1, &never, nullptr);
          else
            mbar_wait(&codes_full[gg % SC], (gg / SC) & 1, &never, nullptr);
        }
        if (MODE != kRouter && it > 0) {
          const int last = it - 1;
          mbar_wait(&sc_full[last & 1], (last >> 1) & 1, &never, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const Tile t = decode_tile(a, tile, s_tile_base);
        const int buf = it & 1;
        if (!(ok = mbar_wait_backoff(&acc_empty[buf], ((it >> 1) & 1) ^ 1, abort, a.status, kMmaSleepNs))) break;
        tc_fence_after();
        const uint32_t n16 = uint32_t((t.n + 15) & ~15);
        const uint32_t idesc = umma_idesc_bf16(BM, n16);
        const uint32_t d0 = tmem_base + uint32_t(buf * NACC * BN);
        for (int ks = 0; ks < KS; ++ks, ++g) {
          const int sa = g % SA, sbuf = g % SB;
          if (!(ok = mbar_wait_backoff(&opA_full[sa], (g / SA) & 1, abort, a.status, kMmaSleepNs))) break;
          if (!(ok = mbar_wait_backoff(&opB_full[sbuf], (g / SB) & 1, abort, a.status, kMmaSleepNs))) break;
          // the token rows landed through cp.async (generic proxy): order them
          // before the tensor core's (async proxy) reads
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + sa * NACC * kTileBytes);
          const uint32_t b_addr = smem_u32(sB + sbuf * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = umma_desc_sw128(b_addr + kk * 32);
#pragma unroll
            for (int c = 0; c < NACC; ++c) {
              const uint64_t adesc = umma_desc_sw128(a_addr + c * kTileBytes + kk * 32);
              umma_bf16(d0 + c * BN, adesc, bdesc, idesc, (ks | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&opA_empty[sa]);
          umma_commit(&opB_empty[sbuf]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
      if (!ok) {
        volatile int never = 0;
        umma_commit(drain);
        mbar_wait(drain, 0, &never, nullptr);
      }
    }
  } else if (MODE == kDown && (warp == 2 || warp == 3)) {
    // ------------------------------------------------------------ activation tiles
    // The expert's activation rows are contiguous in sorted-row order: one
    // 2-D TMA copy (64 k x 128 rows, 128-byte swizzle) per stage.  Rows past
    // the expert's count belong to the next experts (their columns are not
    // used); rows past the array read as zeros.
    if (warp == 2 && lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const Tile t = decode_tile(a, tile, s_tile_base);
        for (int ks = 0; ks < KS; ++ks, ++g) {
          const int s = g % SB;
          if (!(ok = mbar_wait_backoff(&opB_empty[s], ((g / SB) & 1) ^ 1, abort, a.status, kProducerSleepNs))) break;
          mbar_arrive_expect_tx(&opB_full[s], kTileBytes);
          tma_load_2d(sB + s * kTileBytes, &tmap_b, &opB_full[s], ks * BK, t.p_begin);
        }
      }
      if (!ok) {
        // let copies already in flight land before the CTA unwinds
        volatile int never = 0;
        for (uint32_t i = 0; i < SB && i < g; ++i) {
          const uint32_t gg = g - 1 - i;
          mbar_wait(&opB_full[gg % SB], (gg / SB) & 1, &never, nullptr);
        }
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ token gather
    // The stage's copies signal its full barrier themselves when they land
    // (cp.async.mbarrier.arrive.noinc), so the gather never waits on its own
    // copies and runs up to SB stages ahead of the tensor core.
    const int lt = threadIdx.x - 64;  // 0..63
    const int c = lt & 7;             // 16-byte chunk of the 128-byte row slice
    const int r0 = lt >> 3;           // rows r0, r0+8, ..., r0+120
    uint32_t g = 0;
    bool ok = true;
    const int ld = (MODE == kDown) ? a.I : a.H;  // row length of the token operand
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const Tile t = decode_tile(a, tile, s_tile_base);
      const int n16 = (t.n + 15) & ~15;
      const uint16_t* src[BN / 8];
#pragma unroll
      for (int i = 0; i < BN / 8; ++i) {
        const int r = r0 + 8 * i;
        long row;
        if (MODE == kGateUp) row = a.sorted_rows[t.p_begin + (r < t.n ? r : 0)] / a.top_k;
        else row = t.p_begin + (r < t.n ? r : 0);
        src[i] = a.bsrc + row * ld + c * 8;
      }
      for (int ks = 0; ks < KS; ++ks, ++g) {
        const int s = g % SB;
        if (!(ok = mbar_wait_backoff(&opB_empty[s], ((g / SB) & 1) ^ 1, abort, a.status, kProducerSleepNs))) break;
        const uint32_t base = smem_u32(sB + s * kTileBytes);
#pragma unroll
        for (int i = 0; i < BN / 8; ++i) {
          const int r = r0 + 8 * i;
          if (r < n16) cp_async_16(base + sw128_offset(r, c), src[i] + ks * BK);
        }
        cp_async_mbar_arrive_noinc(&opB_full[s]);
      }
    }
    cp_async_wait<0>();  // nothing in flight into shared memory when the CTA exits
  } else if (warp >= 4 && warp < kEpiWarp0) {
    // ------------------------------------------------------------ dequantisation
    // Two threads per weight row: thread half h writes the row's 32 k at
    // 32 h .. 32 h + 31 of every 64-wide stage.
    if (MODE != kRouter) {
      const int d = threadIdx.x - 128;  // 0..255
      const int r = d >> 1, h = d & 1;
      uint32_t g = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const Tile t = decode_tile(a, tile, s_tile_base);
        const int f = t.fb * BM + r;
        const bool valid = f < a.M_total;
        const int slot = it & 1;
        if (!(ok = dq_wait(&sc_full[slot], (it >> 1) & 1, abort, a.status))) break;
        const uint8_t* srows = sS + slot * NACC * BM * kSrow + r * sb;
        const float gsc = FMT == MOE_FMT_NVFP4_G16 ? a.gscale[t.eb] : 0.f;
        for (int ks = 0; ks < KS; ++ks, ++g) {
          const int sc = g % SC, so = g % SA;
          if (!(ok = dq_wait(&codes_full[sc], (g / SC) & 1, abort, a.status))) break;
          if (!(ok = dq_wait(&opA_empty[so], ((g / SA) & 1) ^ 1, abort, a.status))) break;
#pragma unroll
          for (int c = 0; c < NACC; ++c) {
            const uint8_t* ctile = sC + (sc * NACC + c) * kCodeBytes + r * (BK / 2);
            const uint4 cw = *reinterpret_cast<const uint4*>(ctile + 16 * h);
            uint32_t m = 0, m2 = 0, two = 0;
            if (valid) {
              const uint8_t* srow = srows + c * BM * kSrow;
              if (FMT == MOE_FMT_INT4_G128) {
                const uint32_t sv = reinterpret_cast<const uint16_t*>(srow)[(ks * BK) / 128];
                m = sv | (sv << 16);
                m2 = m;
              } else if (FMT == MOE_FMT_NVFP4_G16) {
                // blocks of 16: (ks * 64 + 32 h) / 16 and the next one
                nv_mult_pair_scaled(srow + (ks * BK) / 16 + 2 * h, gsc, m, m2, two);
              } else {
                const int e = int(srow[(ks * BK) / 32 + h]) - 127;
                two = e > 1 ? 1u : 0u;
                m = pow2x2(two ? e : e + 126);
                m2 = m;
              }
            }
            dequant_store32<FMT>(cw, m, m2, two, sA + (so * NACC + c) * kTileBytes, r, h);
          }
          // this thread's bf16 stores before the tensor core reads them
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&opA_full[so]);
            mbar_arrive(&codes_empty[sc]);
          }
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sc_empty[slot]);  // the tile's scale rows are no longer read
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kEpiWarp0;  // TMEM lanes 32*ew .. 32*ew+31
    const int r = ew * 32 + lane;     // weight row inside the tile
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const Tile t = decode_tile(a, tile, s_tile_base);
      const int buf = it & 1;
      if (!(ok = mbar_wait_backoff(&acc_full[buf], (it >> 1) & 1, abort, a.status, kEpilogueSleepNs))) break;
      tc_fence_after();
      const int f = t.fb * BM + r;
      const bool row_ok = f < a.M_total;
      const uint32_t taddr = tmem_base + (uint32_t(ew * 32) << 16) + uint32_t(buf * NACC * BN);
      if (MODE == kDown) {
        // the previous tile's bulk reductions must have read the staging buffer
        if (it > 0) {
          if (r < BN) bulk_wait_read_all();
          named_barrier_sync(1, 128);
        }
      }
      for (int c0 = 0; c0 < t.n; c0 += 32) {
        uint32_t v0[32];
        tmem_ld32(taddr + c0, v0);
        if (MODE == kGateUp) {
          uint32_t v1[32];
          tmem_ld32(taddr + BN + c0, v1);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (c0 + j < t.n)
                a.act[size_t(t.p_begin + c0 + j) * a.I + f] =
                    f32_to_bf16_rn(silu_mul(__uint_as_float(v0[j]), __uint_as_float(v1[j])));
            }
          }
        } else if (MODE == kDown) {
          tmem_ld_wait();
          // weights of the 32 columns: lane j fetches column c0 + j
          float wgt = 0.f;
          if (c0 + lane < t.n) wgt = a.topk_w[a.sorted_rows[t.p_begin + c0 + lane]];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wgt, j);
            sD[(c0 + j) * BM + r] = wj * __uint_as_float(v0[j]);  // row-contiguous per token
          }
        } else {
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (c0 + j < t.n) a.logits[size_t(t.p_begin + c0 + j) * a.E + f] = __uint_as_float(v0[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (MODE == kDown) {
        // every row of the weighted tile is staged: one bulk add per token
        fence_proxy_async_smem();
        named_barrier_sync(1, 128);
        if (r < t.n) {
          const int rows = min(BM, a.M_total - t.fb * BM);
          if (a.ypart) {
            // the row's own slot of the per-row outputs: summed in slot order later
            bulk_s2g(a.ypart + size_t(t.p_begin + r) * a.H + t.fb * BM, sD + r * BM, uint32_t(rows * 4));
          } else {
            const int tok = a.sorted_rows[t.p_begin + r] / a.top_k;
            bulk_reduce_add_f32(a.out_acc + size_t(tok) * a.H + t.fb * BM, sD + r * BM, uint32_t(rows * 4));
          }
          bulk_commit_group();
        }
      }
    }
    if (MODE == kDown) bulk_wait_all();  // the reductions are complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// fp32 accumulator (+ the shared expert's gated output) -> bf16 output
__global__ void finalize_kernel(const float* __restrict__ acc, long n, int H, const float* __restrict__ sh_gate,
                                const float* __restrict__ sh_y, uint16_t* __restrict__ out) {
  const long i = (long(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 v = *reinterpret_cast<const float4*>(acc + i);
  if (sh_y) {
    const float g = sh_gate[i / H];  // H % 4 == 0: the four elements share a token
    const float4 y = *reinterpret_cast<const float4*>(sh_y + i);
    v.x += g * y.x;
    v.y += g * y.y;
    v.z += g * y.z;
    v.w += g * y.w;
  }
  uint2 o;
  o.x = pack_bf16x2(v.x, v.y);
  o.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(out + i) = o;
}

// out[t] = bf16(sum over slots j in order of ypart[pos[t k + j]] (+ the shared
// expert's gated output)): the deterministic combine of per-row outputs that
// already carry their routing weight.  With partial_out, the fp32 sum over
// the slots whose sorted position lies in [offsets[e_lo], offsets[e_hi]) (an
// expert-parallel shard's experts) instead.  One thread per 4 features.
__global__ void combine_rows_kernel(const float* __restrict__ ypart, const int32_t* __restrict__ pos,
                                    const int32_t* __restrict__ offsets, int e_lo, int e_hi, int T, int H, int k,
                                    const float* __restrict__ sh_gate, const float* __restrict__ sh_y,
                                    uint16_t* __restrict__ out, float* __restrict__ partial_out) {
  pdl_wait();
  pdl_trigger();
  const long i = (long(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= long(T) * H) return;
  const int t = int(i / H), f = int(i % H);
  const int p_lo = offsets[e_lo], p_hi = offsets[e_hi];
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int p = pos[size_t(t) * k + j];
    if (p < p_lo || p >= p_hi) continue;
    const float4 y = *reinterpret_cast<const float4*>(ypart + size_t(p) * H + f);
    v.x += y.x;
    v.y += y.y;
    v.z += y.z;
    v.w += y.w;
  }
  if (partial_out) {
    *reinterpret_cast<float4*>(partial_out + i) = v;
    return;
  }
  if (sh_y) {
    const float g = sh_gate[t];
    const float4 y = *reinterpret_cast<const float4*>(sh_y + i);
    v.x += g * y.x;
    v.y += g * y.y;
    v.z += g * y.z;
    v.w += g * y.w;
  }
  uint2 o;
  o.x = pack_bf16x2(v.x, v.y);
  o.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(out + i) = o;
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launches
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load();
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cached.store(fn);
    }
  }
  return fn;
}

// Codes of a packed bank viewed as [Z][rows][K/2] bytes, box 32 bytes x 128 rows.
bool make_codes_map(CUtensorMap* m, const uint8_t* codes, int K, int rows, long Z) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {cuuint64_t(K / 2), cuuint64_t(rows), cuuint64_t(Z)};
  const cuuint64_t strides[2] = {cuuint64_t(K / 2), cuuint64_t(K / 2) * rows};
  const cuuint32_t box[3] = {BK / 2, BM, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 matrix [rows][K] with the 128-byte swizzle, box 64 x 128.
bool make_bf16_sw128_map(CUtensorMap* m, const uint16_t* base, int K, int rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(K) * 2};
  const cuuint32_t box[2] = {BK, BM};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
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

template <int MODE, int FMT>
cudaError_t launch_gemm(const CUtensorMap& map, const CUtensorMap& map_b, const GemmArgs& args, int max_ctas,
                        cudaStream_t stream) {
  auto kern = grouped_gemm_kernel<MODE, FMT>;
  const int smem = Cfg<MODE, FMT>::SMEM;
  // once per process (and per device), outside any stream capture of later calls
  static std::atomic<int> configured_device{-1};
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_device.load() != dev) {  // setting it twice from two threads is harmless
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    configured_device.store(dev);
  }
  const int grid = max(1, min(sm_count(), max_ctas));
  kern<<<grid, kThreads, smem, stream>>>(map, map_b, args);
  return cudaGetLastError();
}

GemmArgs base_args(const moe_shape_t& s, int T, const ExpertRange& er, const Workspace& ws) {
  GemmArgs a{};
  a.e_lo = er.lo;
  a.e_hi = er.hi;
  a.fmt = int(s.fmt);
  a.T = T;
  a.top_k = s.top_k;
  a.I = s.inter;
  a.H = s.hidden;
  a.E = s.num_experts;
  a.offsets = ws.offsets;
  a.sorted_rows = ws.sorted_rows;
  a.tile_base = ws.tile_base;
  a.topk_w = ws.topk_w;
  a.logits = ws.logits;
  a.act = ws.act;
  a.out_acc = ws.out_acc;
  a.status = ws.status;
  return a;
}

// Upper bound of the grouped tile count (host side, no device read): every
// row in its own expert's partial block, bounded by the full count.
int grouped_tiles_bound(int T, int k, int E, int ftiles) {
  const long rows = long(T) * k;
  const long blocks = (rows + BN - 1) / BN + std::min<long>(E, rows);
  return int(std::min<long>(blocks * ftiles, 1L << 30));
}

}  // namespace

cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* wr, int T, int H, int E, float* logits,
                               uint32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  CUtensorMap map;
  if (!make_bf16_sw128_map(&map, wr, H, E)) return cudaErrorInvalidValue;
  GemmArgs a{};
  a.mode = kRouter;
  a.K = H;
  a.M_total = E;
  a.n_ftiles = (E + BM - 1) / BM;
  a.T = T;
  a.H = H;
  a.E = E;
  a.bsrc = x;
  a.logits = logits;
  a.status = status;
  const int tiles = a.n_ftiles * ((T + BN - 1) / BN);
  return launch_gemm<kRouter, 0>(map, map, a, tiles, stream);
}

bool grouped_supported(const moe_shape_t& s) {
  // a tile's scale rows are staged in shared memory, up to kMaxScaleRow(Nv) bytes per row
  const auto row_bytes = [&](int K) {
    return s.fmt == MOE_FMT_INT4_G128 ? 2 * int4_groups(K) : s.fmt == MOE_FMT_NVFP4_G16 ? K / 16 : K / 32;
  };
  const int cap = s.fmt == MOE_FMT_NVFP4_G16 ? kMaxScaleRowNv
                  : s.fmt == MOE_FMT_INT4_G128 ? kMaxScaleRowInt4 : kMaxScaleRow;
  return row_bytes(s.hidden) <= cap && row_bytes(s.inter) <= cap;
}

cudaError_t launch_grouped_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu,
                                   const ExpertRange& er, const Workspace& ws, cudaStream_t stream) {
  if (T == 0 || er.hi <= er.lo) return cudaSuccess;
  CUtensorMap map;
  if (!make_codes_map(&map, gu.codes, gu.K, s.inter, 2L * (er.hi - er.lo))) return cudaErrorInvalidValue;
  GemmArgs a = base_args(s, T, er, ws);
  a.mode = kGateUp;
  a.K = s.hidden;
  a.M_total = s.inter;
  a.n_ftiles = (s.inter + BM - 1) / BM;
  a.bsrc = x;
  a.scales = gu.scales;
  a.scale_row_stride = s.fmt == MOE_FMT_INT4_G128 ? int4_groups(gu.K) : s.fmt == MOE_FMT_NVFP4_G16 ? gu.K / 16 : gu.K / 32;
  a.gscale = gu.gscale;
  const int bound = grouped_tiles_bound(T, s.top_k, s.num_experts, a.n_ftiles);
  if (s.fmt == MOE_FMT_INT4_G128) return launch_gemm<kGateUp, MOE_FMT_INT4_G128>(map, map, a, bound, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return launch_gemm<kGateUp, MOE_FMT_NVFP4_G16>(map, map, a, bound, stream);
  return launch_gemm<kGateUp, MOE_FMT_MXFP4_G32>(map, map, a, bound, stream);
}

cudaError_t launch_grouped_down(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er,
                                const Workspace& ws, float* acc, float* ypart, cudaStream_t stream) {
  if (T == 0 || er.hi <= er.lo) return cudaSuccess;
  CUtensorMap map;
  if (!make_codes_map(&map, dn.codes, dn.K, s.hidden, er.hi - er.lo)) return cudaErrorInvalidValue;
  GemmArgs a = base_args(s, T, er, ws);
  a.out_acc = acc;
  a.ypart = ypart;
  a.mode = kDown;
  a.K = s.inter;
  a.M_total = s.hidden;
  a.n_ftiles = (s.hidden + BM - 1) / BM;
  a.bsrc = ws.act;
  a.scales = dn.scales;
  a.scale_row_stride = s.fmt == MOE_FMT_INT4_G128 ? int4_groups(dn.K) : s.fmt == MOE_FMT_NVFP4_G16 ? dn.K / 16 : dn.K / 32;
  a.gscale = dn.gscale;
  const int bound = grouped_tiles_bound(T, s.top_k, s.num_experts, a.n_ftiles);
  // the activation rows [T*k, I] bf16 in sorted order, tiles of 64 k x 128 rows
  CUtensorMap map_b;
  if (!make_bf16_sw128_map(&map_b, ws.act, s.inter, T * s.top_k)) return cudaErrorInvalidValue;
  if (s.fmt == MOE_FMT_INT4_G128) return launch_gemm<kDown, MOE_FMT_INT4_G128>(map, map_b, a, bound, stream);
  if (s.fmt == MOE_FMT_NVFP4_G16) return launch_gemm<kDown, MOE_FMT_NVFP4_G16>(map, map_b, a, bound, stream);
  return launch_gemm<kDown, MOE_FMT_MXFP4_G32>(map, map_b, a, bound, stream);
}

cudaError_t launch_combine_rows(const moe_shape_t& s, int T, const ExpertRange& er, const Workspace& ws,
                                const float* ypart, const float* sh_gate, const float* sh_y, uint16_t* out,
                                float* partial_out, cudaStream_t stream) {
  const long n = long(T) * s.hidden;
  if (n == 0) return cudaSuccess;
  const int block = 256;
  const long threads = (n + 3) / 4;
  return launch_pdl(combine_rows_kernel, dim3(unsigned((threads + block - 1) / block)), dim3(block), 0, stream,
                    ypart, (const int32_t*)ws.pos, (const int32_t*)ws.offsets, er.lo, er.hi, T, s.hidden, s.top_k,
                    sh_gate, sh_y, out, partial_out);
}

cudaError_t launch_finalize_out(const float* acc, int T, int H, const float* sh_gate, const float* sh_y,
                                uint16_t* out, cudaStream_t stream) {
  const long n = long(T) * H;
  if (n == 0) return cudaSuccess;
  const int block = 256;
  const long threads = (n + 3) / 4;
  finalize_kernel<<<unsigned((threads + block - 1) / block), block, 0, stream>>>(acc, n, H, sh_gate, sh_y, out);
  return cudaGetLastError();
}

}  // namespace moe
