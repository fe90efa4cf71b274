// Device helpers of the decode (small-batch) expert kernels: mma.sync
// m16n8k16 on dequantised 4-bit weight fragments, the fragment k-permutation
// shared by weights and activations, and the shared-memory layouts the
// kernels stage weights and activations in.
//
// Fragment k-permutation.  Inside a 128-k block, lane (g = lane/4, q = lane%4)
// owns k in [32q, 32q+32).  For MMA step s = 2*j + h (j = 32-bit code word,
// h = 0/1) the lane's fragment positions {2q, 2q+1, 2q+8, 2q+9} hold
// k0+2h, k0+2h+4, k0+2h+1, k0+2h+5 with k0 = 32q + 8j.  A dot product does not
// depend on the order of its terms, so weights and activations only need the
// same assignment; this one lets one mask instruction produce a fragment
// register's pair of codes directly.
//
// INT4 dequantisation, bf16(q * s) with q = u - 8 from the offset-binary nibble
// u.  A bf16 bit pattern below 256 (exponent field 0 or 1) has the value
// pattern * 2^-133: linear, across the subnormal range and the first normal
// binade.  So masking a code word with 0x000F000F leaves two bf16 values
// u * 2^-133 (nibbles 0 and 4), and masking with 0x00F000F0 two values
// u * 2^-129 (nibbles 1 and 5); the word shifted right by 8 gives nibbles
// (2, 6) and (3, 7) the same way.  One bf16 fused multiply-add
//     fma(u * 2^-133, s * 2^133, -8 s) = (u - 8) s = q s
// computes the product exactly before its single rounding, i.e. bf16(q * s).
// s * 2^133 and s * 2^129 are bf16 values when s is normal and below 2^-5
// (exponent field 1..121); they are built by adding to the exponent field.
// Other scales (zero, subnormal, >= 2^-5) take the two-step path: the exact
// small integer q = (128 + u) - 136, then one multiply by s.  The choice is
// made once per warp and work unit, so the inner loop has no branches.
//
// Shared-memory layouts.
//  * Weight tiles (gate_up): the 16 gate rows of a unit, then 64 bytes of
//    padding, then its 16 up rows, each run one bulk copy.  A 16-byte load of
//    rows g and g + 1 by one 8-lane phase would hit the same bank half when
//    both rows sit in one run (rows are a multiple of 128 bytes long); lanes
//    with odd g therefore take the up row as their low MMA row and the gate
//    row as their high one, so the two rows of a phase are in different runs,
//    64 bytes apart modulo 128.
//  * Activation rows in fragment order: row r, k-block b starts at
//    r * pstride + 256 b, and its 16-byte unit 4 i + q holds lane slice q's
//    fragment words of MMA steps 2i and 2i+1, so a lane's 16 fragment words
//    are four 16-byte loads with no permutes and four consecutive lanes read
//    64 consecutive bytes.  pstride = 256 * blocks + 64 puts consecutive rows
//    in opposite bank halves.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

MOE_DEV void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  // not volatile: a pure function of its registers, free to be scheduled
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16x2 with both halves = 2^e (e in [-127, 127]; 2^-127 is subnormal).
MOE_DEV uint32_t pow2_bf16x2(int e) {
  const uint32_t b = e >= -126 ? uint32_t(e + 127) << 7 : 0x0040u;
  return b | (b << 16);
}

// MXFP4 multiplier of exponent e for E2M1 codes placed as value * 2^-126:
// 2^(e + 126) when that is a bf16 value (e <= 1), else 2^e with the two-step
// flag (the codes are first multiplied by 2^126).
MOE_DEV void mx_mult(int e, uint32_t& mult, uint32_t& two) {
  two = e > 1 ? 1u : 0u;
  mult = pow2_bf16x2(two ? e : e + 126);
}

MOE_DEV uint32_t word_of(const uint4& c, int j) {
  return j == 0 ? c.x : j == 1 ? c.y : j == 2 ? c.z : c.w;
}

// Scale bytes per weight row of a bank with reduction length K.
__host__ __device__ inline int scale_row_bytes(int fmt, int K) {
  return fmt == MOE_FMT_INT4_G128 ? int4_groups(K) * 2 : fmt == MOE_FMT_NVFP4_G16 ? K / 16 : K / 32;
}

// What turns a lane's 16 code bytes of one weight row at one 128-k block into
// bf16 weights:
//   INT4:  m0 = s * 2^133, m1 = s * 2^129, m2 = -8 s (bf16x2, both halves
//          equal); the two-step path multiplies by s, recovered as m0 minus
//          the constant that added 133 to the exponent field.
//   MXFP4: m0 = m1 = the multiplier of its 32-element block, m2 = the
//          two-step flag.
//   NVFP4: m0 / m1 = the multipliers of its two 16-element blocks (code words
//          0-1 / 2-3), m2 = the two-step flag.
// A slice past K has zero multipliers (and zero codes): zero weights.
struct Mult {
  uint32_t m0, m1, m2;
};

// The raw scale bits of one lane slice of one weight row at k-block b: INT4
// the bf16 scale of group b, MXFP4 the exponent byte of 32-element block
// 4b + q, NVFP4 the two E4M3 bytes of 16-element blocks 8b + 2q, 8b + 2q + 1.
// `row` points at the row's scales in shared memory, or in global memory
// (read-only for the kernel's lifetime) with GLOBAL.
template <int FMT, bool GLOBAL>
MOE_DEV uint32_t raw_scale(const uint8_t* row, int b, int q) {
  if (FMT == MOE_FMT_INT4_G128) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(row) + b;
    return GLOBAL ? __ldg(p) : *p;
  }
  if (FMT == MOE_FMT_NVFP4_G16) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(row + 8 * b + 2 * q);
    return GLOBAL ? __ldg(p) : *p;
  }
  const uint8_t* p = row + 4 * b + q;
  return GLOBAL ? __ldg(p) : *p;
}

// Multipliers from raw scale bits; `fast` is cleared when the
// single-instruction path is not exact for them.  A slice outside the row
// (`in` false) gets zero weights.
template <int FMT>
MOE_DEV Mult mult_of(uint32_t raw, float gsc, bool in, bool& fast) {
  Mult m;
  if (!in) {
    // zero weights on both paths (INT4's two-step multiplier m0 - C is 0)
    m.m0 = FMT == MOE_FMT_INT4_G128 ? 0x42804280u : 0u;
    m.m1 = m.m2 = 0u;
    return m;
  }
  if (FMT == MOE_FMT_INT4_G128) {
    const uint32_t sd = raw * 0x00010001u;
    m.m0 = sd + 0x42804280u;  // exponent + 133
    m.m1 = sd + 0x40804080u;  // exponent + 129
    m.m2 = sd + 0x81808180u;  // exponent + 3, sign set: -8 s
    fast = fast && (raw - 0x0080u < 0x3D00u - 0x0080u);
  } else if (FMT == MOE_FMT_NVFP4_G16) {
    nv_mult_pair_scaled_v(uint16_t(raw), gsc, m.m0, m.m1, m.m2);
    fast = fast && m.m2 == 0u;
  } else {
    mx_mult(int(raw) - 127, m.m0, m.m2);
    m.m1 = m.m0;
    fast = fast && m.m2 == 0u;
  }
  return m;
}

// The bf16 pair (nibbles i, i+4) of code word j.
template <int FMT, bool FAST>
MOE_DEV uint32_t dq(const Mult& m, uint32_t word, int i, int j) {
  if (FMT == MOE_FMT_INT4_G128) {
    if (FAST) {
      const uint32_t t = i >= 2 ? word >> 8 : word;
      const uint32_t v = t & ((i & 1) ? 0x00F000F0u : 0x000F000Fu);
      return bf16x2_fma(v, (i & 1) ? m.m1 : m.m0, m.m2);
    }
    return bf16x2_mul(int4_pair(word, i), m.m0 - 0x42804280u);
  }
  // E2M1: codes as value * 2^-126; the multipliers carry 2^126 unless m2
  uint32_t v = e2m1_pair_scaled(word, i);
  if (!FAST && m.m2) v = bf16x2_mul(v, kBf16x2Pow126);
  return bf16x2_mul(v, (FMT == MOE_FMT_NVFP4_G16 && j >= 2) ? m.m1 : m.m0);
}

// acc[c0 + h] += W(rows r, r+8; one 128-k block) x activation fragments: the
// two MMA steps of each code word go to two accumulator chains, so chains of
// independent MMAs are in flight instead of one.
template <int FMT, bool FAST, int CH>
MOE_DEV void mma_kblock(float (&acc)[CH][4], int c0, const uint4& lo, const uint4& hi, const Mult& mlo,
                        const Mult& mhi, const uint32_t (&b)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wl = word_of(lo, j), wh = word_of(hi, j);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a[4];
      a[0] = dq<FMT, FAST>(mlo, wl, 2 * h, j);
      a[1] = dq<FMT, FAST>(mhi, wh, 2 * h, j);
      a[2] = dq<FMT, FAST>(mlo, wl, 2 * h + 1, j);
      a[3] = dq<FMT, FAST>(mhi, wh, 2 * h + 1, j);
      mma_bf16_16816(acc[c0 + h], a, b[2 * j + h][0], b[2 * j + h][1]);
    }
  }
}

// Raw words X[m] = (v[32q+2m], v[32q+2m+1]) -> the permuted fragment pairs of
// the 8 MMA steps (see the fragment k-permutation above).
MOE_DEV void act_frags_from_raw(const uint32_t (&X)[16], uint32_t (&b)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    b[2 * j][0] = prmt(X[4 * j], X[4 * j + 2], 0x5410u);
    b[2 * j][1] = prmt(X[4 * j], X[4 * j + 2], 0x7632u);
    b[2 * j + 1][0] = prmt(X[4 * j + 1], X[4 * j + 3], 0x5410u);
    b[2 * j + 1][1] = prmt(X[4 * j + 1], X[4 * j + 3], 0x7632u);
  }
}

// Activation fragments of one lane's 32-k slice (64 bytes at p) of a bf16 row
// in global memory.  SRC 1: read-only for the kernel's lifetime
// (ld.global.nc); 2: written by an earlier kernel (ld.global.cg).  With
// `valid` false the fragments are zero (slices past K).
template <int SRC>
MOE_DEV void act_frags_global(const uint16_t* p, bool valid, uint32_t (&b)[8][2]) {
  uint32_t X[16];
  if (valid) {
    const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w = SRC == 1 ? __ldg(v + i) : __ldcg(v + i);
      X[4 * i] = w.x; X[4 * i + 1] = w.y; X[4 * i + 2] = w.z; X[4 * i + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
  act_frags_from_raw(X, b);
}

// Activation fragments of lane slice q of a k-block staged in fragment order
// (`blk` = the row's block start).
MOE_DEV void act_frags_staged(const uint8_t* blk, int q, bool valid, uint32_t (&b)[8][2]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = valid ? *reinterpret_cast<const uint4*>(blk + (4 * i + q) * 16) : make_uint4(0, 0, 0, 0);
    b[2 * i][0] = v.x;
    b[2 * i][1] = v.y;
    b[2 * i + 1][0] = v.z;
    b[2 * i + 1][1] = v.w;
  }
}

// Number of 128-k blocks of a row of length K, and the row stride of bf16
// rows staged in fragment order.
__host__ __device__ inline int kblocks(int K) { return (K + 127) / 128; }
__host__ __device__ inline int staged_act_stride(int K) { return 256 * kblocks(K) + 64; }

// Stage `rows` bf16 rows of length K (global, row stride K) in fragment order
// at `dst`; slices past K are zero.  Threads `tid` of `nthreads` share the
// work, one (row, block, lane slice) of 64 bytes at a time: four adjacent
// threads read 256 consecutive bytes and write 64-byte runs.
template <int SRC>
MOE_DEV void stage_act_rows(uint8_t* dst, const uint16_t* src, int rows, int K, int tid, int nthreads) {
  const int nblk = kblocks(K);
  const int pstride = staged_act_stride(K);
  const int items = rows * nblk * 4;
  for (int it = tid; it < items; it += nthreads) {
    const int q = it & 3, rb = it >> 2;
    const int r = rb / nblk, b = rb - r * nblk;
    const int k0 = 128 * b + 32 * q;
    uint32_t X[16];
    if (k0 < K) {
      const uint4* v = reinterpret_cast<const uint4*>(src + size_t(r) * K + k0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = SRC == 1 ? __ldg(v + i) : __ldcg(v + i);
        X[4 * i] = w.x; X[4 * i + 1] = w.y; X[4 * i + 2] = w.z; X[4 * i + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) X[i] = 0;
    }
    uint32_t f[8][2];
    act_frags_from_raw(X, f);
    uint8_t* o = dst + size_t(r) * pstride + 256 * b + 16 * q;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(o + 64 * i) = make_uint4(f[2 * i][0], f[2 * i][1], f[2 * i + 1][0], f[2 * i + 1][1]);
  }
}

// One warp: acc[j][t] += W_t x B_j over NB k-blocks b0, b0 + bstep, ... of
// MT 16-row weight tiles whose codes sit in shared memory (tile t: the lane's
// row at c_lo[t], its row + 8 at c_hi[t], scales at s_lo[t] / s_hi[t]), for
// the token tiles j < ntiles.  `act.load(j, b, in, frags)` gives token tile
// j's fragments of block b.  With `partial` (NB = 1) the block may end inside
// K: lane slices past K contribute zero.  The fast / two-step choice is made
// once for all NB blocks; CH accumulator chains per tile (blocks alternate
// between chain pairs when CH = 4).
template <int FMT, int NT, int MT, int CH, int NB, typename Act>
MOE_DEV void smem_blocks(float (&acc)[NT][MT][CH][4], const uint8_t* const (&c_lo)[MT],
                         const uint8_t* const (&c_hi)[MT], const uint8_t* const (&s_lo)[MT],
                         const uint8_t* const (&s_hi)[MT], int b0, int bstep, int K, int q, float gsc, int ntiles,
                         bool partial, const Act& act) {
  Mult mlo[MT][NB], mhi[MT][NB];
  bool fast = true;
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int b = b0 + i * bstep;
    const bool in = !partial || 128 * b + 32 * q < K;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      mlo[t][i] = mult_of<FMT>(in ? raw_scale<FMT, false>(s_lo[t], b, q) : 0u, gsc, in, fast);
      mhi[t][i] = mult_of<FMT>(in ? raw_scale<FMT, false>(s_hi[t], b, q) : 0u, gsc, in, fast);
    }
  }
  // warp-uniform: mma.sync needs the whole warp on one path (the two-step
  // path is exact for every scale)
  const bool all_fast = __all_sync(0xffffffffu, fast);
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    const int b = b0 + i * bstep;
    const bool in = !partial || 128 * b + 32 * q < K;
    uint4 lo[MT], hi[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      lo[t] = in ? *reinterpret_cast<const uint4*>(c_lo[t] + 64 * b) : make_uint4(0, 0, 0, 0);
      hi[t] = in ? *reinterpret_cast<const uint4*>(c_hi[t] + 64 * b) : make_uint4(0, 0, 0, 0);
    }
    const int c0 = CH == 4 ? 2 * (i & 1) : 0;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j > 0 && j >= ntiles) break;
      uint32_t bf[8][2];
      act.load(j, b, in, bf);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        if (all_fast) mma_kblock<FMT, true, CH>(acc[j][t], c0, lo[t], hi[t], mlo[t][i], mhi[t][i], bf);
        else mma_kblock<FMT, false, CH>(acc[j][t], c0, lo[t], hi[t], mlo[t][i], mhi[t][i], bf);
      }
    }
  }
}

// One warp's share of a unit staged in shared memory: the nb full k-blocks
// b0, b0 + bstep, ... (UNB at a time where possible) and, if tail_b >= 0,
// the partial block tail_b.
template <int FMT, int NT, int MT, int CH, int UNB, typename Act>
MOE_DEV void smem_unit(float (&acc)[NT][MT][CH][4], const uint8_t* const (&c_lo)[MT], const uint8_t* const (&c_hi)[MT],
                       const uint8_t* const (&s_lo)[MT], const uint8_t* const (&s_hi)[MT], int b0, int bstep, int nb,
                       int tail_b, int K, int q, float gsc, int ntiles, const Act& act) {
  int i = 0;
  for (; i + UNB <= nb; i += UNB)
    smem_blocks<FMT, NT, MT, CH, UNB>(acc, c_lo, c_hi, s_lo, s_hi, b0 + i * bstep, bstep, K, q, gsc, ntiles, false,
                                      act);
  for (; i < nb; ++i)
    smem_blocks<FMT, NT, MT, CH, 1>(acc, c_lo, c_hi, s_lo, s_hi, b0 + i * bstep, bstep, K, q, gsc, ntiles, false, act);
  if (tail_b >= 0)
    smem_blocks<FMT, NT, MT, CH, 1>(acc, c_lo, c_hi, s_lo, s_hi, tail_b, 1, K, q, gsc, ntiles, true, act);
}

// Four consecutive k-blocks b0 .. b0 + 3 of one 16-row weight tile held in
// registers (loaded from global memory): the lane's codes of its row (lo) and
// row + 8 (hi) and their raw scales.  Blocks at or past nblk, and lane slices
// past K, hold zeros.
struct RegChunk {
  uint4 lo[4], hi[4];
  uint32_t slo[4], shi[4];
};

// Load a RegChunk: codes_lo / codes_hi point at the two rows' codes plus the
// lane's slice offset 16q, scales_lo / scales_hi at their scales (global,
// read-only for the kernel's lifetime; the codes are read once, so they are
// not kept in L1).  FULL: all four blocks lie inside K (no checks).
template <int FMT, bool FULL>
MOE_DEV void load_chunk(RegChunk& c, const uint8_t* codes_lo, const uint8_t* codes_hi, const uint8_t* scales_lo,
                        const uint8_t* scales_hi, int b0, int nblk, int K, int q) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + i;
    if (FULL) {
      c.lo[i] = ldg_nc_v4(codes_lo + 64 * b);
      c.hi[i] = ldg_nc_v4(codes_hi + 64 * b);
      c.slo[i] = raw_scale<FMT, true>(scales_lo, b, q);
      c.shi[i] = raw_scale<FMT, true>(scales_hi, b, q);
    } else {
      const bool in = b < nblk && 128 * b + 32 * q < K;
      c.lo[i] = in ? ldg_nc_v4(codes_lo + 64 * b) : make_uint4(0, 0, 0, 0);
      c.hi[i] = in ? ldg_nc_v4(codes_hi + 64 * b) : make_uint4(0, 0, 0, 0);
      c.slo[i] = in ? raw_scale<FMT, true>(scales_lo, b, q) : 0u;
      c.shi[i] = in ? raw_scale<FMT, true>(scales_hi, b, q) : 0u;
    }
  }
}

// acc[j] += W x B_j over the blocks of a RegChunk (block b0 + i for i < 4
// while b0 + i < nblk), for the token tiles j < ntiles.  FULL: all four
// blocks lie inside K.
template <int FMT, int NT, int CH, bool FULL, typename Act>
MOE_DEV void chunk_mma(float (&acc)[NT][CH][4], const RegChunk& c, int b0, int nblk, int K, int q, float gsc,
                       int ntiles, const Act& act) {
  Mult mlo[4], mhi[4];
  bool fast = true;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + i;
    const bool in = FULL || (b < nblk && 128 * b + 32 * q < K);
    mlo[i] = mult_of<FMT>(c.slo[i], gsc, in, fast);
    mhi[i] = mult_of<FMT>(c.shi[i], gsc, in, fast);
  }
  const bool all_fast = __all_sync(0xffffffffu, fast);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = b0 + i;
    if (!FULL && b >= nblk) break;  // warp-uniform
    const bool in = FULL || 128 * b + 32 * q < K;
    const int c0 = CH == 4 ? 2 * (i & 1) : 0;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j > 0 && j >= ntiles) break;
      uint32_t bf[8][2];
      act.load(j, b, in, bf);
      if (all_fast) mma_kblock<FMT, true, CH>(acc[j], c0, c.lo[i], c.hi[i], mlo[i], mhi[i], bf);
      else mma_kblock<FMT, false, CH>(acc[j], c0, c.lo[i], c.hi[i], mlo[i], mhi[i], bf);
    }
  }
}

// Bytes staged for `rows` consecutive weight rows (codes + scales).
template <int FMT>
MOE_DEV uint32_t staged_bytes(const Bank& bk, int rows) {
  return uint32_t(rows) * (bk.K / 2) + uint32_t(rows) * scale_row_bytes(FMT, bk.K);
}

// Prefetch into L2 the codes and scales of `rows` consecutive weight rows
// (one lane each: codes, scales).
template <int FMT>
MOE_DEV void prefetch_codes(const Bank& bk, long row0, int rows) {
  bulk_prefetch_l2(bk.codes + row0 * (bk.K / 2), uint32_t(rows) * (bk.K / 2));
}
template <int FMT>
MOE_DEV void prefetch_scales(const Bank& bk, long row0, int rows) {
  const int sb = scale_row_bytes(FMT, bk.K);
  bulk_prefetch_l2(static_cast<const uint8_t*>(bk.scales) + row0 * sb, uint32_t(rows) * sb);
}

}  // namespace moe
