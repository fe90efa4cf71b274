// Device helpers of the decode (small-batch) expert kernels: mma.sync
// m16n8k16 on dequantised 4-bit weight fragments, the fragment k-permutation
// shared by weights and activations, and the bulk-copy staging of packed rows.
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
// small integer q = (128 + u) - 136, then one multiply by s.
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

// A lane's 32-k slice of one weight row at one 128-k block: its 16 code bytes
// and what turns them into bf16 weights.
//   INT4:  m0 = s * 2^133, m1 = s * 2^129, m2 = -8 s (bf16x2, both halves
//          equal) and fast = 1 when those are exact, else fast = 0; sd = s in
//          both halves (the two-step path's multiplier).
//   MXFP4: m0 = m1 = the multiplier of its 32-element block, m2 = the
//          two-step flag.
//   NVFP4: m0 / m1 = the multipliers of its two 16-element blocks (code words
//          0-1 / 2-3), m2 = the two-step flag.
// A slice past K has zero codes and zero multipliers (zero weights).
struct RowChunk {
  uint4 codes;
  uint32_t m0, m1, m2;
  uint32_t sd;
  uint32_t fast;
};

// INT4 multipliers of scale bits s (see the top of this file).
MOE_DEV void int4_mults(uint32_t s, RowChunk& rc) {
  const uint32_t sd = s * 0x00010001u;
  rc.sd = sd;
  rc.m0 = sd + 0x42804280u;  // exponent + 133
  rc.m1 = sd + 0x40804080u;  // exponent + 129
  rc.m2 = sd + 0x81808180u;  // exponent + 3, sign set: -8 s
  rc.fast = (s - 0x0080u < 0x3D00u - 0x0080u) ? 1u : 0u;
}

// The chunk of k-block b of one staged weight row: `codes` points at the row's
// codes plus the lane's slice offset 16q, `scales` at the row's scales; `in` is
// false for a slice past K; `g` is the matrix's NVFP4 global scale.
template <int FMT>
MOE_DEV RowChunk row_chunk_at(const uint8_t* codes, const uint8_t* scales, int b, int q, bool in, float g = 0.f) {
  RowChunk rc;
  if (in) {
    rc.codes = *reinterpret_cast<const uint4*>(codes + 64 * b);
    if (FMT == MOE_FMT_INT4_G128) {
      int4_mults(reinterpret_cast<const uint16_t*>(scales)[b], rc);  // group b = k-block b
    } else if (FMT == MOE_FMT_NVFP4_G16) {
      // the slice holds two 16-element blocks: 8b + 2q and 8b + 2q + 1
      nv_mult_pair_scaled(scales + 8 * b + 2 * q, g, rc.m0, rc.m1, rc.m2);
      rc.fast = 1u;
    } else {
      mx_mult(int(scales[4 * b + q]) - 127, rc.m0, rc.m2);  // the slice is one 32-element block
      rc.m1 = rc.m0;
      rc.fast = 1u;
    }
  } else {
    rc.codes = make_uint4(0, 0, 0, 0);
    rc.m0 = rc.m1 = rc.m2 = rc.sd = 0u;
    rc.fast = 1u;
  }
  return rc;
}

// The bf16 pair (nibbles i, i+4) of code word j of a chunk.
template <int FMT, bool FAST>
MOE_DEV uint32_t dq(const RowChunk& rc, uint32_t word, int i, int j) {
  if (FMT == MOE_FMT_INT4_G128) {
    if (FAST) {
      const uint32_t t = i >= 2 ? word >> 8 : word;
      const uint32_t v = t & ((i & 1) ? 0x00F000F0u : 0x000F000Fu);
      return bf16x2_fma(v, (i & 1) ? rc.m1 : rc.m0, rc.m2);
    }
    return bf16x2_mul(int4_pair(word, i), rc.sd);
  }
  // E2M1: codes as value * 2^-126; the multipliers carry 2^126 unless m2
  uint32_t v = e2m1_pair_scaled(word, i);
  if (rc.m2) v = bf16x2_mul(v, kBf16x2Pow126);
  return bf16x2_mul(v, (FMT == MOE_FMT_NVFP4_G16 && j >= 2) ? rc.m1 : rc.m0);
}

// acc[h][4] += W(rows r, r+8; one 128-k block) x activation fragments: the
// MMA steps of a block alternate between two accumulators (h = 0 / 1), so two
// independent dependency chains are in flight instead of one.
template <int FMT, bool FAST>
MOE_DEV void mma_block2(float (&acc)[2][4], const RowChunk& lo, const RowChunk& hi, const uint32_t (&b)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wl = word_of(lo.codes, j), wh = word_of(hi.codes, j);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a[4];
      a[0] = dq<FMT, FAST>(lo, wl, 2 * h, j);
      a[1] = dq<FMT, FAST>(hi, wh, 2 * h, j);
      a[2] = dq<FMT, FAST>(lo, wl, 2 * h + 1, j);
      a[3] = dq<FMT, FAST>(hi, wh, 2 * h + 1, j);
      mma_bf16_16816(acc[h], a, b[2 * j + h][0], b[2 * j + h][1]);
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

// Activation fragments of one lane's 32-k slice (64 bytes at p) of a bf16 row.
// SRC 0: shared memory; 1: global, read-only for the kernel's lifetime
// (ld.global.nc); 2: global, written by an earlier kernel (ld.global.cg).
// With VALID false the fragments are zero (slices past K).
template <int SRC>
MOE_DEV void act_frags(const uint16_t* p, bool valid, uint32_t (&b)[8][2]) {
  uint32_t X[16];
  if (valid) {
    const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w = SRC == 0 ? v[i] : SRC == 1 ? __ldg(v + i) : __ldcg(v + i);
      X[4 * i] = w.x; X[4 * i + 1] = w.y; X[4 * i + 2] = w.z; X[4 * i + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
  act_frags_from_raw(X, b);
}

// One warp's pass over the 128-k blocks b0, b0 + step, ... below nblk_full of
// one 16-row weight tile (rows r and r + 8 of the lane: codes c_lo / c_hi and
// scales sc_lo / sc_hi in shared memory), then the optional block `tail`
// (>= 0) whose lane slices may lie past K.  The next block's weights and first
// token tile's activations are loaded before the current block's math (two
// register buffers, no copies).  `act.load(j, b, in, bf)` gives token tile j's
// fragments of block b.  acc[j][h] are the two accumulator chains of tile j.
template <int FMT, int NT, typename Act>
MOE_DEV void stream_kblocks(float (&acc)[NT][2][4], int b0, int step, int nblk_full, int tail, int K, int q,
                            const uint8_t* c_lo, const uint8_t* c_hi, const uint8_t* sc_lo, const uint8_t* sc_hi,
                            float gsc, int ntiles, const Act& act) {
  auto compute = [&](const RowChunk& lo, const RowChunk& hi, const uint32_t (&f0)[8][2], int b, bool in) {
    // warp-uniform: mma.sync needs the whole warp on one path (the two-step
    // path is exact for every scale)
    const bool fast = __all_sync(0xffffffffu, (lo.fast & hi.fast) != 0u);
    if (fast) mma_block2<FMT, true>(acc[0], lo, hi, f0);
    else mma_block2<FMT, false>(acc[0], lo, hi, f0);
#pragma unroll
    for (int j = 1; j < NT; ++j) {
      if (j >= ntiles) break;
      uint32_t fj[8][2];
      act.load(j, b, in, fj);
      if (fast) mma_block2<FMT, true>(acc[j], lo, hi, fj);
      else mma_block2<FMT, false>(acc[j], lo, hi, fj);
    }
  };
  int b = b0;
  if (b < nblk_full) {
    RowChunk a_lo = row_chunk_at<FMT>(c_lo, sc_lo, b, q, true, gsc);
    RowChunk a_hi = row_chunk_at<FMT>(c_hi, sc_hi, b, q, true, gsc);
    uint32_t fa[8][2];
    act.load(0, b, true, fa);
    for (;;) {
      const int b1 = b + step;
      RowChunk b_lo, b_hi;
      uint32_t fb[8][2];
      if (b1 < nblk_full) {
        b_lo = row_chunk_at<FMT>(c_lo, sc_lo, b1, q, true, gsc);
        b_hi = row_chunk_at<FMT>(c_hi, sc_hi, b1, q, true, gsc);
        act.load(0, b1, true, fb);
      }
      compute(a_lo, a_hi, fa, b, true);
      if (b1 >= nblk_full) break;
      const int b2 = b1 + step;
      if (b2 < nblk_full) {
        a_lo = row_chunk_at<FMT>(c_lo, sc_lo, b2, q, true, gsc);
        a_hi = row_chunk_at<FMT>(c_hi, sc_hi, b2, q, true, gsc);
        act.load(0, b2, true, fa);
      }
      compute(b_lo, b_hi, fb, b1, true);
      if (b2 >= nblk_full) break;
      b = b2;
    }
  }
  if (tail >= 0) {
    const bool in = 128 * tail + 32 * q < K;
    const RowChunk lo = row_chunk_at<FMT>(c_lo, sc_lo, tail, q, in, gsc);
    const RowChunk hi = row_chunk_at<FMT>(c_hi, sc_hi, tail, q, in, gsc);
    uint32_t f0[8][2];
    act.load(0, tail, in, f0);
    compute(lo, hi, f0, tail, in);
  }
}

// Number of 128-k blocks in which lane slice q (k in [kb + 32q, kb + 32q + 32))
// lies inside K (K a multiple of 32).
MOE_DEV int lane_kblocks(int K, int q) { return (K - 32 * q + 127) >> 7; }

// Row stride of bf16 rows of length K staged in shared memory: 16 bytes of
// padding shift consecutive rows by four banks, so the eight rows of an MMA
// fragment load do not all start in the same bank.
__host__ __device__ inline int staged_row_stride(int K) { return 2 * K + 16; }

// Start one bulk copy per bf16 row of length K (rows [lane, lane+32, ...) <
// `rows`) from global `src` into shared memory at `dst` with the padded row
// stride, all completing on `bar`.  Called by every lane of one warp after
// lane 0 announced rows * 2K bytes on `bar`.
MOE_DEV void stage_bf16_rows(uint8_t* dst, const uint16_t* src, int rows, int K, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const int stride = staged_row_stride(K);
  for (int r = lane; r < rows; r += 32) bulk_g2s(dst + size_t(r) * stride, src + size_t(r) * K, uint32_t(2 * K), bar);
}

// Bytes staged for `rows` consecutive weight rows (codes + scales).
template <int FMT>
MOE_DEV uint32_t staged_bytes(const Bank& bk, int rows) {
  return uint32_t(rows) * (bk.K / 2) + uint32_t(rows) * scale_row_bytes(FMT, bk.K);
}

// Start the two bulk copies (codes, scales) of `rows` consecutive weight rows
// of a bank into shared memory, completing on `bar`.  Packed weights are read
// once per launch: they are evicted first from L2.
template <int FMT>
MOE_DEV void stage_rows(const Bank& bk, long row0, int rows, uint8_t* s_codes, uint8_t* s_scales, uint64_t* bar,
                        uint64_t policy) {
  const uint32_t cbytes = uint32_t(rows) * (bk.K / 2);
  const int sb = scale_row_bytes(FMT, bk.K);
  bulk_g2s_hint(s_codes, bk.codes + row0 * (bk.K / 2), cbytes, bar, policy);
  bulk_g2s_hint(s_scales, static_cast<const uint8_t*>(bk.scales) + row0 * sb, uint32_t(rows) * sb, bar, policy);
}

// Prefetch into L2 the codes and scales of `rows` consecutive weight rows.
template <int FMT>
MOE_DEV void prefetch_rows(const Bank& bk, long row0, int rows) {
  const int sb = scale_row_bytes(FMT, bk.K);
  bulk_prefetch_l2(bk.codes + row0 * (bk.K / 2), uint32_t(rows) * (bk.K / 2));
  bulk_prefetch_l2(static_cast<const uint8_t*>(bk.scales) + row0 * sb, uint32_t(rows) * sb);
}

// Shared-memory layout of one staged work unit of `rows` weight rows: codes,
// then scales padded to 16 bytes.
struct UnitLayout {
  int cbytes, sbytes, stage_bytes;
};

__host__ __device__ inline UnitLayout unit_layout(int fmt, int K, int rows) {
  UnitLayout l;
  l.cbytes = rows * (K / 2);
  l.sbytes = rows * scale_row_bytes(fmt, K);
  l.stage_bytes = l.cbytes + ((l.sbytes + 15) & ~15);
  return l;
}

}  // namespace moe
