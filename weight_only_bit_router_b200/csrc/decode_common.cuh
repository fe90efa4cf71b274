// Device helpers of the decode (small-batch) expert kernels: mma.sync
// m16n8k16 on dequantised 4-bit weight fragments, the fragment k-permutation
// shared by weights and activations, and the bulk-copy staging of packed rows.
//
// Fragment k-permutation.  Inside a 128-k block, lane (g = lane/4, q = lane%4)
// owns k in [32q, 32q+32).  For MMA step s = 2*j + h (j = 32-bit code word,
// h = 0/1) the lane's fragment positions {2q, 2q+1, 2q+8, 2q+9} hold
// k0+2h, k0+2h+4, k0+2h+1, k0+2h+5 with k0 = 32q + 8j.  A dot product does not
// depend on the order of its terms, so weights and activations only need the
// same assignment; this one lets one nibble-extraction instruction produce a
// fragment register directly.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kDecWarps = 4;       // warps per CTA
constexpr int kDecRows = 16;       // weight rows (features) per warp tile
constexpr int kDecNT = 4;          // token tiles of 8 held in registers at once

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

// One bf16 pair (nibbles i, i+4 of `word`) times its multiplier.  E2M1 codes
// enter as value * 2^-126 (e2m1_pair_scaled) and `mult` carries the 2^126
// unless `two` is set, in which case the codes are first scaled back.
template <int FMT>
MOE_DEV uint32_t dq_pair(uint32_t word, int i, uint32_t mult, uint32_t two = 0) {
  if (FMT == MOE_FMT_INT4_G128) return bf16x2_mul(int4_pair(word, i), mult);
  uint32_t v = e2m1_pair_scaled(word, i);
  if (two) v = bf16x2_mul(v, kBf16x2Pow126);
  return bf16x2_mul(v, mult);
}

// MXFP4 multiplier of exponent e for dq_pair: 2^(e + 126) when that is a
// bf16 value (e <= 1), else 2^e with the two-step flag.
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

// One row's 16 code bytes for the lane's k-slice [kb + 32q, kb + 32q + 32) and
// the bf16x2 multiplier (scale, or 2^e for MXFP4), read from shared memory.
// Slices past K read as zero weights.
struct RowChunk {
  uint4 codes;
  uint32_t mult;   // bf16x2 multiplier: the INT4 scale, 2^e for MXFP4, or (NVFP4) the first 16-block's
  uint32_t mult2;  // NVFP4: the second 16-block's multiplier (code words 2 and 3); otherwise = mult
  uint32_t two;    // E2M1 formats: 1 if the multipliers do not carry the 2^126 (see dq_pair)
};

template <int FMT>
MOE_DEV RowChunk smem_row_chunk(const uint8_t* codes, const uint8_t* scales, int r, int K, int kb, int q) {
  static_assert(FMT != MOE_FMT_NVFP4_G16, "NVFP4 chunks come from row_chunk_at");
  RowChunk rc;
  const int k = kb + 32 * q;
  if (k < K) {
    rc.codes = *reinterpret_cast<const uint4*>(codes + r * (K / 2) + k / 2);
    if (FMT == MOE_FMT_INT4_G128) {
      const uint32_t s = reinterpret_cast<const uint16_t*>(scales)[r * int4_groups(K) + k / 128];
      rc.mult = s | (s << 16);
      rc.two = 0;
    } else {
      mx_mult(int(scales[r * (K / 32) + k / 32]) - 127, rc.mult, rc.two);
    }
  } else {
    rc.codes = make_uint4(0, 0, 0, 0);  // INT4 nibble 0 would be -8: zero the multiplier instead
    rc.mult = 0;
    rc.two = 0;
  }
  rc.mult2 = rc.mult;
  return rc;
}

// Activation fragments of one 128-k block for one token row: 16 words X[m] =
// (v[32q+2m], v[32q+2m+1]), permuted into the (k0+2h, k0+2h+4) / (k0+2h+1,
// k0+2h+5) pairs of the 8 MMA steps.
MOE_DEV void load_act_frags(const uint16_t* rowp, int K, int kb, int q, bool valid, uint32_t (&b)[8][2]) {
  uint32_t X[16];
  const int k = kb + 32 * q;
  if (valid && k < K) {
    const uint4* p = reinterpret_cast<const uint4*>(rowp + k);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = __ldg(p + i);
      X[4 * i] = v.x; X[4 * i + 1] = v.y; X[4 * i + 2] = v.z; X[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    b[2 * j][0] = prmt(X[4 * j], X[4 * j + 2], 0x5410u);
    b[2 * j][1] = prmt(X[4 * j], X[4 * j + 2], 0x7632u);
    b[2 * j + 1][0] = prmt(X[4 * j + 1], X[4 * j + 3], 0x5410u);
    b[2 * j + 1][1] = prmt(X[4 * j + 1], X[4 * j + 3], 0x7632u);
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

// Activation fragments of one 128-k block for one token row held in shared
// memory: `p` points at the lane's 64-byte k-slice (row + 2 * (kb + 32q));
// same layout and permutation as load_act_frags.  Plain loads, so that the
// compiler orders them after the barrier waits that make the data visible.
MOE_DEV void load_act_frags_smem(const uint8_t* p, bool valid, uint32_t (&b)[8][2]) {
  uint32_t X[16];
  if (valid) {
    const uint4* v = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w = v[i];
      X[4 * i] = w.x; X[4 * i + 1] = w.y; X[4 * i + 2] = w.z; X[4 * i + 3] = w.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
  act_frags_from_raw(X, b);
}

// A lane's 16 code bytes and multiplier(s) of k-block b of one staged weight
// row: `codes` points at the row's codes plus the lane's slice offset 16q,
// `scales` at the row's scales; `in` is false for a slice past K (zero
// weights); `g` is the matrix's NVFP4 global scale (unused otherwise).
template <int FMT>
MOE_DEV RowChunk row_chunk_at(const uint8_t* codes, const uint8_t* scales, int b, int q, bool in, float g = 0.f) {
  RowChunk rc;
  if (in) {
    rc.codes = *reinterpret_cast<const uint4*>(codes + 64 * b);
    if (FMT == MOE_FMT_INT4_G128) {
      const uint32_t sc = reinterpret_cast<const uint16_t*>(scales)[b];  // group b = k-block b
      rc.mult = sc | (sc << 16);
      rc.mult2 = rc.mult;
      rc.two = 0;
    } else if (FMT == MOE_FMT_NVFP4_G16) {
      // the slice holds two 16-element blocks: 8b + 2q and 8b + 2q + 1
      nv_mult_pair_scaled(scales + 8 * b + 2 * q, g, rc.mult, rc.mult2, rc.two);
    } else {
      mx_mult(int(scales[4 * b + q]) - 127, rc.mult, rc.two);  // the slice is one 32-element block
      rc.mult2 = rc.mult;
    }
  } else {
    rc.codes = make_uint4(0, 0, 0, 0);
    rc.mult = 0;
    rc.mult2 = 0;
    rc.two = 0;
  }
  return rc;
}

// Number of 128-k blocks in which lane slice q (k in [kb + 32q, kb + 32q + 32))
// lies inside K (K a multiple of 32).
MOE_DEV int lane_kblocks(int K, int q) { return (K - 32 * q + 127) >> 7; }

// Row stride of bf16 activation rows of length K staged in shared memory:
// 16 bytes of padding shift consecutive rows by four banks, so the eight rows
// of an MMA fragment load do not all start in the same bank.
__host__ __device__ inline int staged_row_stride(int K) { return 2 * K + 16; }

// Start one bulk copy per bf16 row of length K (rows [lane, lane+32, ...) <
// `rows`) from global `src` into shared memory at `dst` with the padded row
// stride, all completing on `bar`.  Called by every lane of one warp after
// lane 0 announced rows * 2K bytes on `bar`.
MOE_DEV void stage_act_rows(uint8_t* dst, const uint16_t* src, int rows, int K, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const int stride = staged_row_stride(K);
  for (int r = lane; r < rows; r += 32) bulk_g2s(dst + size_t(r) * stride, src + size_t(r) * K, uint32_t(2 * K), bar);
}

// The 16 raw activation words of one 128-k block for the lane's k-slice,
// read through L2 (ld.global.cg): for data that other CTAs of the same grid
// wrote.  Rows past K, or an invalid row, read as zeros.
MOE_DEV void load_act_raw_cg(const uint16_t* rowp, int K, int kb, int q, bool valid, uint32_t (&X)[16]) {
  const int k = kb + 32 * q;
  if (valid && k < K) {
    const uint4* p = reinterpret_cast<const uint4*>(rowp + k);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = __ldcg(p + i);
      X[4 * i] = v.x; X[4 * i + 1] = v.y; X[4 * i + 2] = v.z; X[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) X[i] = 0;
  }
}

// One bf16 pair (nibbles i, i+4 of code word j) of a row chunk.
template <int FMT>
MOE_DEV uint32_t dq(const RowChunk& rc, uint32_t word, int i, int j = 0) {
  return dq_pair<FMT>(word, i, (FMT == MOE_FMT_NVFP4_G16 && j >= 2) ? rc.mult2 : rc.mult, rc.two);
}

// acc[4] += W(rows r, r+8; one 128-k block) x activation fragments.
template <int FMT>
MOE_DEV void mma_block(float (&acc)[4], const RowChunk& lo, const RowChunk& hi, const uint32_t (&b)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wl = word_of(lo.codes, j), wh = word_of(hi.codes, j);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a[4];
      a[0] = dq<FMT>(lo, wl, 2 * h, j);
      a[1] = dq<FMT>(hi, wh, 2 * h, j);
      a[2] = dq<FMT>(lo, wl, 2 * h + 1, j);
      a[3] = dq<FMT>(hi, wh, 2 * h + 1, j);
      mma_bf16_16816(acc, a, b[2 * j + h][0], b[2 * j + h][1]);
    }
  }
}

// Bytes staged for `rows` consecutive weight rows (codes + scales).
template <int FMT>
MOE_DEV uint32_t staged_bytes(const Bank& bk, int rows) {
  return uint32_t(rows) * (bk.K / 2) + uint32_t(rows) * scale_row_bytes(FMT, bk.K);
}

// Start the two bulk copies (codes, scales) of `rows` consecutive weight rows
// of a bank into shared memory, completing on `bar`.  The caller has already
// announced the total bytes with ONE arrive.expect_tx on `bar`.
template <int FMT>
MOE_DEV void stage_rows(const Bank& bk, long row0, int rows, uint8_t* s_codes, uint8_t* s_scales, uint64_t* bar) {
  const uint32_t cbytes = uint32_t(rows) * (bk.K / 2);
  const int sb = scale_row_bytes(FMT, bk.K);
  // packed weights are read once per launch: evict them first from L2
  const uint64_t policy = l2_policy_evict_first();
  bulk_g2s_hint(s_codes, bk.codes + row0 * (bk.K / 2), cbytes, bar, policy);
  bulk_g2s_hint(s_scales, static_cast<const uint8_t*>(bk.scales) + row0 * sb, uint32_t(rows) * sb, bar, policy);
}

// Per-stage shared-memory layout of a work unit: codes then scales, each
// matrix slice 16-byte aligned.
struct UnitLayout {
  int cbytes, sbytes, sbytes_pad, stage_bytes;
};

MOE_DEV UnitLayout unit_layout(int fmt, int K, int rows, int mats) {
  UnitLayout l;
  l.cbytes = rows * (K / 2);
  l.sbytes = rows * scale_row_bytes(fmt, K);
  l.sbytes_pad = (l.sbytes + 15) & ~15;
  l.stage_bytes = mats * (l.cbytes + l.sbytes_pad);
  return l;
}

}  // namespace moe
