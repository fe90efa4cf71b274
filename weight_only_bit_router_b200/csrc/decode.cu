// Decode path (small token counts): weight-streaming expert GEMVs.
//
// The time goes into streaming the touched experts' packed weights from HBM
// ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", Measured: at concurrency 32
// the bottleneck is weight bandwidth).  Each warp owns 16 weight rows and a
// slice of K; a lane loads 16 contiguous bytes (32 codes) per row and 128-k
// block with one 128-bit load, dequantises them to bf16 in registers
// (bf16(q*s) for INT4, e2m1*2^e for MXFP4) and feeds mma.sync m16n8k16 with
// up to 8 tokens per tile.
//
// Fragment k-permutation.  Inside a 128-k block, lane (g = lane/4, q = lane%4)
// owns k in [32q, 32q+32).  For MMA step s = 2*j + h (j = 32-bit code word,
// h = 0/1) the lane's fragment positions {2q, 2q+1, 2q+8, 2q+9} hold
// k0+2h, k0+2h+4, k0+2h+1, k0+2h+5 with k0 = 32q + 8j.  A dot product does not
// depend on the order of its terms, so weights and activations only need the
// same assignment; this one lets one nibble-extraction instruction produce a
// fragment register directly.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kDecWarps = 4;   // warps per CTA
constexpr int kDecRows = 16;   // weight rows (features) per warp tile
constexpr int kDecPF = 4;      // 128-k blocks prefetched per warp at once
constexpr int kDecNT = 4;      // token tiles of 8 held in registers at once

MOE_DEV void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
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

// Per-row dequantisation state for one 128-k block: the 16 code bytes of the
// lane's k-slice and the bf16x2 multiplier (scale, or 2^e for MXFP4).
struct RowChunk {
  uint4 codes;
  uint32_t mult;
};

template <int FMT>
MOE_DEV uint32_t dq_pair(uint32_t word, int i, uint32_t mult) {
  const uint32_t v = (FMT == MOE_FMT_INT4_G128) ? int4_pair(word, i) : e2m1_pair(word, i);
  return bf16x2_mul(v, mult);
}

MOE_DEV uint32_t word_of(const uint4& c, int j) {
  return j == 0 ? c.x : j == 1 ? c.y : j == 2 ? c.z : c.w;
}

// Load one row's 16-byte code chunk and its multiplier for the lane's k-slice
// [kb + 32q, kb + 32q + 32).  Slices past K read as zero weights.
template <int FMT>
MOE_DEV RowChunk load_row_chunk(const Bank& bk, long row, int kb, int q) {
  RowChunk rc;
  const int k = kb + 32 * q;
  if (k < bk.K) {
    rc.codes = ldg_nc_v4(bk.codes + row * (bk.K / 2) + k / 2);
    if (FMT == MOE_FMT_INT4_G128) {
      const uint32_t s = static_cast<const uint16_t*>(bk.scales)[row * int4_groups(bk.K) + k / 128];
      rc.mult = s | (s << 16);
    } else {
      const int e = int(static_cast<const uint8_t*>(bk.scales)[row * (bk.K / 32) + k / 32]) - 127;
      rc.mult = pow2_bf16x2(e);
    }
  } else {
    rc.codes = make_uint4(0, 0, 0, 0);  // INT4 nibble 0 would be -8: zero the multiplier instead
    rc.mult = 0;
  }
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

// acc[4] += W(rows r, r+8; one 128-k block) x act fragments, for one 16-row tile.
template <int FMT>
MOE_DEV void mma_block(float (&acc)[4], const RowChunk& lo, const RowChunk& hi, const uint32_t (&b)[8][2]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wl = word_of(lo.codes, j), wh = word_of(hi.codes, j);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t a[4];
      a[0] = dq_pair<FMT>(wl, 2 * h, lo.mult);
      a[1] = dq_pair<FMT>(wh, 2 * h, hi.mult);
      a[2] = dq_pair<FMT>(wl, 2 * h + 1, lo.mult);
      a[3] = dq_pair<FMT>(wh, 2 * h + 1, hi.mult);
      mma_bf16_16816(acc, a, b[2 * j + h][0], b[2 * j + h][1]);
    }
  }
}

// ---------------------------------------------------------------------------
// gate_up + SwiGLU.  grid = (max experts touched) x (I / 16).  The CTA's 4
// warps split K; partial tiles are summed in shared memory, then
// a = bf16(silu(gate) * up) goes to act[p][f] for the expert's sorted rows p.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(kDecWarps * 32) decode_gate_up_kernel(
    const uint16_t* __restrict__ x, Bank gu, int I, int top_k, const int32_t* __restrict__ touched,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ sorted_rows, uint16_t* __restrict__ act) {
  __shared__ float red[kDecWarps][kDecNT][2][4][32];
  const int ftiles = I / kDecRows;
  const int slot = blockIdx.x / ftiles;
  const int f0 = (blockIdx.x % ftiles) * kDecRows;
  if (slot >= touched[0]) return;
  const int e = touched[1 + slot];
  const int p0 = offsets[e], n_e = offsets[e + 1] - p0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int K = gu.K, N = gu.N;
  const int nblk = (K + 127) / 128;
  const long row_g = long(e) * N + f0 + g;       // gate rows g, g+8
  const long row_u = long(e) * N + I + f0 + g;   // up rows g, g+8
  const int ntiles = (n_e + 7) / 8;

  for (int nt0 = 0; nt0 < ntiles; nt0 += kDecNT) {
    float acc[kDecNT][2][4];
#pragma unroll
    for (int j = 0; j < kDecNT; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[j][t][i] = 0.f;
    // token row of this lane in each of the tiles
    const uint16_t* xrow[kDecNT];
    bool xval[kDecNT];
#pragma unroll
    for (int j = 0; j < kDecNT; ++j) {
      const int c = (nt0 + j) * 8 + g;
      xval[j] = c < n_e;
      xrow[j] = x + size_t(xval[j] ? sorted_rows[p0 + c] / top_k : 0) * K;
    }
    for (int b0 = warp; b0 < nblk; b0 += kDecWarps * kDecPF) {
      RowChunk cg[kDecPF][2], cu[kDecPF][2];
#pragma unroll
      for (int u = 0; u < kDecPF; ++u) {
        const int kb = (b0 + u * kDecWarps) * 128;
        const bool ok = kb < K;
        cg[u][0] = load_row_chunk<FMT>(gu, row_g, ok ? kb : K, q);
        cg[u][1] = load_row_chunk<FMT>(gu, row_g + 8, ok ? kb : K, q);
        cu[u][0] = load_row_chunk<FMT>(gu, row_u, ok ? kb : K, q);
        cu[u][1] = load_row_chunk<FMT>(gu, row_u + 8, ok ? kb : K, q);
      }
#pragma unroll
      for (int u = 0; u < kDecPF; ++u) {
        const int kb = (b0 + u * kDecWarps) * 128;
        if (kb >= K) break;
#pragma unroll
        for (int j = 0; j < kDecNT; ++j) {
          if (nt0 + j >= ntiles) break;
          uint32_t bf[8][2];
          load_act_frags(xrow[j], K, kb, q, xval[j], bf);
          mma_block<FMT>(acc[j][0], cg[u][0], cg[u][1], bf);
          mma_block<FMT>(acc[j][1], cu[u][0], cu[u][1], bf);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kDecNT; ++j)
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp][j][t][i][lane] = acc[j][t][i];
    __syncthreads();
    // warp w finishes token tile nt0 + w
    const int j = warp;
    if (nt0 + j < ntiles) {
      float gsum[4], usum[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        gsum[i] = 0.f;
        usum[i] = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
          gsum[i] += red[w][j][0][i][lane];
          usum[i] += red[w][j][1][i][lane];
        }
      }
      // c0,c1: feature g, tokens 2q, 2q+1; c2,c3: feature g+8
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = (nt0 + j) * 8 + 2 * q + (i & 1);
        const int f = f0 + g + ((i >> 1) << 3);
        if (col < n_e) act[size_t(p0 + col) * I + f] = f32_to_bf16_rn(silu_mul(gsum[i], usum[i]));
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// down projection.  grid = (max experts touched) x (H / 64): each warp owns 16
// output features over the whole K = I; y[p][f] is written in fp32.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(kDecWarps * 32) decode_down_kernel(
    Bank dn, const int32_t* __restrict__ touched, const int32_t* __restrict__ offsets,
    const uint16_t* __restrict__ act, float* __restrict__ y) {
  const int H = dn.N, K = dn.K;  // K = I
  const int ftiles = H / (kDecRows * kDecWarps);
  const int slot = blockIdx.x / ftiles;
  if (slot >= touched[0]) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int f0 = (blockIdx.x % ftiles) * (kDecRows * kDecWarps) + warp * kDecRows;
  const int e = touched[1 + slot];
  const int p0 = offsets[e], n_e = offsets[e + 1] - p0;
  const int nblk = (K + 127) / 128;
  const long row = long(e) * H + f0 + g;
  const int ntiles = (n_e + 7) / 8;
  for (int nt0 = 0; nt0 < ntiles; nt0 += kDecNT) {
    float acc[kDecNT][4];
#pragma unroll
    for (int j = 0; j < kDecNT; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
    for (int b0 = 0; b0 < nblk; b0 += kDecPF) {
      RowChunk c[kDecPF][2];
#pragma unroll
      for (int u = 0; u < kDecPF; ++u) {
        const int kb = (b0 + u) * 128;
        c[u][0] = load_row_chunk<FMT>(dn, row, kb < K ? kb : K, q);
        c[u][1] = load_row_chunk<FMT>(dn, row + 8, kb < K ? kb : K, q);
      }
#pragma unroll
      for (int u = 0; u < kDecPF; ++u) {
        const int kb = (b0 + u) * 128;
        if (kb >= K) break;
#pragma unroll
        for (int j = 0; j < kDecNT; ++j) {
          if (nt0 + j >= ntiles) break;
          const int col = (nt0 + j) * 8 + g;
          uint32_t bf[8][2];
          load_act_frags(act + size_t(p0 + (col < n_e ? col : 0)) * K, K, kb, q, col < n_e, bf);
          mma_block<FMT>(acc[j], c[u][0], c[u][1], bf);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kDecNT; ++j) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = (nt0 + j) * 8 + 2 * q + (i & 1);
        const int f = f0 + g + ((i >> 1) << 3);
        if (nt0 + j < ntiles && col < n_e) y[size_t(p0 + col) * H + f] = acc[j][i];
      }
    }
  }
}

// out[t][h] = bf16(sum_j w[t][j] * y[pos[t*k+j]][h]), slots in order j = 0..k-1.
__global__ void decode_combine_kernel(const float* __restrict__ y, const float* __restrict__ w,
                                      const int32_t* __restrict__ pos, int T, int H, int k,
                                      uint16_t* __restrict__ out) {
  const long i = long(blockIdx.x) * blockDim.x + threadIdx.x;  // one thread per 4 outputs
  const long n4 = long(T) * H / 4;
  if (i >= n4) return;
  const int t = int(i / (H / 4));
  const int h = int(i % (H / 4)) * 4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int p = pos[size_t(t) * k + j];
    if (p < 0) continue;
    const float wj = w[size_t(t) * k + j];
    const float4 v = *reinterpret_cast<const float4*>(y + size_t(p) * H + h);
    s.x = fmaf(wj, v.x, s.x);
    s.y = fmaf(wj, v.y, s.y);
    s.z = fmaf(wj, v.z, s.z);
    s.w = fmaf(wj, v.w, s.w);
  }
  uint2 o;
  o.x = pack_bf16x2(s.x, s.y);
  o.y = pack_bf16x2(s.z, s.w);
  *reinterpret_cast<uint2*>(out + size_t(t) * H + h) = o;
}

int max_touched(int T, int k, int E) { return (long(T) * k < E) ? T * k : E; }

}  // namespace

cudaError_t launch_decode_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu,
                                  const Workspace& ws, cudaStream_t stream) {
  const int slots = max_touched(T, s.top_k, s.num_experts);
  const int grid = slots * (s.inter / kDecRows);
  if (grid == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128)
    decode_gate_up_kernel<MOE_FMT_INT4_G128><<<grid, kDecWarps * 32, 0, stream>>>(
        x, gu, s.inter, s.top_k, ws.touched, ws.offsets, ws.sorted_rows, ws.act);
  else
    decode_gate_up_kernel<MOE_FMT_MXFP4_G32><<<grid, kDecWarps * 32, 0, stream>>>(
        x, gu, s.inter, s.top_k, ws.touched, ws.offsets, ws.sorted_rows, ws.act);
  return cudaGetLastError();
}

cudaError_t launch_decode_down(const moe_shape_t& s, int T, const Bank& dn, const Workspace& ws,
                               cudaStream_t stream) {
  const int slots = max_touched(T, s.top_k, s.num_experts);
  const int grid = slots * (s.hidden / (kDecRows * kDecWarps));
  if (grid == 0) return cudaSuccess;
  if (s.fmt == MOE_FMT_INT4_G128)
    decode_down_kernel<MOE_FMT_INT4_G128><<<grid, kDecWarps * 32, 0, stream>>>(dn, ws.touched, ws.offsets,
                                                                                ws.act, ws.y);
  else
    decode_down_kernel<MOE_FMT_MXFP4_G32><<<grid, kDecWarps * 32, 0, stream>>>(dn, ws.touched, ws.offsets,
                                                                                ws.act, ws.y);
  return cudaGetLastError();
}

cudaError_t launch_decode_combine(const moe_shape_t& s, int T, const Workspace& ws, uint16_t* out,
                                  cudaStream_t stream) {
  const long n4 = long(T) * s.hidden / 4;
  if (n4 == 0) return cudaSuccess;
  const int block = 256;
  decode_combine_kernel<<<unsigned((n4 + block - 1) / block), block, 0, stream>>>(ws.y, ws.topk_w, ws.pos, T,
                                                                                  s.hidden, s.top_k, out);
  return cudaGetLastError();
}

}  // namespace moe
