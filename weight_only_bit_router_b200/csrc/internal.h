// Internal declarations shared by the host dispatcher (api.cu) and the kernel
// translation units.  Nothing here is part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_w4a16.h"

namespace moe {

constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kDecodeMaxT = 32;  // MOE_PATH_AUTO switches to the grouped GEMMs above this

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline size_t bank_codes_bytes(int E, int N, int K) { return size_t(E) * N * (K / 2); }
__host__ __device__ inline int int4_groups(int K) { return (K + 127) / 128; }
inline size_t bank_scale_offset(moe_format_t fmt, int E, int N, int K) {
  (void)fmt;
  return align_up(bank_codes_bytes(E, N, K), 256);
}
inline size_t bank_scale_bytes(moe_format_t fmt, int E, int N, int K) {
  if (fmt == MOE_FMT_INT4_G128) return size_t(E) * N * int4_groups(K) * 2;
  return fmt == MOE_FMT_NVFP4_G16 ? size_t(E) * N * (K / 16) : size_t(E) * N * (K / 32);
}
// NVFP4: the per-matrix fp32 global scales follow the block scales
inline size_t bank_gscale_offset(moe_format_t fmt, int E, int N, int K) {
  return align_up(bank_scale_offset(fmt, E, N, K) + bank_scale_bytes(fmt, E, N, K), 256);
}
inline size_t bank_total_bytes(moe_format_t fmt, int E, int N, int K) {
  if (fmt == MOE_FMT_NVFP4_G16) return bank_gscale_offset(fmt, E, N, K) + size_t(E) * 4;
  return bank_scale_offset(fmt, E, N, K) + bank_scale_bytes(fmt, E, N, K);
}

// The experts a packed bank holds: [lo, hi) of the layer's E (all of them,
// or one expert-parallel shard).  Routing always runs over all E experts.
struct ExpertRange {
  int lo, hi;
};

// Device view of one packed bank.
struct Bank {
  const uint8_t* codes;  // [E][N][K/2]
  const void* scales;    // INT4: bf16 [E][N][G]; MXFP4: u8 [E][N][K/32]; NVFP4: E4M3 u8 [E][N][K/16]
  const float* gscale;   // NVFP4: fp32 [E] per-matrix global scales; null otherwise
  int N, K;
};

// Workspace carve-up for T tokens (all offsets 256-byte aligned).
// The first kStatusBytes of a workspace: the status word and the kernels'
// device counters (small-batch routing completion at int32 index 1).  Zeroed once by moe_workspace_init; every kernel
// that counts leaves its counters at zero when it finishes.
constexpr size_t kStatusBytes = 4096;

struct Workspace {
  uint32_t* status;       // status word (device-side failures)
  int32_t* route_counter; // CTAs done in the one-kernel small-batch routing (shapes outside the split-K form)
  float* logits;          // [T, E]
  int32_t* topk_ids;      // [T, k]
  float* topk_w;          // [T, k]
  int32_t* offsets;       // [E+1]
  int32_t* sorted_rows;   // [T*k]
  int32_t* pos;           // [T*k]
  int32_t* touched;       // [E+1]: number of experts with rows, then their ids ascending
  int32_t* tile_base;     // [E+1]: prefix of per-expert token blocks (grouped GEMMs)
  int32_t* block_hist;    // [nblk, E] per-block expert histograms (large-T permutation)
  uint16_t* act;          // [T*k, I] bf16 SwiGLU output, expert-sorted rows
  float* out_acc;         // [T, H] fp32 combine accumulator (grouped-GEMM path)
  float* ypart;           // [T*k, H] fp32 per-row down outputs (deterministic grouped combine)
  float* route_part;      // [H/256, T, E] fp32 split-K router partials (small-batch routing)
  size_t bytes;
};

// flags: MOE_FLAG_* of the call (the deterministic grouped combine adds the
// per-row output buffer above kDecodeMaxT tokens)
Workspace carve_workspace(void* base, const moe_shape_t& s, int T, uint32_t flags = 0);
size_t permute_block_rows();

// The bf16 shared expert folded into the small-batch kernels (T <= kDecodeMaxT
// with the split-K routing and the decode kernels): its gate_up rows and its
// gate vector are extra rows of the routing GEMV, the gate_up kernel turns
// their split partials into the SwiGLU activation and the sigmoid gate, and
// the down kernel multiplies the activation by its down matrix inside the
// combine.  Null members: no shared expert.
struct SharedFold {
  const uint16_t* w_gate_up;  // [2 I_s, H] bf16 (gate rows, then up rows)
  const uint16_t* w_gate;     // [H] bf16 shared_expert_gate
  const uint16_t* w_down;     // [H, I_s] bf16
  int inter;                  // I_s (a multiple of 64, at most kSharedFoldMaxInter)
  int splits;                 // k-splits of the routing GEMV
  float* h;                   // [splits][T][2 I_s + 1] fp32 partials: gate_up rows, then the gate logit
  uint16_t* a;                // [T, I_s] bf16 SwiGLU activation
  float* g;                   // [T] fp32 sigmoid gate
};
constexpr int kSharedFoldMaxInter = 512;  // the down kernel's four 128-k sub-units

// pack.cu
cudaError_t launch_pack(moe_format_t fmt, const uint16_t* w, int E, int N, int K, void* packed,
                        int32_t* nonfinite, cudaStream_t stream);
// MXFP4 packing with an exponent rule (moe_mx_exp_rule_t as int)
cudaError_t launch_pack_mxfp4_rule(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                                   int rule, cudaStream_t stream);
cudaError_t launch_dequant(moe_format_t fmt, const void* packed, int E, int N, int K, uint16_t* out,
                           cudaStream_t stream);

// route.cu
// Router GEMV + top-k + permutation for T <= kDecodeMaxT: split-K GEMV then
// a one-CTA finalize kernel, or one kernel for other shapes.
// With `sf` (the split-K form only) the GEMV also writes the shared expert's
// partials sf->h.
cudaError_t launch_route_small(const uint16_t* x, const uint16_t* wr, const float* bias, int T, int H, int E, int k,
                               const Workspace& ws, int block_n, cudaStream_t stream,
                               const SharedFold* sf = nullptr);
// the split-K form applies (T <= 32, E <= 256, k <= 8, H <= 2048, E % 4 == 0)
bool route_fast_applies(int T, int H, int E, int k);
// k-splits of its GEMV
int route_gemv_splits(int H);
// split-K partial logits of the small-batch routing kernel (0 when it does not apply)
size_t route_part_bytes(int T, int H, int E, int k);
// kernels launch_route_small launches: 2 (split-K GEMV + finalize) where the
// split-K form applies, else 1
int route_small_launches(int T, int H, int E, int k);
cudaError_t launch_topk(const float* logits, const float* bias, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t stream);
// Small-T permutation (R = T*k <= 1024) in one CTA, with the touched-expert
// list and the token-block prefix.
cudaError_t launch_permute_small(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* sorted_rows,
                                 int32_t* pos, int32_t* touched, int32_t* tile_base, int block_n,
                                 cudaStream_t stream);
// Any-T permutation (three kernels) + tile prefix for the grouped GEMMs.
cudaError_t launch_permute_large(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* sorted_rows,
                                 int32_t* pos, int32_t* block_hist, int32_t* touched, int32_t* tile_base,
                                 int block_n, cudaStream_t stream);
size_t permute_large_hist_bytes(int T, int E, int k);

// decode.cu
// the decode kernels take this shape and token count (T <= kDecodeMaxT and the
// stages fit in shared memory)
bool decode_supported(const moe_shape_t& s, int T);
// ... and with the folded shared expert's products in the down kernel
bool decode_shared_fits(const moe_shape_t& s, int T);
// gate_up + SwiGLU into ws.act; also requests the touched experts' rows of
// the down bank `dn` into L2 for the down kernel that follows; with `sf`
// also the shared expert's activation sf->a and gate sf->g
cudaError_t launch_decode_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu, const Bank& dn,
                                  const ExpertRange& er, const Workspace& ws, cudaStream_t stream,
                                  const SharedFold* sf = nullptr);
// the down products of the bank's experts and the combine: out = bf16(sum
// over each token's slots in slot order of w * y (+ sh_gate[t] * sh_y[t])),
// or the fp32 sum over the bank's experts into partial_out (sh_* nullable);
// with `sf` (bf16 output only) the shared term is g[t] * (W_down a[t]),
// computed here
cudaError_t launch_decode_down(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er,
                               const Workspace& ws, const float* sh_gate, const float* sh_y, uint16_t* out,
                               float* partial_out, cudaStream_t stream, const SharedFold* sf = nullptr);

// gemm_sm100.cu
constexpr int kGemmBN = 128;  // token columns per grouped-GEMM tile
// the grouped GEMMs support the shape (scale rows of a tile fit their staging buffer)
bool grouped_supported(const moe_shape_t& s);
cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* wr, int T, int H, int E, float* logits,
                               uint32_t* status, cudaStream_t stream);
cudaError_t launch_grouped_gate_up(const moe_shape_t& s, int T, const uint16_t* x, const Bank& gu,
                                   const ExpertRange& er, const Workspace& ws, cudaStream_t stream);
// adds the weighted expert outputs into acc [T, H] fp32 (zeroed by the
// caller), or with ypart stores each (token, slot) row's weighted output in
// ypart [T*k, H] (sorted-row order) for combine_rows
cudaError_t launch_grouped_down(const moe_shape_t& s, int T, const Bank& dn, const ExpertRange& er,
                                const Workspace& ws, float* acc, float* ypart, cudaStream_t stream);
// out = bf16(sum over slots in order of ypart rows (+ shared)), or the fp32 sum
// over the range's slots into partial_out
cudaError_t launch_combine_rows(const moe_shape_t& s, int T, const ExpertRange& er, const Workspace& ws,
                                const float* ypart, const float* sh_gate, const float* sh_y, uint16_t* out,
                                float* partial_out, cudaStream_t stream);
// out = bf16(acc [+ sh_gate[t] * sh_y[t][f]]) over [T, H] (sh_* nullable)
cudaError_t launch_finalize_out(const float* acc, int T, int H, const float* sh_gate, const float* sh_y,
                                uint16_t* out, cudaStream_t stream);

// shared.cu: the shared expert's SwiGLU and sigmoid gate from the fp32 gate_up
// product h [T, 2 I_s]: a [T, I_s] bf16, g [T] fp32 (g = sigmoid(x . w_gate))
cudaError_t launch_shared_swiglu_gate(const uint16_t* x, const uint16_t* w_gate, const float* h, int splits, int T,
                                      int H, int I_s, uint16_t* a, float* g, cudaStream_t stream);
// T <= 32: part [splits][T][N] fp32 = W [N][K] x [T][K]^T per 512-k split (N % 16 == 0, K % 64 == 0)
int shared_gemv_splits(int K);
cudaError_t launch_shared_gemv(const uint16_t* x, const uint16_t* w, int T, int K, int N, float* part,
                               cudaStream_t stream);

// selftest of the bounded device-side wait (api.cu)
cudaError_t launch_bounded_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t stream);

// moe_forward's argument checks without the workspace (api.cu)
moe_status_t check_forward_args(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                                const float* logit_bias, const void* gu, const void* dn, uint16_t* out);

// Device address of moe_forward_noalloc's scratch array on the current device
// (noalloc.cu); looked up when the device's context is new to the library,
// which is refused while `stream` is being captured.
cudaError_t noalloc_scratch_address(cudaStream_t stream, void** out);

}  // namespace moe
