/*
 * moe_w4a16.h - C ABI of the B200 (sm_100a) weight-only 4-bit routed-expert
 * MoE layer (W4A16: 4-bit expert weights, bf16 activations).
 *
 * The operation is the forward pass of one Qwen3.5-MoE expert layer:
 *
 *   logits = x Wr^T (+ bias)                     router, fp32
 *   ids, w = top-k(logits), softmax over the k   per token
 *   h      = W_gate_up[e] x_t                    per (token, slot), e = ids
 *   a      = bf16(silu(h[0:I]) * h[I:2I])        SwiGLU
 *   y      = W_down[e] a
 *   out_t  = sum_j w_tj y_tj                     bf16 output
 *
 * Sources (model cards of quantised builds of one 35B MoE model):
 *   "Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe: routed experts INT4,
 *     symmetric, group 128, round-to-nearest with min-max scales; the fused
 *     banks experts.gate_up_proj [256, 1024, 2048] (gate rows then up rows)
 *     and experts.down_proj [256, 2048, 512]; routers stay bf16.
 *   "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Model summary and
 *     Quantization method: MXFP4 W4A16 experts (E2M1 codes, one E8M0 scale
 *     per 32 elements, exponents of the floor(log2(x / 6)) family).
 *   "cbert33/Nex-N2.5-mini-FP8-Calibrated", Artifact summary: 256 routed
 *     experts per layer, 8 active per token.
 * Where the cards are silent the library takes the plain reading documented
 * at each entry point (softmax top-k renormalised, SwiGLU, ties to the lower
 * expert index).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major,
 *     16-byte aligned unless stated.  bf16 tensors are passed as uint16_t
 *     bit patterns.
 *   - Nothing allocates device memory: scratch comes from a caller-provided
 *     workspace whose size a query function returns.
 *   - Calls only enqueue work on `stream` (asynchronous, no host sync); the
 *     only process-wide state is a set of thread-safe caches of launch
 *     parameters (SM count, occupancy, kernel attributes), so calls are
 *     reentrant across host threads and streams as long as workspaces are not
 *     shared.  (moe_workspace_status synchronises its stream; the no-alloc
 *     entry point shares one scratch array, see there.)
 *   - Argument errors are detected on the host before anything is enqueued
 *     and leave every output untouched.
 */
#ifndef MOE_W4A16_H
#define MOE_W4A16_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

/* Exported symbol marker (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED = 2,   /* shape outside the supported envelope (see moe_shape_t) */
  MOE_ERR_WORKSPACE = 3,     /* workspace null or smaller than the query returned */
  MOE_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed */
  MOE_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired (reported by moe_workspace_status) */
  MOE_ERR_NONFINITE = 6      /* NaN/Inf met while packing (reported through the count pointer) */
} moe_status_t;

typedef enum {
  MOE_FMT_INT4_G128 = 1,     /* INT4 symmetric RTN, bf16 scale per 128 elements along K */
  MOE_FMT_MXFP4_G32 = 2,     /* MXFP4: E2M1 codes, E8M0 scale per 32 elements along K */
  MOE_FMT_NVFP4_G16 = 3      /* NVFP4: E2M1 codes, E4M3 scale per 16 elements along K, fp32 scale per matrix */
} moe_format_t;

/* Layer shape.  Supported: hidden and inter multiples of 64 (>= 64),
 * 1 <= top_k <= 32, top_k <= num_experts <= 1024. */
typedef struct {
  int hidden;          /* H */
  int inter;           /* I, expert intermediate size; gate_up bank is [E, 2I, H] */
  int num_experts;     /* E */
  int top_k;           /* k */
  moe_format_t fmt;    /* format of both expert banks */
} moe_shape_t;

/* Returns a static, NUL-terminated description of a status code. */
MOE_API const char* moe_status_str(moe_status_t status);

/* Returns MOE_ABI_VERSION of the loaded library. */
MOE_API int moe_abi_version(void);

/* ------------------------------------------------------------------------
 * Packed bank layout
 *
 * A packed bank of E matrices [N, K] is ONE buffer:
 *   bytes [0, E*N*K/2)          codes, [E][N][K/2]: element 2j of a row in the
 *                               low nibble of byte j, element 2j+1 in the high
 *                               nibble.  INT4: offset binary q + 8 (q in
 *                               [-8, 7]).  MXFP4: sign<<3 | E2M1 magnitude code.
 *                               NVFP4: the same E2M1 nibbles as MXFP4.
 *   bytes [scale_offset, ...)   scales.  INT4: bf16 [E][N][ceil(K/128)] (the
 *                               last group of a row holds K mod 128 elements).
 *                               MXFP4: E8M0 uint8 [E][N][K/32], byte = e + 127.
 *                               NVFP4: E4M3 uint8 [E][N][K/16].
 *   NVFP4 only: fp32 [E] global scales (one per matrix; for a gate_up bank the
 *                               gate and up halves of an expert share it) at
 *                               scale_offset + E*N*K/16 rounded up to 256 bytes.
 * scale_offset is E*N*K/2 rounded up to 256 bytes; the total is what
 * moe_bank_bytes returns.
 * ---------------------------------------------------------------------- */

/* Total bytes of a packed bank of E matrices [N, K]; 0 if the arguments are invalid. */
MOE_API size_t moe_bank_bytes(moe_format_t fmt, int E, int N, int K);

/* Byte offset of the scale plane inside a packed bank; 0 if invalid. */
MOE_API size_t moe_bank_scale_offset(moe_format_t fmt, int E, int N, int K);

/* Bytes of the packed gate_up bank (which = 0, [E, 2I, H]) or down bank
 * (which = 1, [E, H, I]) of a layer; 0 if invalid. */
MOE_API size_t moe_packed_bytes(const moe_shape_t* shape, int which);

/* ------------------------------------------------------------------------
 * Packing (offline step, bandwidth-bound)
 * ---------------------------------------------------------------------- */

/* Quantise a bf16 bank w [E, N, K] (device) to INT4 symmetric RTN with one
 * bf16 scale per 128 consecutive K elements of a row
 * ("Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe):
 *   s = bf16_rne(fp32(amax) / 7)          (the group max maps to +-7)
 *   q = clamp(rint_half_even(fp32(w / s)), -8, 7), q = 0 when s == 0.
 * K must be a positive multiple of 32; N, E >= 1.  Writes moe_bank_bytes()
 * bytes at `packed` (device, 256-byte aligned).  If `nonfinite_count`
 * (device int32, nullable) is given, the number of NaN/Inf inputs is ADDED
 * to it; such elements produce unspecified codes. */
MOE_API moe_status_t moe_pack_int4_g128(const uint16_t* w, int E, int N, int K, void* packed,
                                int32_t* nonfinite_count, cudaStream_t stream);

/* Quantise a bf16 bank w [E, N, K] to MXFP4 ("kirillbilchenko/Nex-N2.5-mini-
 * MXFP4-MxWave", Model summary and Quantization method), per block of 32
 * consecutive K elements:
 *   e = floor(log2(amax / 6)) clamped to [-127, 127] (-127 when amax == 0),
 *   scale byte e + 127; code = nearest E2M1 magnitude of |w| / 2^e (ties to
 *   the even code, saturating at 6), sign bit set only for nonzero codes.
 * Same arguments and errors as moe_pack_int4_g128. */
MOE_API moe_status_t moe_pack_mxfp4(const uint16_t* w, int E, int N, int K, void* packed,
                            int32_t* nonfinite_count, cudaStream_t stream);

/* Exponent rules of the MXFP4 packer (all members of the floor(log2(x / 6))
 * family of "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Quantization
 * method), per block of 32 with amax = max |w| (amax == 0 always gives
 * e = -127 and zero codes; every e is clamped to [-127, 127]):
 *   MOE_MX_EXP_FLOOR  e = floor(log2(amax / 6)): largest e with 6 * 2^e <=
 *                     amax (the block max may clip to 6 * 2^e); this is what
 *                     moe_pack_mxfp4 uses.
 *   MOE_MX_EXP_CEIL   e = ceil(log2(amax / 6)): smallest e with amax <=
 *                     6 * 2^e (nothing clips; the card's "smallest exponent
 *                     that avoids clipping").
 *   MOE_MX_EXP_OCP    e = floor(log2(amax)) - 2 (2 = largest E2M1 exponent).
 *   MOE_MX_EXP_MSE    the card's scale search: candidates e0 - 4 ... e0 + 1
 *                     with e0 = floor(log2(p / 6)), p the block's 99.5th
 *                     percentile of |w| (v30 + 0.845 * (v31 - v30) of the
 *                     sorted magnitudes, fp64, multiply rounded before the
 *                     add), plus the CEIL exponent; the candidate with the
 *                     smallest sum of squared reconstruction errors wins (fp64,
 *                     squares of exact differences summed pairwise: element i
 *                     with i + 16, then i + 8, i + 4, i + 2, i + 1), ties to
 *                     the smaller exponent. */
typedef enum {
  MOE_MX_EXP_FLOOR = 0,
  MOE_MX_EXP_CEIL = 1,
  MOE_MX_EXP_OCP = 2,
  MOE_MX_EXP_MSE = 3
} moe_mx_exp_rule_t;

/* moe_pack_mxfp4 with the given exponent rule (codes are always the nearest
 * E2M1 magnitude of |w| / 2^e, ties to the even code, saturating at 6).  The
 * packed layout is the same for every rule, so moe_forward consumes any of
 * them.  Same arguments and errors as moe_pack_int4_g128, plus
 * MOE_ERR_INVALID_ARG for an unknown rule. */
MOE_API moe_status_t moe_pack_mxfp4_rule(const uint16_t* w, int E, int N, int K, void* packed,
                                 int32_t* nonfinite_count, moe_mx_exp_rule_t rule, cudaStream_t stream);

/* Quantise a bf16 bank w [E, N, K] to NVFP4 with bf16 block multipliers
 * (W4A16) ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", What's quantized to
 * what: NVFP4 experts with group 16, one weight_global_scale per expert shared
 * by gate and up, weights-only round-to-nearest).  Per matrix e (all N rows,
 * the gate and up halves of a gate_up bank together):
 *   g    = fp32(amax_e / 2688)            (2688 = 6 * 448: the largest E2M1
 *                                          times the largest E4M3 value)
 * per block of 16 consecutive K elements of a row:
 *   code = E4M3 nearest to fp32(amax_b / fp32(6 g)), ties to even, saturating
 *          at 448
 *   d    = bf16_rne(fp32(e4m3(code) * g)) the block's multiplier
 *   c    = nearest E2M1 magnitude of fp32(w / d) (ties to the even code,
 *          saturating at 6), sign bit only for nonzero codes; 0 when d == 0
 * and the forward pass dequantises w = bf16_rne(e2m1(c) * d).  K must be a
 * positive multiple of 32.  The call enqueues four kernels (matrix maxima,
 * global scales, codes); otherwise arguments and errors as
 * moe_pack_int4_g128. */
MOE_API moe_status_t moe_pack_nvfp4(const uint16_t* w, int E, int N, int K, void* packed,
                            int32_t* nonfinite_count, cudaStream_t stream);

/* Expand a packed bank back to bf16 w_out [E, N, K] (device):
 * INT4 w = bf16_rne(q * s); MXFP4 w = e2m1(c) * 2^e (exact); NVFP4
 * w = bf16_rne(e2m1(c) * d).  Debug and test
 * entry; the forward pass dequantises inside its GEMMs instead. */
MOE_API moe_status_t moe_dequant(const void* packed, moe_format_t fmt, int E, int N, int K,
                         uint16_t* w_out, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Routing
 * ---------------------------------------------------------------------- */

/* Top-k routing of fp32 logits [T, E] (+ optional fp32 bias [E], nullable)
 * ("cbert33/Nex-N2.5-mini-FP8-Calibrated", Artifact summary: 8 of 256
 * experts active).  Per token: the k largest biased logits, equal values
 * ordered by the lower expert index, written in that order to topk_ids
 * [T, k] (int32); topk_w [T, k] (fp32) = exp(l_j - l_max) / sum over the
 * selected k (the softmax over all experts renormalised over the top-k).
 * T >= 0 (T == 0 is a no-op), 1 <= k <= min(32, E), E <= 1024.
 * No 16-byte alignment requirement (4-byte alignment suffices). */
MOE_API moe_status_t moe_route(const float* logits, const float* bias, int T, int E, int k,
                       int32_t* topk_ids, float* topk_w, cudaStream_t stream);

/* Workspace bytes moe_permute needs for T tokens. */
MOE_API size_t moe_permute_workspace_bytes(int T, int E, int k);

/* Stable counting sort of the flat (token, slot) rows r = t*k + j by expert
 * id (topk_ids [T, k], values in [0, E)):
 *   offsets [E+1]      offsets[e] = number of rows with expert < e
 *   sorted_rows [T*k]  rows of expert e at [offsets[e], offsets[e+1]) in
 *                      ascending r
 *   pos [T*k]          inverse permutation: sorted_rows[pos[r]] = r.
 * Ids outside [0, E) are a contract violation (results unspecified, no
 * out-of-bounds access). */
MOE_API moe_status_t moe_permute(const int32_t* topk_ids, int T, int E, int k, int32_t* offsets,
                         int32_t* sorted_rows, int32_t* pos, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Layer forward
 * ---------------------------------------------------------------------- */

typedef enum {
  MOE_PATH_AUTO = 0,      /* decode path for T <= 32, grouped tcgen05 GEMMs above */
  MOE_PATH_DECODE = 1,    /* weight-streaming GEMV kernels (any T; meant for T <= 32: above that
                             the down projection re-streams its weights per 32 tokens) */
  MOE_PATH_PREFILL = 2    /* grouped tcgen05 GEMMs (any T >= 1) */
} moe_path_t;

/* Number of timed stages moe_forward reports through stage_events. */
#define MOE_NUM_STAGES 5
/* Stage ids: 0 router logits, 1 top-k + permutation, 2 gate_up + SwiGLU,
 * 3 down projection, 4 weighted combine / output conversion.  Where one
 * kernel does two stages (small batches: routing and permutation in one; the
 * decode path's down projection and combine in one) the second stage's
 * events bracket nothing and it reads zero. */

/* Optional extras of moe_forward / moe_forward_routed.  Every pointer may be
 * NULL; a NULL opts pointer means all defaults. */
typedef struct {
  moe_path_t path;
  int32_t* topk_ids_out;     /* [T, k]  routing ids (moe_forward only) */
  float* topk_w_out;         /* [T, k]  routing weights (moe_forward only) */
  float* logits_out;         /* [T, E]  fp32 router logits, before the bias */
  int32_t* offsets_out;      /* [E+1]   per-expert row offsets */
  int32_t* sorted_rows_out;  /* [T*k]   expert-sorted rows */
  uint16_t* act_out;         /* [T*k, I] bf16 SwiGLU activations, expert-sorted rows */
  uint32_t flags;            /* MOE_FLAG_* bits (0: defaults) */
  cudaEvent_t* stage_events; /* [2*MOE_NUM_STAGES]: recorded before / after each stage
                                (as external event nodes when the stream is being
                                captured into a CUDA graph) */
} moe_forward_opts_t;

/* moe_forward_opts_t.flags: MOE_FLAG_DETERMINISTIC makes the grouped path's
 * combine run-to-run deterministic: every (token, slot) row's weighted expert
 * output is stored in its own fp32 row and each token's k rows are summed in
 * slot order, instead of being added into the output accumulator in arrival
 * order.  It needs the larger workspace of moe_workspace_bytes_flags.  The
 * decode path (up to 32 tokens) is always deterministic: its down kernel sums
 * each token's k slot outputs in slot order. */
#define MOE_FLAG_DETERMINISTIC 1u

/* Workspace bytes moe_forward / moe_forward_routed need for T tokens. */
MOE_API size_t moe_workspace_bytes(const moe_shape_t* shape, int T);

/* Workspace bytes for T tokens with the given MOE_FLAG_* bits (flags = 0:
 * moe_workspace_bytes; MOE_FLAG_DETERMINISTIC adds T*k*H*4 bytes for the
 * grouped path's per-row outputs). */
MOE_API size_t moe_workspace_bytes_flags(const moe_shape_t* shape, int T, uint32_t flags);

/* Forward pass of the routed-expert layer.
 *   x            [T, H] bf16 hidden states
 *   router_w     [E, H] bf16 router weight (logits = x router_w^T, fp32 accumulation)
 *   logit_bias   [E] fp32 added to the logits before top-k (nullable)
 *   gate_up_packed  packed bank of [E, 2I, H] (gate rows [0, I), up rows [I, 2I))
 *   down_packed     packed bank of [E, H, I]
 *   workspace    >= moe_workspace_bytes(shape, T) bytes, 256-byte aligned
 *   out          [T, H] bf16 output: sum_j w_tj W_down[e] bf16(silu(g) * u),
 *                accumulated in fp32 and rounded to bf16 once.
 * T >= 0 (T == 0 is a no-op).  Device-side waits are bounded; an expired
 * wait is reported by moe_workspace_status. */
MOE_API moe_status_t moe_forward(const moe_shape_t* shape, const uint16_t* x, int T,
                         const uint16_t* router_w, const float* logit_bias,
                         const void* gate_up_packed, const void* down_packed,
                         void* workspace, size_t workspace_bytes, uint16_t* out,
                         const moe_forward_opts_t* opts, cudaStream_t stream);

/* Workspace bytes moe_forward_host needs for T tokens: moe_forward's plus
 * device staging for the hidden states and the output; 0 if invalid. */
MOE_API size_t moe_workspace_bytes_host(const moe_shape_t* shape, int T);

/* moe_forward with the hidden states and the output in HOST memory (the
 * weights, router and workspace stay device memory): enqueues on `stream` the
 * copy of x_host [T, H] bf16 into the workspace, the forward pass, and the
 * copy of the output back to out_host [T, H] bf16.  Asynchronous like every
 * other call: out_host holds the result once the stream has been
 * synchronised, and x_host must stay unchanged until then.  Page-locked host
 * buffers (cudaHostAlloc / cudaHostRegister) make the copies asynchronous;
 * pageable ones work but the copies then synchronise with the host.
 * workspace >= moe_workspace_bytes_host(shape, T) bytes, 256-byte aligned;
 * other arguments, paths and errors as moe_forward (the debug outputs of
 * opts, if given, are device pointers; opts->flags must be 0, else
 * MOE_ERR_UNSUPPORTED). */
MOE_API moe_status_t moe_forward_host(const moe_shape_t* shape, const uint16_t* x_host, int T,
                                      const uint16_t* router_w, const float* logit_bias,
                                      const void* gate_up_packed, const void* down_packed, void* workspace,
                                      size_t workspace_bytes, uint16_t* out_host, const moe_forward_opts_t* opts,
                                      cudaStream_t stream);

/* The same layer with the routing given: topk_ids [T, k] int32 (distinct
 * experts per token, values in [0, E)) and topk_w [T, k] fp32.  Used to check
 * the expert path on its own (e.g. with the oracle's routing). */
MOE_API moe_status_t moe_forward_routed(const moe_shape_t* shape, const uint16_t* x, int T,
                                const int32_t* topk_ids, const float* topk_w,
                                const void* gate_up_packed, const void* down_packed,
                                void* workspace, size_t workspace_bytes, uint16_t* out,
                                const moe_forward_opts_t* opts, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Expert parallelism ("Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Serving: the
 * model runs with expert parallelism over a pair of GPUs).  Each GPU holds the
 * packed banks of a contiguous range of experts; every GPU routes all tokens
 * over all E experts (the router weight is replicated), computes the
 * contribution of its own experts, and the fp32 contributions are summed
 * across GPUs (the caller's collective, e.g. an NCCL reduce-scatter) before
 * the single bf16 rounding of moe_partial_to_bf16.
 * ---------------------------------------------------------------------- */

/* The routed layer restricted to experts [expert_begin, expert_begin +
 * num_local_experts) of the layer's E:
 *   partial_out [T, H] fp32 = sum over the slots j whose expert e = ids[t, j]
 *                             lies in the range of w_tj W_down[e] a_tj,
 * not rounded (zero for tokens with no local expert).  The routing (logits,
 * top-k, weights) is over all E experts, exactly as moe_forward's, so the sum
 * of partial_out over a partition of the experts, rounded once to bf16, is
 * moe_forward's output.  gate_up_local / down_local are packed banks of
 * num_local_experts matrices ([n, 2I, H] and [n, H, I], the range's experts
 * in order; moe_bank_bytes with E = n).  shape->num_experts is the layer's E.
 * partial_out is 16-byte aligned device memory; the workspace is
 * moe_workspace_bytes(shape, T).  Other arguments, paths and errors as
 * moe_forward; MOE_ERR_INVALID_ARG for a range outside [0, E). */
MOE_API moe_status_t moe_forward_partial(const moe_shape_t* shape, const uint16_t* x, int T,
                                         const uint16_t* router_w, const float* logit_bias, int expert_begin,
                                         int num_local_experts, const void* gate_up_local,
                                         const void* down_local, void* workspace, size_t workspace_bytes,
                                         float* partial_out, const moe_forward_opts_t* opts, cudaStream_t stream);

/* out [T, H] bf16 = bf16_rne(partial [T, H] fp32): the layer output from the
 * summed expert-parallel contributions.  H a multiple of 4, both pointers
 * 16-byte aligned device memory. */
MOE_API moe_status_t moe_partial_to_bf16(const float* partial, int T, int H, uint16_t* out, cudaStream_t stream);

/* The dense shared expert of a Qwen3.5-MoE block, beside the routed ones
 * ("Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe table: shared expert
 * gate/up/down_proj and shared_expert_gate; "kirillbilchenko/Nex-N2.5-mini-
 * MXFP4-MxWave", What was quantized: shared experts stay bf16).  Weights are
 * bf16 (not quantised), device pointers, 16-byte aligned. */
typedef struct {
  int inter;                /* I_s, a positive multiple of 64 (512 in the cards' model) */
  const uint16_t* gate_up;  /* [2*I_s, H] bf16: gate rows [0, I_s), up rows [I_s, 2*I_s) */
  const uint16_t* down;     /* [H, I_s] bf16 */
  const uint16_t* gate;     /* [H] bf16 weight of the shared_expert_gate (H -> 1) */
} moe_shared_expert_t;

/* Workspace bytes moe_forward_shared needs for T tokens (the routed layer's
 * workspace plus the shared expert's fp32 and bf16 intermediates); 0 if the
 * arguments are invalid. */
MOE_API size_t moe_workspace_bytes_shared(const moe_shape_t* shape, int inter_shared, int T);

/* moe_forward plus the shared expert:
 *   g_t   = sigmoid(x_t . w_gate)                     fp32
 *   a_s   = bf16(silu(W_gate_s x_t) * (W_up_s x_t))   (the routed experts' rounding)
 *   out_t = bf16( sum_j w_tj y_tj  +  g_t * (W_down_s a_s) )   one final rounding
 * The shared expert's products run on tcgen05 above 32 tokens and as a
 * split-K mma.sync product up to 32; its contribution is added to the routed
 * combine in fp32 before the output's single bf16 rounding.  On the decode
 * path with the split-K routing (up to 32 tokens, E <= 256, k <= 8,
 * H <= 2048) and I_s <= 512 it launches no kernel of its own: its gate_up
 * rows and gate vector are computed by the routing GEMV, its SwiGLU and gate
 * by the gate_up kernel, its down product inside the down kernel's combine
 * (moe_forward_shared_launch_count says which form a call takes).  Other
 * arguments, paths, errors and the workspace rules as moe_forward (workspace
 * >= moe_workspace_bytes_shared bytes; opts->flags must be 0, else
 * MOE_ERR_UNSUPPORTED). */
MOE_API moe_status_t moe_forward_shared(const moe_shape_t* shape, const moe_shared_expert_t* shared,
                                const uint16_t* x, int T, const uint16_t* router_w,
                                const float* logit_bias, const void* gate_up_packed,
                                const void* down_packed, void* workspace, size_t workspace_bytes,
                                uint16_t* out, const moe_forward_opts_t* opts, cudaStream_t stream);

/* Zeroes the status word and the kernels' completion counters at the start
 * of a workspace (its first 4096 bytes; enqueued on `stream`).  Call once
 * after allocating a workspace, before its first use; every forward leaves
 * the counters at zero again. */
MOE_API moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Number of kernels moe_forward (routed = 0) or moe_forward_routed
 * (routed = 1) launches for T tokens on `path` (memsets and the optional
 * debug copies are not kernels and are not counted); -1 if the arguments are
 * invalid or the path does not support them. */
MOE_API int moe_forward_launch_count(const moe_shape_t* shape, int T, moe_path_t path, int routed);

/* Number of kernels moe_forward_shared launches for T tokens on `path` with
 * a shared expert of intermediate size inter_shared: moe_forward's count,
 * plus 3 where the shared expert runs as its own kernels (0 where it rides
 * the decode kernels); -1 if the arguments are invalid or the path does not
 * support them. */
MOE_API int moe_forward_shared_launch_count(const moe_shape_t* shape, int inter_shared, int T, moe_path_t path);

/* Synchronises `stream`, then reports MOE_ERR_TIMEOUT if a bounded
 * device-side wait of a previous moe_forward on this workspace expired (and
 * clears the flag together with every device counter of the workspace, as
 * moe_workspace_init does), MOE_OK otherwise. */
MOE_API moe_status_t moe_workspace_status(void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* moe_forward for callers that cannot allocate device memory.  The model
 * cards have no counterpart to this entry point.  It serves code that may
 * not call cudaMalloc while it issues its work: runtimes and inference
 * engines that reserve their whole device-memory budget at start-up, plugins
 * whose host framework owns the device allocator, and code that records its
 * GPU work for later replay, where an allocation inside the recorded region
 * is not allowed.  The caller passes only inputs and outputs (same meaning,
 * layout and alignment as moe_forward); the scratch is a fixed array inside
 * the library (moe_noalloc_scratch_bytes(), 8 MiB), held by every GPU that
 * loads the library until the process exits.
 *   - Returns MOE_ERR_UNSUPPORTED when moe_workspace_bytes(shape, T) exceeds
 *     that size (e.g. large prefill batches), MOE_ERR_INVALID_ARG for the
 *     argument errors of moe_forward; nothing is enqueued then.
 *   - The first call on a device (and the first after that device's context
 *     was re-created, e.g. by cudaDeviceReset) looks up the array's device
 *     address; make that first call before any stream capture.
 *   - Calls on one device share the array and it keeps the last call's
 *     contents: each call clears the device counters it needs at zero, and
 *     calls that overlap on the GPU (unordered streams) race.
 *   - An expired bounded device wait is recorded in the array's status word,
 *     which later calls leave set (while it is set, their device-wide waits
 *     give up at once); moe_noalloc_status reports and clears it.
 *   - No device allocation and no freeing happen inside this call. */
MOE_API moe_status_t moe_forward_noalloc(const moe_shape_t* shape, const uint16_t* x, int T,
                                         const uint16_t* router_w, const float* logit_bias,
                                         const void* gate_up_packed, const void* down_packed,
                                         uint16_t* out, cudaStream_t stream);

/* Size in bytes of moe_forward_noalloc's fixed scratch array. */
MOE_API size_t moe_noalloc_scratch_bytes(void);

/* Synchronises `stream`, then reports MOE_ERR_TIMEOUT if a bounded device
 * wait of a moe_forward_noalloc call on the current device expired since the
 * last report (and clears the status word and the device counters of the
 * scratch array), MOE_OK otherwise.  Allocates nothing. */
MOE_API moe_status_t moe_noalloc_status(cudaStream_t stream);

/* Self-test of the bounded device-side wait: launches one warp that waits on
 * a barrier nothing ever arrives at, gives up after `limit_ns` nanoseconds of
 * device time (at most 10 s) and raises the workspace status word, so that a
 * following moe_workspace_status returns MOE_ERR_TIMEOUT.  With workspace ==
 * NULL it raises the status word of moe_forward_noalloc's scratch array on
 * the current device instead (reported by moe_noalloc_status).  The GPU
 * context stays usable.  No counterpart on the model cards: this checks the
 * library's own failure reporting. */
MOE_API moe_status_t moe_selftest_bounded_wait(void* workspace, size_t workspace_bytes, uint64_t limit_ns,
                                       cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_W4A16_H */
