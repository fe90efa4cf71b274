// C ABI of the W4A16 routed-expert MoE layer: argument validation, workspace
// carve-up and the order of kernel launches on the caller's stream.
#include <nvtx3/nvToolsExt.h>
#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

uint32_t opt_flags(const moe_forward_opts_t* o) { return o ? o->flags : 0u; }

// NVTX range over the host code that enqueues one stage (or one call): a
// profiler shows which stage each kernel launch belongs to.  NVTX is header
// only; without an attached tool a range costs a pointer check.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool valid_fmt(moe_format_t f) {
  return f == MOE_FMT_INT4_G128 || f == MOE_FMT_MXFP4_G32 || f == MOE_FMT_NVFP4_G16;
}

moe_status_t check_shape(const moe_shape_t* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (!valid_fmt(s->fmt)) return MOE_ERR_INVALID_ARG;
  if (s->hidden <= 0 || s->inter <= 0 || s->num_experts <= 0 || s->top_k <= 0) return MOE_ERR_INVALID_ARG;
  if (s->hidden % 64 || s->inter % 64) return MOE_ERR_UNSUPPORTED;
  if (s->top_k > kMaxTopK || s->top_k > s->num_experts || s->num_experts > kMaxExperts)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_T(const moe_shape_t* s, int T) {
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (long(T) * s->top_k > (1L << 26)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                              \
  do {                                             \
    const moe_status_t _st = cuda_status(expr);    \
    if (_st != MOE_OK) return _st;                 \
  } while (0)

Bank make_bank(const void* packed, moe_format_t fmt, int E, int N, int K) {
  Bank b;
  b.codes = static_cast<const uint8_t*>(packed);
  b.scales = static_cast<const uint8_t*>(packed) + bank_scale_offset(fmt, E, N, K);
  b.gscale = fmt == MOE_FMT_NVFP4_G16
                 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(packed) + bank_gscale_offset(fmt, E, N, K))
                 : nullptr;
  b.N = N;
  b.K = K;
  return b;
}

// Record stage event (after = 0: before the stage, 1: after it) if the caller
// asked for it; inside a stream capture it becomes an external event node so
// that it can be timed when the graph is replayed.
cudaError_t mark(const moe_forward_opts_t* o, int stage, int after, cudaStream_t stream) {
  if (!o || !o->stage_events) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t err = cudaStreamIsCapturing(stream, &cs);
  if (err != cudaSuccess) return err;
  cudaEvent_t ev = o->stage_events[2 * stage + after];
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal)
                                             : cudaEventRecord(ev, stream);
}

__global__ void bounded_wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    // nothing ever arrives: the wait has to give up by itself
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicOr(status, kStatusTimeout);
        break;
      }
    }
  }
}

}  // namespace

Workspace carve_workspace(void* base, const moe_shape_t& s, int T, uint32_t flags) {
  Workspace w{};
  const size_t R = size_t(T) * s.top_k;
  const size_t E = s.num_experts, H = s.hidden, I = s.inter;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    void* r = p ? p + off : nullptr;
    off += align_up(bytes, 256);
    return r;
  };
  w.status = static_cast<uint32_t*>(take(kStatusBytes));
  w.route_counter = p ? reinterpret_cast<int32_t*>(w.status) + 1 : nullptr;
  w.logits = static_cast<float*>(take(size_t(T) * E * 4));
  w.topk_ids = static_cast<int32_t*>(take(R * 4));
  w.topk_w = static_cast<float*>(take(R * 4));
  w.offsets = static_cast<int32_t*>(take((E + 1) * 4));
  w.sorted_rows = static_cast<int32_t*>(take(R * 4));
  w.pos = static_cast<int32_t*>(take(R * 4));
  w.touched = static_cast<int32_t*>(take((E + 1) * 4));
  w.tile_base = static_cast<int32_t*>(take((E + 1) * 4));
  w.block_hist = static_cast<int32_t*>(take(permute_large_hist_bytes(T, int(E), s.top_k)));
  w.act = static_cast<uint16_t*>(take(R * I * 2));
  w.out_acc = static_cast<float*>(take(size_t(T) * H * 4));
  // per-row down outputs of the deterministic grouped combine (the decode
  // path combines inside its down kernel)
  const size_t ypart_bytes = (flags & MOE_FLAG_DETERMINISTIC) ? R * H * 4 : 0;
  w.ypart = static_cast<float*>(take(ypart_bytes));
  w.route_part = static_cast<float*>(take(T <= kDecodeMaxT ? route_part_bytes(T, int(H), int(E), s.top_k) : 0));
  w.bytes = off;
  return w;
}

cudaError_t launch_bounded_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

namespace {

// Routing state (permutation + touched list + tile prefix) from ids in ws.
moe_status_t build_permutation(const moe_shape_t& s, int T, const Workspace& ws, cudaStream_t stream) {
  const long R = long(T) * s.top_k;
  if (R <= 1024)
    return cuda_status(launch_permute_small(ws.topk_ids, T, s.num_experts, s.top_k, ws.offsets, ws.sorted_rows,
                                            ws.pos, ws.touched, ws.tile_base, kGemmBN, stream));
  return cuda_status(launch_permute_large(ws.topk_ids, T, s.num_experts, s.top_k, ws.offsets, ws.sorted_rows,
                                          ws.pos, ws.block_hist, ws.touched, ws.tile_base, kGemmBN, stream));
}

// Stages 0-1: router logits, top-k and the permutation over all E experts
// (with `sf`, the small-batch routing GEMV also computes the folded shared
// expert's rows).
moe_status_t route_all(const moe_shape_t& s, int T, const uint16_t* x, const uint16_t* router_w,
                       const float* logit_bias, const Workspace& ws, const moe_forward_opts_t* opts,
                       cudaStream_t stream, const SharedFold* sf = nullptr) {
  NvtxRange range("moe.route");
  MOE_TRY(mark(opts, 0, 0, stream));
  if (T <= kDecodeMaxT) {
    // router logits, top-k and the permutation: split-K GEMV + finalize, or one kernel
    MOE_TRY(launch_route_small(x, router_w, logit_bias, T, s.hidden, s.num_experts, s.top_k, ws, kGemmBN, stream,
                               sf));
    MOE_TRY(mark(opts, 0, 1, stream));
    MOE_TRY(mark(opts, 1, 0, stream));
  } else {
    MOE_TRY(launch_router_gemm(x, router_w, T, s.hidden, s.num_experts, ws.logits, ws.status, stream));
    MOE_TRY(mark(opts, 0, 1, stream));
    MOE_TRY(mark(opts, 1, 0, stream));
    MOE_TRY(launch_topk(ws.logits, logit_bias, T, s.num_experts, s.top_k, ws.topk_ids, ws.topk_w, stream));
    moe_status_t st = build_permutation(s, T, ws, stream);
    if (st != MOE_OK) return st;
  }
  MOE_TRY(mark(opts, 1, 1, stream));
  return MOE_OK;
}

// Stages 2-4: experts and combine, given routing in the workspace.  The banks
// hold the experts of `er`; with partial_out the result is the fp32 sum over
// those experts (no rounding), else the bf16 output.  sh_gate / sh_y
// (nullable): the shared expert's gate [T] and output [T, H], added before
// the output's bf16 rounding.
moe_status_t run_experts(const moe_shape_t& s, int T, const uint16_t* x, const void* gu_packed,
                         const void* dn_packed, const ExpertRange& er, const Workspace& ws, uint16_t* out,
                         float* partial_out, bool decode, const moe_forward_opts_t* o, cudaStream_t stream,
                         const float* sh_gate = nullptr, const float* sh_y = nullptr,
                         const SharedFold* sf = nullptr) {
  const int n_bank = er.hi - er.lo;
  const Bank gu = make_bank(gu_packed, s.fmt, n_bank, 2 * s.inter, s.hidden);
  const Bank dn = make_bank(dn_packed, s.fmt, n_bank, s.hidden, s.inter);
  {
    NvtxRange range("moe.gate_up");
    MOE_TRY(mark(o, 2, 0, stream));
    if (decode) MOE_TRY(launch_decode_gate_up(s, T, x, gu, dn, er, ws, stream, sf));
    else MOE_TRY(launch_grouped_gate_up(s, T, x, gu, er, ws, stream));
    MOE_TRY(mark(o, 2, 1, stream));
  }
  NvtxRange range("moe.down_combine");
  MOE_TRY(mark(o, 3, 0, stream));
  if (decode) {
    // down products and each token's slots summed in slot order, in one kernel
    MOE_TRY(launch_decode_down(s, T, dn, er, ws, sh_gate, sh_y, out, partial_out, stream, sf));
    MOE_TRY(mark(o, 3, 1, stream));
    MOE_TRY(mark(o, 4, 0, stream));
  } else if (opt_flags(o) & MOE_FLAG_DETERMINISTIC) {
    // every (token, slot) row's weighted output in its own row, then the
    // k rows of each token summed in slot order
    MOE_TRY(launch_grouped_down(s, T, dn, er, ws, nullptr, ws.ypart, stream));
    MOE_TRY(mark(o, 3, 1, stream));
    MOE_TRY(mark(o, 4, 0, stream));
    MOE_TRY(launch_combine_rows(s, T, er, ws, ws.ypart, sh_gate, sh_y, out, partial_out, stream));
  } else {
    float* acc = partial_out ? partial_out : ws.out_acc;
    MOE_TRY(cudaMemsetAsync(acc, 0, size_t(T) * s.hidden * 4, stream));
    MOE_TRY(launch_grouped_down(s, T, dn, er, ws, acc, nullptr, stream));
    MOE_TRY(mark(o, 3, 1, stream));
    MOE_TRY(mark(o, 4, 0, stream));
    if (!partial_out) MOE_TRY(launch_finalize_out(ws.out_acc, T, s.hidden, sh_gate, sh_y, out, stream));
  }
  MOE_TRY(mark(o, 4, 1, stream));
  return MOE_OK;
}

moe_status_t copy_debug_outputs(const moe_shape_t& s, int T, const Workspace& ws, const moe_forward_opts_t* o,
                                bool routed, cudaStream_t stream) {
  if (!o) return MOE_OK;
  const size_t R = size_t(T) * s.top_k;
  auto cp = [&](void* dst, const void* src, size_t bytes) -> cudaError_t {
    return dst ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, stream) : cudaSuccess;
  };
  if (!routed) {
    MOE_TRY(cp(o->topk_ids_out, ws.topk_ids, R * 4));
    MOE_TRY(cp(o->topk_w_out, ws.topk_w, R * 4));
    MOE_TRY(cp(o->logits_out, ws.logits, size_t(T) * s.num_experts * 4));
  }
  MOE_TRY(cp(o->offsets_out, ws.offsets, size_t(s.num_experts + 1) * 4));
  MOE_TRY(cp(o->sorted_rows_out, ws.sorted_rows, R * 4));
  MOE_TRY(cp(o->act_out, ws.act, R * s.inter * 2));
  return MOE_OK;
}

bool valid_path(moe_path_t p) {
  return p == MOE_PATH_AUTO || p == MOE_PATH_DECODE || p == MOE_PATH_PREFILL;
}

// Everything moe_forward checks except the workspace; `decode` gets the path.
moe_status_t check_forward_inputs(const moe_shape_t* shape, const uint16_t* x, int T, const void* gu,
                                  const void* dn, uint16_t* out, const moe_forward_opts_t* opts, bool* decode) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if ((st = check_T(shape, T)) != MOE_OK) return st;
  const moe_path_t path = opts ? opts->path : MOE_PATH_AUTO;
  if (!valid_path(path)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;  // nothing to do; pointers may be null
  if (!x || !gu || !dn || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(gu, 256) || !aligned(dn, 256) || !aligned(out, 16))
    return MOE_ERR_INVALID_ARG;
  const bool dec_ok = decode_supported(*shape, T);
  if (path == MOE_PATH_DECODE && !dec_ok) return MOE_ERR_UNSUPPORTED;
  *decode = path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && dec_ok);
  if (!*decode && !grouped_supported(*shape)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_forward_common(const moe_shape_t* shape, const uint16_t* x, int T, const void* gu,
                                  const void* dn, void* workspace, size_t ws_bytes, uint16_t* out,
                                  const moe_forward_opts_t* opts, bool* decode) {
  moe_status_t st = check_forward_inputs(shape, x, T, gu, dn, out, opts, decode);
  if (st != MOE_OK) return st;
  const uint32_t flags = opts ? opts->flags : 0u;
  if (flags & ~MOE_FLAG_DETERMINISTIC) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_workspace_bytes_flags(shape, T, flags)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace

namespace moe {

// The argument checks of moe_forward that do not involve the workspace (for
// entry points that supply their own scratch).
moe_status_t check_forward_args(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                                const float* logit_bias, const void* gu, const void* dn, uint16_t* out) {
  bool decode = false;
  const moe_status_t st = check_forward_inputs(shape, x, T, gu, dn, out, nullptr, &decode);
  if (st != MOE_OK || T == 0) return st;
  if (!router_w || !aligned(router_w, 16) || (logit_bias && !aligned(logit_bias, 4))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace moe

extern "C" {

const char* moe_status_str(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "bounded device wait expired";
    case MOE_ERR_NONFINITE: return "non-finite input";
  }
  return "unknown status";
}

int moe_abi_version(void) { return MOE_ABI_VERSION; }

size_t moe_bank_bytes(moe_format_t fmt, int E, int N, int K) {
  if (!valid_fmt(fmt) || E <= 0 || N <= 0 || K <= 0 || K % 32) return 0;
  return bank_total_bytes(fmt, E, N, K);
}

size_t moe_bank_scale_offset(moe_format_t fmt, int E, int N, int K) {
  if (!valid_fmt(fmt) || E <= 0 || N <= 0 || K <= 0 || K % 32) return 0;
  return bank_scale_offset(fmt, E, N, K);
}

size_t moe_packed_bytes(const moe_shape_t* s, int which) {
  if (check_shape(s) != MOE_OK) return 0;
  if (which == 0) return moe_bank_bytes(s->fmt, s->num_experts, 2 * s->inter, s->hidden);
  if (which == 1) return moe_bank_bytes(s->fmt, s->num_experts, s->hidden, s->inter);
  return 0;
}

static moe_status_t pack_common(moe_format_t fmt, const uint16_t* w, int E, int N, int K, void* packed,
                                int32_t* nonfinite, cudaStream_t stream) {
  if (!w || !packed) return MOE_ERR_INVALID_ARG;
  if (E <= 0 || N <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(packed, 256) || (nonfinite && !aligned(nonfinite, 4))) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_pack(fmt, w, E, N, K, packed, nonfinite, stream));
}

moe_status_t moe_pack_int4_g128(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                                cudaStream_t stream) {
  return pack_common(MOE_FMT_INT4_G128, w, E, N, K, packed, nonfinite, stream);
}

moe_status_t moe_pack_mxfp4(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                            cudaStream_t stream) {
  return pack_common(MOE_FMT_MXFP4_G32, w, E, N, K, packed, nonfinite, stream);
}

moe_status_t moe_pack_nvfp4(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                            cudaStream_t stream) {
  return pack_common(MOE_FMT_NVFP4_G16, w, E, N, K, packed, nonfinite, stream);
}

moe_status_t moe_pack_mxfp4_rule(const uint16_t* w, int E, int N, int K, void* packed, int32_t* nonfinite,
                                 moe_mx_exp_rule_t rule, cudaStream_t stream) {
  if (rule != MOE_MX_EXP_FLOOR && rule != MOE_MX_EXP_CEIL && rule != MOE_MX_EXP_OCP && rule != MOE_MX_EXP_MSE)
    return MOE_ERR_INVALID_ARG;
  if (!w || !packed) return MOE_ERR_INVALID_ARG;
  if (E <= 0 || N <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(packed, 256) || (nonfinite && !aligned(nonfinite, 4))) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_pack_mxfp4_rule(w, E, N, K, packed, nonfinite, int(rule), stream));
}

moe_status_t moe_dequant(const void* packed, moe_format_t fmt, int E, int N, int K, uint16_t* w_out,
                         cudaStream_t stream) {
  if (!packed || !w_out || !valid_fmt(fmt)) return MOE_ERR_INVALID_ARG;
  if (E <= 0 || N <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARG;
  if (!aligned(packed, 256) || !aligned(w_out, 16)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_dequant(fmt, packed, E, N, K, w_out, stream));
}

moe_status_t moe_route(const float* logits, const float* bias, int T, int E, int k, int32_t* topk_ids,
                       float* topk_w, cudaStream_t stream) {
  if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxTopK || k > E) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4) || (bias && !aligned(bias, 4)))
    return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_topk(logits, bias, T, E, k, topk_ids, topk_w, stream));
}

size_t moe_permute_workspace_bytes(int T, int E, int k) {
  if (T < 0 || E <= 0 || k <= 0) return 0;
  return 4 * align_up(size_t(E + 1) * 4, 256) + align_up(permute_large_hist_bytes(T, E, k), 256) + 256;
}

moe_status_t moe_permute(const int32_t* topk_ids, int T, int E, int k, int32_t* offsets, int32_t* sorted_rows,
                         int32_t* pos, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (T < 0 || E <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxTopK || k > E) return MOE_ERR_UNSUPPORTED;
  if (!offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_ids || !sorted_rows || !pos)) return MOE_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < moe_permute_workspace_bytes(T, E, k))
    return MOE_ERR_WORKSPACE;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  int32_t* touched = reinterpret_cast<int32_t*>(p);
  int32_t* tile_base = reinterpret_cast<int32_t*>(p + align_up(size_t(E + 1) * 4, 256));
  int32_t* hist = reinterpret_cast<int32_t*>(p + 4 * align_up(size_t(E + 1) * 4, 256));
  const long R = long(T) * k;
  if (R <= 1024)
    return cuda_status(
        launch_permute_small(topk_ids, T, E, k, offsets, sorted_rows, pos, touched, tile_base, kGemmBN, stream));
  return cuda_status(launch_permute_large(topk_ids, T, E, k, offsets, sorted_rows, pos, hist, touched, tile_base,
                                          kGemmBN, stream));
}

size_t moe_workspace_bytes(const moe_shape_t* shape, int T) {
  if (check_shape(shape) != MOE_OK || T < 0) return 0;
  return carve_workspace(nullptr, *shape, T).bytes;
}

size_t moe_workspace_bytes_flags(const moe_shape_t* shape, int T, uint32_t flags) {
  if (check_shape(shape) != MOE_OK || T < 0 || (flags & ~MOE_FLAG_DETERMINISTIC)) return 0;
  return carve_workspace(nullptr, *shape, T, flags).bytes;
}

moe_status_t moe_forward(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                         const float* logit_bias, const void* gate_up_packed, const void* down_packed,
                         void* workspace, size_t workspace_bytes, uint16_t* out, const moe_forward_opts_t* opts,
                         cudaStream_t stream) {
  bool decode = false;
  moe_status_t st = check_forward_common(shape, x, T, gate_up_packed, down_packed, workspace, workspace_bytes,
                                         out, opts, &decode);
  if (st != MOE_OK || T == 0) return st;
  if (!router_w || !aligned(router_w, 16) || (logit_bias && !aligned(logit_bias, 4))) return MOE_ERR_INVALID_ARG;
  const moe_shape_t& s = *shape;
  const Workspace ws = carve_workspace(workspace, s, T, opt_flags(opts));
  if ((st = route_all(s, T, x, router_w, logit_bias, ws, opts, stream)) != MOE_OK) return st;
  if ((st = run_experts(s, T, x, gate_up_packed, down_packed, ExpertRange{0, s.num_experts}, ws, out, nullptr, decode,
                        opts, stream)) != MOE_OK)
    return st;
  return copy_debug_outputs(s, T, ws, opts, false, stream);
}

moe_status_t moe_forward_partial(const moe_shape_t* shape, const uint16_t* x, int T, const uint16_t* router_w,
                                 const float* logit_bias, int expert_begin, int num_local_experts,
                                 const void* gate_up_local, const void* down_local, void* workspace,
                                 size_t workspace_bytes, float* partial_out, const moe_forward_opts_t* opts,
                                 cudaStream_t stream) {
  bool decode = false;
  // the checks of moe_forward, with the fp32 output in place of the bf16 one
  moe_status_t st = check_forward_common(shape, x, T, gate_up_local, down_local, workspace, workspace_bytes,
                                         reinterpret_cast<uint16_t*>(partial_out), opts, &decode);
  if (st != MOE_OK) return st;
  if (expert_begin < 0 || num_local_experts < 1 || long(expert_begin) + num_local_experts > shape->num_experts)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!router_w || !aligned(router_w, 16) || (logit_bias && !aligned(logit_bias, 4))) return MOE_ERR_INVALID_ARG;
  const moe_shape_t& s = *shape;
  const Workspace ws = carve_workspace(workspace, s, T, opt_flags(opts));
  if ((st = route_all(s, T, x, router_w, logit_bias, ws, opts, stream)) != MOE_OK) return st;
  const ExpertRange er{expert_begin, expert_begin + num_local_experts};
  if ((st = run_experts(s, T, x, gate_up_local, down_local, er, ws, nullptr, partial_out, decode, opts, stream)) !=
      MOE_OK)
    return st;
  return copy_debug_outputs(s, T, ws, opts, false, stream);
}

moe_status_t moe_partial_to_bf16(const float* partial, int T, int H, uint16_t* out, cudaStream_t stream) {
  if (T < 0 || H <= 0 || H % 4) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!partial || !out || !aligned(partial, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
  return cuda_status(launch_finalize_out(partial, T, H, nullptr, nullptr, out, stream));
}

size_t moe_workspace_bytes_host(const moe_shape_t* shape, int T) {
  const size_t base = moe_workspace_bytes(shape, T);
  if (base == 0) return 0;
  return base + 2 * align_up(size_t(T) * shape->hidden * 2, 256);
}

moe_status_t moe_forward_host(const moe_shape_t* shape, const uint16_t* x_host, int T, const uint16_t* router_w,
                              const float* logit_bias, const void* gate_up_packed, const void* down_packed,
                              void* workspace, size_t workspace_bytes, uint16_t* out_host,
                              const moe_forward_opts_t* opts, cudaStream_t stream) {
  if (check_shape(shape) != MOE_OK || T < 0) return check_shape(shape) != MOE_OK ? check_shape(shape) : MOE_ERR_INVALID_ARG;
  if (opt_flags(opts)) return MOE_ERR_UNSUPPORTED;  // the flags' larger workspace is not laid out here
  if (T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < moe_workspace_bytes_host(shape, T))
    return MOE_ERR_WORKSPACE;
  // device staging of x and out after the forward's own workspace
  const size_t base = moe_workspace_bytes(shape, T);
  const size_t io = size_t(T) * shape->hidden * 2;
  uint16_t* x_dev = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + base);
  uint16_t* out_dev = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + base + align_up(io, 256));
  bool decode = false;
  moe_status_t st = check_forward_common(shape, x_dev, T, gate_up_packed, down_packed, workspace, base, out_dev,
                                         opts, &decode);
  if (st != MOE_OK) return st;
  if (!router_w || !aligned(router_w, 16) || (logit_bias && !aligned(logit_bias, 4))) return MOE_ERR_INVALID_ARG;
  MOE_TRY(cudaMemcpyAsync(x_dev, x_host, io, cudaMemcpyHostToDevice, stream));
  if ((st = moe_forward(shape, x_dev, T, router_w, logit_bias, gate_up_packed, down_packed, workspace, base, out_dev,
                        opts, stream)) != MOE_OK)
    return st;
  MOE_TRY(cudaMemcpyAsync(out_host, out_dev, io, cudaMemcpyDeviceToHost, stream));
  return MOE_OK;
}

moe_status_t moe_forward_routed(const moe_shape_t* shape, const uint16_t* x, int T, const int32_t* topk_ids,
                                const float* topk_w, const void* gate_up_packed, const void* down_packed,
                                void* workspace, size_t workspace_bytes, uint16_t* out,
                                const moe_forward_opts_t* opts, cudaStream_t stream) {
  bool decode = false;
  moe_status_t st = check_forward_common(shape, x, T, gate_up_packed, down_packed, workspace, workspace_bytes,
                                         out, opts, &decode);
  if (st != MOE_OK || T == 0) return st;
  if (!topk_ids || !topk_w || !aligned(topk_ids, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
  const moe_shape_t& s = *shape;
  Workspace ws = carve_workspace(workspace, s, T, opt_flags(opts));
  ws.topk_ids = const_cast<int32_t*>(topk_ids);
  ws.topk_w = const_cast<float*>(topk_w);
  MOE_TRY(mark(opts, 1, 0, stream));
  if ((st = build_permutation(s, T, ws, stream)) != MOE_OK) return st;
  MOE_TRY(mark(opts, 1, 1, stream));
  if ((st = run_experts(s, T, x, gate_up_packed, down_packed, ExpertRange{0, s.num_experts}, ws, out, nullptr, decode,
                        opts, stream)) != MOE_OK)
    return st;
  return copy_debug_outputs(s, T, ws, opts, true, stream);
}

// The shared expert's intermediates after the routed layer's workspace.
struct SharedWs {
  uint16_t* a;   // [T, I_s] bf16 SwiGLU (first: its offset is the routed workspace's size)
  float* g;      // [T] fp32 sigmoid gate
  float* y;      // [T, H] fp32 down product
  float* h;      // [splits][T, 2 I_s] fp32 gate_up product (split-K partials for T <= 32)
  int splits;
  size_t bytes;  // total workspace bytes, routed part included
};

static SharedWs carve_shared(void* base, const moe_shape_t& s, int I_s, int T) {
  SharedWs w{};
  size_t off = carve_workspace(nullptr, s, T).bytes;
  uint8_t* p = static_cast<uint8_t*>(base);
  auto take = [&](size_t bytes) -> void* {
    void* r = p ? p + off : nullptr;
    off += align_up(bytes, 256);
    return r;
  };
  w.splits = T <= kDecodeMaxT ? shared_gemv_splits(s.hidden) : 1;
  w.a = static_cast<uint16_t*>(take(size_t(T) * I_s * 2));
  w.g = static_cast<float*>(take(size_t(T) * 4));
  w.y = static_cast<float*>(take(size_t(T) * s.hidden * 4 * (T <= kDecodeMaxT ? shared_gemv_splits(I_s) : 1)));
  // h: the split-K gate_up partials, or (folded form) the routing GEMV's
  // partials of the gate_up rows and the gate
  const size_t h_fold = T <= kDecodeMaxT ? size_t(route_gemv_splits(s.hidden)) * T * (2 * I_s + 1) : 0;
  w.h = static_cast<float*>(take(std::max(size_t(w.splits) * T * 2 * I_s, h_fold) * 4));
  w.bytes = off;
  return w;
}

// The shared expert rides the small-batch kernels (routing GEMV, decode
// gate_up and down) instead of its own three: the decode kernels and the
// split-K routing take the shape, and its down product fits the down
// kernel's four 128-k sub-units.
static bool shared_folds(const moe_shape_t& s, int T, int I_s, bool decode) {
  return decode && T <= kDecodeMaxT && I_s <= kSharedFoldMaxInter &&
         route_fast_applies(T, s.hidden, s.num_experts, s.top_k) && decode_shared_fits(s, T);
}

size_t moe_workspace_bytes_shared(const moe_shape_t* shape, int inter_shared, int T) {
  if (check_shape(shape) != MOE_OK || T < 0 || inter_shared <= 0 || inter_shared % 64) return 0;
  return carve_shared(nullptr, *shape, inter_shared, T).bytes;
}

moe_status_t moe_forward_shared(const moe_shape_t* shape, const moe_shared_expert_t* shared, const uint16_t* x,
                                int T, const uint16_t* router_w, const float* logit_bias,
                                const void* gate_up_packed, const void* down_packed, void* workspace,
                                size_t workspace_bytes, uint16_t* out, const moe_forward_opts_t* opts,
                                cudaStream_t stream) {
  if (!shared) return MOE_ERR_INVALID_ARG;
  if (shared->inter <= 0) return MOE_ERR_INVALID_ARG;
  if (shared->inter % 64) return MOE_ERR_UNSUPPORTED;
  if (opt_flags(opts)) return MOE_ERR_UNSUPPORTED;  // the flags' larger workspace is not laid out here
  bool decode = false;
  moe_status_t st = check_forward_common(shape, x, T, gate_up_packed, down_packed, workspace, workspace_bytes,
                                         out, opts, &decode);
  if (st != MOE_OK || T == 0) return st;
  if (!router_w || !aligned(router_w, 16) || (logit_bias && !aligned(logit_bias, 4))) return MOE_ERR_INVALID_ARG;
  if (!shared->gate_up || !shared->down || !shared->gate || !aligned(shared->gate_up, 16) ||
      !aligned(shared->down, 16) || !aligned(shared->gate, 16))
    return MOE_ERR_INVALID_ARG;
  const moe_shape_t& s = *shape;
  const int I_s = shared->inter;
  if (workspace_bytes < carve_shared(nullptr, s, I_s, T).bytes) return MOE_ERR_WORKSPACE;
  const Workspace ws = carve_workspace(workspace, s, T, opt_flags(opts));
  const SharedWs sw = carve_shared(workspace, s, I_s, T);
  if (shared_folds(s, T, I_s, decode)) {
    const SharedFold sf{shared->gate_up, shared->gate, shared->down, I_s, route_gemv_splits(s.hidden),
                        sw.h, sw.a, sw.g};
    if ((st = route_all(s, T, x, router_w, logit_bias, ws, opts, stream, &sf)) != MOE_OK) return st;
    if ((st = run_experts(s, T, x, gate_up_packed, down_packed, ExpertRange{0, s.num_experts}, ws, out, nullptr,
                          decode, opts, stream, nullptr, nullptr, &sf)) != MOE_OK)
      return st;
    return copy_debug_outputs(s, T, ws, opts, false, stream);
  }
  // the shared expert needs only x: gate_up product, SwiGLU and gate, down
  // product (split-K mma.sync for small batches, tcgen05 above)
  {
    NvtxRange range("moe.shared_expert");
    if (T <= kDecodeMaxT && I_s <= 512) {
      MOE_TRY(launch_shared_gemv(x, shared->gate_up, T, s.hidden, 2 * I_s, sw.h, stream));
      MOE_TRY(launch_shared_swiglu_gate(x, shared->gate, sw.h, sw.splits, T, s.hidden, I_s, sw.a, sw.g, stream));
      MOE_TRY(launch_shared_gemv(sw.a, shared->down, T, I_s, s.hidden, sw.y, stream));  // one split: I_s <= 512
    } else {
      MOE_TRY(launch_router_gemm(x, shared->gate_up, T, s.hidden, 2 * I_s, sw.h, ws.status, stream));
      MOE_TRY(launch_shared_swiglu_gate(x, shared->gate, sw.h, 1, T, s.hidden, I_s, sw.a, sw.g, stream));
      MOE_TRY(launch_router_gemm(sw.a, shared->down, T, I_s, s.hidden, sw.y, ws.status, stream));
    }
  }
  // the routed experts, their combine and the shared expert's gated output
  if ((st = route_all(s, T, x, router_w, logit_bias, ws, opts, stream)) != MOE_OK) return st;
  if ((st = run_experts(s, T, x, gate_up_packed, down_packed, ExpertRange{0, s.num_experts}, ws, out, nullptr, decode,
                        opts, stream, sw.g, sw.y)) != MOE_OK)
    return st;
  return copy_debug_outputs(s, T, ws, opts, false, stream);
}

int moe_forward_launch_count(const moe_shape_t* shape, int T, moe_path_t path, int routed) {
  if (check_shape(shape) != MOE_OK || check_T(shape, T) != MOE_OK) return -1;
  if (!valid_path(path)) return -1;
  if (T == 0) return 0;
  const bool dec_ok = decode_supported(*shape, T);
  if (path == MOE_PATH_DECODE && !dec_ok) return -1;
  const bool decode = path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && dec_ok);
  if (!decode && !grouped_supported(*shape)) return -1;
  const int perm = (long(T) * shape->top_k <= 1024) ? 1 : 3;
  int n = 0;
  if (routed) n += perm;
  else if (T <= kDecodeMaxT) n += route_small_launches(T, shape->hidden, shape->num_experts, shape->top_k);
  else n += 2 + perm;                                         // router GEMM, top-k, permutation
  n += decode ? 2 : 3;  // gate_up, down (+ combine / finalize for the grouped GEMMs)
  return n;
}

int moe_forward_shared_launch_count(const moe_shape_t* shape, int inter_shared, int T, moe_path_t path) {
  const int n = moe_forward_launch_count(shape, T, path, 0);
  if (n < 0 || inter_shared <= 0 || inter_shared % 64) return -1;
  if (T == 0) return 0;
  const bool decode = path == MOE_PATH_DECODE || (path == MOE_PATH_AUTO && decode_supported(*shape, T));
  return n + (shared_folds(*shape, T, inter_shared, decode) ? 0 : 3);
}

moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!workspace || workspace_bytes < kStatusBytes || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(workspace, 0, kStatusBytes, stream));
}

moe_status_t moe_workspace_status(void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!workspace || workspace_bytes < 256) return MOE_ERR_WORKSPACE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & kStatusTimeout) {
    // an expired wait can leave device counters mid-count: clear them all
    if (cudaMemset(workspace, 0, workspace_bytes < kStatusBytes ? workspace_bytes : kStatusBytes) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_ERR_TIMEOUT;
  }
  return MOE_OK;
}

moe_status_t moe_selftest_bounded_wait(void* workspace, size_t workspace_bytes, uint64_t limit_ns,
                                       cudaStream_t stream) {
  if (limit_ns > 10ull * 1000000000ull) return MOE_ERR_INVALID_ARG;
  if (!workspace) {
    // the status word of moe_forward_noalloc's scratch array on this device
    void* scratch = nullptr;
    MOE_TRY(noalloc_scratch_address(stream, &scratch));
    workspace = scratch;
  } else if (workspace_bytes < 256 || !aligned(workspace, 256)) {
    return MOE_ERR_WORKSPACE;
  }
  return cuda_status(launch_bounded_wait_probe(static_cast<uint32_t*>(workspace), limit_ns, stream));
}

}  // extern "C"
