"""ctypes binding of libmoe_w4a16.so: argument marshalling only.

Every function has the name of the C entry point it wraps and takes torch
tensors (device memory owned by the caller) in place of raw pointers.  All
computation happens in the library's CUDA kernels; there is no Python or CPU
fallback.  A missing library or a non-CUDA tensor raises immediately.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_w4a16.so")
_lib = None

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_NONFINITE = 6
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_NONFINITE"}

MOE_FMT_INT4_G128 = 1
MOE_FMT_MXFP4_G32 = 2
MOE_FMT_NVFP4_G16 = 3
FORMATS = {"int4_g128": MOE_FMT_INT4_G128, "mxfp4": MOE_FMT_MXFP4_G32, "nvfp4": MOE_FMT_NVFP4_G16}

MOE_PATH_AUTO, MOE_PATH_DECODE, MOE_PATH_PREFILL = 0, 1, 2
MOE_NUM_STAGES = 5
STAGE_NAMES = ("router", "route_permute", "gate_up", "down", "combine")


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}")
        self.status = status


class MoeShape(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("num_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("fmt", ctypes.c_int)]


class SharedExpert(ctypes.Structure):
    _fields_ = [("inter", ctypes.c_int), ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("gate", ctypes.c_void_p)]


class ForwardOpts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("topk_ids_out", ctypes.c_void_p), ("topk_w_out", ctypes.c_void_p),
                ("logits_out", ctypes.c_void_p), ("offsets_out", ctypes.c_void_p),
                ("sorted_rows_out", ctypes.c_void_p), ("act_out", ctypes.c_void_p),
                ("flags", ctypes.c_uint32), ("stage_events", ctypes.c_void_p)]


MOE_FLAG_DETERMINISTIC = 1


_SIGS = {
    "moe_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_abi_version": (ctypes.c_int, []),
    "moe_bank_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "moe_bank_scale_offset": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "moe_packed_bytes": (ctypes.c_size_t, [ctypes.POINTER(MoeShape), ctypes.c_int]),
    "moe_pack_int4_g128": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_pack_mxfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_pack_nvfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_pack_mxfp4_rule": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "moe_dequant": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   ctypes.c_void_p, ctypes.c_void_p]),
    "moe_route": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_permute_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "moe_permute": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                   ctypes.c_void_p]),
    "moe_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(MoeShape), ctypes.c_int]),
    "moe_workspace_bytes_flags": (ctypes.c_size_t, [ctypes.POINTER(MoeShape), ctypes.c_int, ctypes.c_uint32]),
    "moe_forward": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_size_t, ctypes.c_void_p, ctypes.POINTER(ForwardOpts),
                                   ctypes.c_void_p]),
    "moe_forward_routed": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                          ctypes.POINTER(ForwardOpts), ctypes.c_void_p]),
    "moe_workspace_bytes_host": (ctypes.c_size_t, [ctypes.POINTER(MoeShape), ctypes.c_int]),
    "moe_forward_host": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p, ctypes.POINTER(ForwardOpts),
                                        ctypes.c_void_p]),
    "moe_forward_partial": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                           ctypes.POINTER(ForwardOpts), ctypes.c_void_p]),
    "moe_partial_to_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p]),
    "moe_workspace_bytes_shared": (ctypes.c_size_t, [ctypes.POINTER(MoeShape), ctypes.c_int, ctypes.c_int]),
    "moe_forward_shared": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.POINTER(SharedExpert), ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                          ctypes.POINTER(ForwardOpts), ctypes.c_void_p]),
    "moe_forward_launch_count": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int]),
    "moe_forward_shared_launch_count": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_int, ctypes.c_int,
                                                       ctypes.c_int]),
    "moe_forward_noalloc": (ctypes.c_int, [ctypes.POINTER(MoeShape), ctypes.c_void_p, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "moe_noalloc_scratch_bytes": (ctypes.c_size_t, []),
    "moe_noalloc_status": (ctypes.c_int, [ctypes.c_void_p]),
    "moe_workspace_init": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "moe_workspace_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64,
                                                 ctypes.c_void_p]),
}


def lib():
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {_LIB_PATH} is missing "
                               "(run `python -m weight_only_bit_router_b200.build`)")
        handle = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(fn: str, status: int):
    if status != MOE_OK:
        raise MoeError(fn, status)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        return t  # already an address
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return stream


def _bits(t):
    """bf16 tensor -> the same memory (uint16 bit patterns for the C side)."""
    if t is not None and t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TypeError(f"expected a bf16 tensor, got {t.dtype}")
    return t


def make_shape(hidden, inter, num_experts, top_k, fmt) -> MoeShape:
    return MoeShape(hidden, inter, num_experts, top_k, FORMATS.get(fmt, fmt))


# ------------------------------------------------------------------ queries

def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_status_str(status: int) -> str:
    return lib().moe_status_str(status).decode()


def moe_bank_bytes(fmt, E, N, K) -> int:
    return lib().moe_bank_bytes(FORMATS.get(fmt, fmt), E, N, K)


def moe_bank_scale_offset(fmt, E, N, K) -> int:
    return lib().moe_bank_scale_offset(FORMATS.get(fmt, fmt), E, N, K)


def moe_packed_bytes(shape: MoeShape, which: int) -> int:
    return lib().moe_packed_bytes(ctypes.byref(shape), which)


def moe_workspace_bytes(shape: MoeShape, T: int) -> int:
    return lib().moe_workspace_bytes(ctypes.byref(shape), T)


def moe_workspace_bytes_flags(shape: MoeShape, T: int, flags: int) -> int:
    return lib().moe_workspace_bytes_flags(ctypes.byref(shape), T, int(flags))


def moe_permute_workspace_bytes(T, E, k) -> int:
    return lib().moe_permute_workspace_bytes(T, E, k)


# ------------------------------------------------------------------ packing

def _pack(name, fmt, w, packed, nonfinite, stream):
    E, N, K = w.shape
    if packed is None:
        packed = torch.empty(moe_bank_bytes(fmt, E, N, K), dtype=torch.uint8, device=w.device)
    _check(name, getattr(lib(), name)(_ptr(_bits(w)), E, N, K, _ptr(packed), _ptr(nonfinite), _stream(stream)))
    return packed


def moe_pack_int4_g128(w, packed=None, nonfinite=None, stream=None):
    return _pack("moe_pack_int4_g128", MOE_FMT_INT4_G128, w, packed, nonfinite, stream)


def moe_pack_mxfp4(w, packed=None, nonfinite=None, stream=None):
    return _pack("moe_pack_mxfp4", MOE_FMT_MXFP4_G32, w, packed, nonfinite, stream)


def moe_pack_nvfp4(w, packed=None, nonfinite=None, stream=None):
    return _pack("moe_pack_nvfp4", MOE_FMT_NVFP4_G16, w, packed, nonfinite, stream)


MX_EXP_RULES = {"floor": 0, "ceil": 1, "ocp": 2, "mse": 3}


def moe_pack_mxfp4_rule(w, rule, packed=None, nonfinite=None, stream=None):
    """MXFP4 packing with an exponent rule: "floor" | "ceil" | "ocp" | "mse" (or its enum value)."""
    E, N, K = w.shape
    if packed is None:
        packed = torch.empty(moe_bank_bytes(MOE_FMT_MXFP4_G32, E, N, K), dtype=torch.uint8, device=w.device)
    _check("moe_pack_mxfp4_rule",
           lib().moe_pack_mxfp4_rule(_ptr(_bits(w)), E, N, K, _ptr(packed), _ptr(nonfinite),
                                     MX_EXP_RULES.get(rule, rule), _stream(stream)))
    return packed


def moe_dequant(packed, fmt, E, N, K, out=None, stream=None):
    if out is None:
        out = torch.empty((E, N, K), dtype=torch.bfloat16, device=packed.device)
    _check("moe_dequant", lib().moe_dequant(_ptr(packed), FORMATS.get(fmt, fmt), E, N, K, _ptr(out),
                                            _stream(stream)))
    return out


def split_bank(packed, fmt, E, N, K):
    """(codes uint8 [E, N, K/2], scales) views of a packed bank (no copy)."""
    fmt = FORMATS.get(fmt, fmt)
    ncode = E * N * K // 2
    off = moe_bank_scale_offset(fmt, E, N, K)
    codes = packed[:ncode].view(E, N, K // 2)
    if fmt == MOE_FMT_INT4_G128:
        G = (K + 127) // 128
        scales = packed[off:off + E * N * G * 2].view(torch.int16).view(E, N, G)
    elif fmt == MOE_FMT_NVFP4_G16:
        # (E4M3 block scales [E, N, K/16], fp32 global scales [E])
        nsc = E * N * (K // 16)
        goff = (off + nsc + 255) // 256 * 256
        scales = (packed[off:off + nsc].view(E, N, K // 16), packed[goff:goff + 4 * E].view(torch.float32))
    else:
        scales = packed[off:off + E * N * (K // 32)].view(E, N, K // 32)
    return codes, scales


# ------------------------------------------------------------------ routing

def moe_route(logits, k, bias=None, ids=None, weights=None, stream=None):
    T, E = logits.shape
    if ids is None:
        ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    if weights is None:
        weights = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check("moe_route", lib().moe_route(_ptr(logits), _ptr(bias), T, E, k, _ptr(ids), _ptr(weights),
                                        _stream(stream)))
    return ids, weights


def moe_permute(topk_ids, E, stream=None):
    T, k = topk_ids.shape
    dev = topk_ids.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_rows = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    wsb = moe_permute_workspace_bytes(T, E, k)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    _check("moe_permute", lib().moe_permute(_ptr(topk_ids), T, E, k, _ptr(offsets), _ptr(sorted_rows), _ptr(pos),
                                            _ptr(ws), wsb, _stream(stream)))
    return offsets, sorted_rows, pos


# ------------------------------------------------------------------ forward

def alloc_workspace(shape: MoeShape, T: int, device="cuda", stream=None, flags=0):
    nbytes = moe_workspace_bytes_flags(shape, T, flags)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream=stream)
    return ws


def _opts(path, debug, events, flags=0):
    if path is None and not debug and events is None and not flags:
        return None, None
    o = ForwardOpts()
    o.path = path or MOE_PATH_AUTO
    o.flags = int(flags)
    for name, t in (debug or {}).items():
        setattr(o, name, _ptr(t))
    keep = None
    if events is not None:
        keep = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(ev.cuda_event) for ev in events])
        o.stage_events = ctypes.cast(keep, ctypes.c_void_p)
    return o, keep


def moe_forward(shape: MoeShape, x, router_w, gate_up_packed, down_packed, workspace, out=None, bias=None,
                path=None, debug=None, events=None, stream=None, flags=0):
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device=x.device)
    o, _keep = _opts(path, debug, events, flags)
    st = lib().moe_forward(ctypes.byref(shape), _ptr(_bits(x)), T, _ptr(_bits(router_w)), _ptr(bias),
                           _ptr(gate_up_packed), _ptr(down_packed), _ptr(workspace), workspace.numel(),
                           _ptr(out), ctypes.byref(o) if o is not None else None, _stream(stream))
    _check("moe_forward", st)
    return out


def moe_forward_partial(shape: MoeShape, x, router_w, expert_begin: int, num_local: int, gate_up_local, down_local,
                        workspace, partial_out=None, bias=None, path=None, debug=None, stream=None, flags=0):
    """The layer's fp32 contribution of experts [expert_begin, expert_begin + num_local)."""
    T = x.shape[0]
    if partial_out is None:
        partial_out = torch.empty((T, shape.hidden), dtype=torch.float32, device=x.device)
    o, _keep = _opts(path, debug, None, flags)
    st = lib().moe_forward_partial(ctypes.byref(shape), _ptr(_bits(x)), T, _ptr(_bits(router_w)), _ptr(bias),
                                   int(expert_begin), int(num_local), _ptr(gate_up_local), _ptr(down_local),
                                   _ptr(workspace), workspace.numel(), _ptr(partial_out),
                                   ctypes.byref(o) if o is not None else None, _stream(stream))
    _check("moe_forward_partial", st)
    return partial_out


def moe_partial_to_bf16(partial, out=None, stream=None):
    T, H = partial.shape
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=partial.device)
    _check("moe_partial_to_bf16", lib().moe_partial_to_bf16(_ptr(partial), T, H, _ptr(out), _stream(stream)))
    return out


def moe_workspace_bytes_host(shape: MoeShape, T: int) -> int:
    return lib().moe_workspace_bytes_host(ctypes.byref(shape), T)


def _host_ptr(t):
    if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
        raise ValueError("host-buffer arguments must be contiguous CPU tensors")
    return t.data_ptr()


def moe_forward_host(shape: MoeShape, x_host, router_w, gate_up_packed, down_packed, workspace, out_host,
                     bias=None, path=None, stream=None):
    """moe_forward with x_host / out_host [T, H] bf16 in (preferably pinned) host
    memory; asynchronous: out_host is valid after the stream is synchronised."""
    T = x_host.shape[0]
    o, _keep = _opts(path, None, None)
    st = lib().moe_forward_host(ctypes.byref(shape), _host_ptr(_bits(x_host)), T, _ptr(_bits(router_w)), _ptr(bias),
                                _ptr(gate_up_packed), _ptr(down_packed), _ptr(workspace), workspace.numel(),
                                _host_ptr(_bits(out_host)), ctypes.byref(o) if o is not None else None,
                                _stream(stream))
    _check("moe_forward_host", st)
    return out_host


def moe_workspace_bytes_shared(shape: MoeShape, inter_shared: int, T: int) -> int:
    return lib().moe_workspace_bytes_shared(ctypes.byref(shape), inter_shared, T)


def alloc_workspace_shared(shape: MoeShape, inter_shared: int, T: int, device="cuda", stream=None):
    nbytes = moe_workspace_bytes_shared(shape, inter_shared, T)
    ws = torch.empty(max(nbytes, 4096), dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream=stream)
    return ws


def moe_forward_shared(shape: MoeShape, shared, x, router_w, gate_up_packed, down_packed, workspace, out=None,
                       bias=None, path=None, debug=None, events=None, stream=None):
    """moe_forward plus the bf16 shared expert; shared = (gate_up [2 I_s, H], down [H, I_s], gate [H])."""
    gu_s, dn_s, gate_s = shared
    sh = SharedExpert(int(dn_s.shape[1]), _ptr(_bits(gu_s)), _ptr(_bits(dn_s)), _ptr(_bits(gate_s)))
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device=x.device)
    o, _keep = _opts(path, debug, events)
    st = lib().moe_forward_shared(ctypes.byref(shape), ctypes.byref(sh), _ptr(_bits(x)), T, _ptr(_bits(router_w)),
                                  _ptr(bias), _ptr(gate_up_packed), _ptr(down_packed), _ptr(workspace),
                                  workspace.numel(), _ptr(out), ctypes.byref(o) if o is not None else None,
                                  _stream(stream))
    _check("moe_forward_shared", st)
    return out


def moe_forward_routed(shape: MoeShape, x, topk_ids, topk_w, gate_up_packed, down_packed, workspace, out=None,
                       path=None, debug=None, events=None, stream=None, flags=0):
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device=x.device)
    o, _keep = _opts(path, debug, events, flags)
    st = lib().moe_forward_routed(ctypes.byref(shape), _ptr(_bits(x)), T, _ptr(topk_ids), _ptr(topk_w),
                                  _ptr(gate_up_packed), _ptr(down_packed), _ptr(workspace), workspace.numel(),
                                  _ptr(out), ctypes.byref(o) if o is not None else None, _stream(stream))
    _check("moe_forward_routed", st)
    return out


def moe_forward_launch_count(shape: MoeShape, T: int, path=MOE_PATH_AUTO, routed=False) -> int:
    return lib().moe_forward_launch_count(ctypes.byref(shape), T, path, int(routed))


def moe_forward_shared_launch_count(shape: MoeShape, inter_shared: int, T: int, path=MOE_PATH_AUTO) -> int:
    return lib().moe_forward_shared_launch_count(ctypes.byref(shape), inter_shared, T, path)


def moe_noalloc_scratch_bytes() -> int:
    return lib().moe_noalloc_scratch_bytes()


def moe_forward_noalloc(shape: MoeShape, x, router_w, gate_up_packed, down_packed, out=None, bias=None,
                        stream=None):
    """moe_forward on the library's fixed scratch array (no workspace argument)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, shape.hidden), dtype=torch.bfloat16, device=x.device)
    st = lib().moe_forward_noalloc(ctypes.byref(shape), _ptr(_bits(x)), T, _ptr(_bits(router_w)), _ptr(bias),
                                   _ptr(gate_up_packed), _ptr(down_packed), _ptr(out), _stream(stream))
    _check("moe_forward_noalloc", st)
    return out


def moe_noalloc_status(stream=None) -> int:
    """Synchronises the stream; MOE_ERR_TIMEOUT if a no-alloc call's bounded
    device wait expired since the last report (the report clears it), else MOE_OK."""
    return lib().moe_noalloc_status(_stream(stream))


def moe_workspace_init(workspace, stream=None):
    _check("moe_workspace_init", lib().moe_workspace_init(_ptr(workspace), workspace.numel(), _stream(stream)))


def moe_workspace_status(workspace, stream=None) -> int:
    """Synchronises the stream; returns the status code (MOE_OK or MOE_ERR_TIMEOUT)."""
    return lib().moe_workspace_status(_ptr(workspace), workspace.numel(), _stream(stream))


def moe_selftest_bounded_wait(workspace, limit_ns: int, stream=None):
    """workspace None: the status word of the no-alloc scratch array on the current device."""
    _check("moe_selftest_bounded_wait",
           lib().moe_selftest_bounded_wait(_ptr(workspace), 0 if workspace is None else workspace.numel(),
                                           int(limit_ns), _stream(stream)))
