"""C ABI checks that need no GPU: the library loads, exports every entry point
include/moe_w4a16.h declares, answers size queries, and rejects bad arguments
on the host before touching the device."""
import ctypes
import os
import re

import pytest

import moe_synth
import weight_only_bit_router_b200 as moe
from conftest import ROOT
from oracle import moe_oracle as o

HEADER = os.path.join(ROOT, "include", "moe_w4a16.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_library_loads_and_reports_abi_version():
    assert moe.moe_abi_version() == 2


def test_every_declared_symbol_is_exported_and_bound():
    names = declared_functions()
    assert len(names) >= 15
    handle = moe.lib()
    for n in names:
        assert hasattr(handle, n), n
    assert sorted(moe.exported_symbols()) == names


def test_status_strings():
    assert moe.moe_status_str(0) == "ok"
    assert "timeout" in moe.moe_status_str(5) or "expired" in moe.moe_status_str(5)


@pytest.mark.parametrize("fmt", ["int4_g128", "mxfp4", "nvfp4"])
def test_bank_sizes_match_closed_form(fmt):
    s = moe.make_shape(2048, 512, 256, 8, fmt)
    gu, dn = moe.moe_packed_bytes(s, 0), moe.moe_packed_bytes(s, 1)
    ofmt = {"int4_g128": o.FMT_INT4, "mxfp4": o.FMT_MXFP4, "nvfp4": o.FMT_NVFP4}[fmt]
    per_expert = o.packed_bytes_per_expert(ofmt, 2048, 512)
    # 256-byte alignment pads (codes -> scales, and for NVFP4 scales -> global scales, per bank)
    pads = 4 if fmt == "nvfp4" else 2
    assert 0 <= gu + dn - 256 * per_expert < pads * 256
    assert moe.moe_packed_bytes(s, 2) == 0
    assert moe.moe_bank_scale_offset(fmt, 256, 1024, 2048) == 256 * 1024 * 1024


def test_bank_bytes_rejects_bad_sizes():
    assert moe.moe_bank_bytes("int4_g128", 1, 1, 48) == 0   # K % 32 != 0
    assert moe.moe_bank_bytes("int4_g128", 0, 1, 64) == 0
    assert moe.moe_bank_bytes(7, 1, 1, 64) == 0


def test_workspace_bytes_grow_with_tokens_and_reject_bad_shapes():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    a, b = moe.moe_workspace_bytes(s, 1), moe.moe_workspace_bytes(s, 8192)
    assert 0 < a < b
    assert moe.moe_workspace_bytes(s, -1) == 0
    assert moe.moe_workspace_bytes(moe.make_shape(2000, 512, 256, 8, "int4_g128"), 4) == 0
    assert moe.moe_workspace_bytes(moe.make_shape(2048, 512, 256, 33, "int4_g128"), 4) == 0


def _c(fn, *args):
    return getattr(moe.lib(), fn)(*args)


def test_pack_rejects_null_and_bad_k_without_a_gpu():
    L = moe.lib()
    assert L.moe_pack_int4_g128(None, 1, 1, 64, 256, None, None) == 1
    assert L.moe_pack_mxfp4(16, 1, 1, 48, 256, None, None) == 1        # K % 32
    assert L.moe_pack_mxfp4(16, 1, 1, 64, 255, None, None) == 1        # misaligned output
    assert L.moe_dequant(None, 1, 1, 1, 64, 16, None) == 1


def test_new_packers_reject_bad_arguments_without_a_gpu():
    L = moe.lib()
    assert L.moe_pack_nvfp4(None, 1, 1, 64, 256, None, None) == 1
    assert L.moe_pack_nvfp4(16, 1, 1, 48, 256, None, None) == 1        # K % 32
    assert L.moe_pack_mxfp4_rule(16, 1, 1, 64, 256, None, 4, None) == 1  # unknown rule
    assert L.moe_pack_mxfp4_rule(16, 1, 1, 64, 255, None, 3, None) == 1  # misaligned output
    assert L.moe_bank_bytes(3, 1, 1, 48) == 0                           # NVFP4 K % 32


def test_forward_shared_validation_happens_on_the_host():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    ws_plain = moe.moe_workspace_bytes(s, 4)
    ws_sh = moe.moe_workspace_bytes_shared(s, 512, 4)
    assert ws_sh > ws_plain
    assert moe.moe_workspace_bytes_shared(s, 500, 4) == 0               # I_s % 64
    assert moe.moe_workspace_bytes_shared(s, 0, 4) == 0
    L = moe.lib()
    sh = moe.SharedExpert(512, 256, 256, 256)
    def call(shared=ctypes.byref(sh), ws=4096, wsb=None, opts=None, T=4):
        return L.moe_forward_shared(ctypes.byref(s), shared, 256, T, 256, None, 256, 512, ws,
                                    ws_sh if wsb is None else wsb, 256, opts, None)
    assert call(shared=None) == 1
    assert call(wsb=ws_plain) == 3                                       # the routed workspace is too small
    assert call(wsb=ws_sh - 1) == 3                                      # one byte short of the shared part
    bad = moe.SharedExpert(96, 256, 256, 256)
    assert call(shared=ctypes.byref(bad)) == 2                           # I_s not a multiple of 64
    unaligned = moe.SharedExpert(512, 258, 256, 256)
    assert call(shared=ctypes.byref(unaligned)) == 1
    o = moe.ForwardOpts()
    o.path = 3
    assert call(opts=ctypes.byref(o)) == 1                               # unknown path
    assert call(T=0) == 0                                                # nothing to do


def test_route_and_permute_validation():
    L = moe.lib()
    assert L.moe_route(16, None, 4, 256, 33, 16, 16, None) == 2        # k > 32
    assert L.moe_route(16, None, 4, 8, 9, 16, 16, None) == 2           # k > E
    assert L.moe_route(16, None, -1, 8, 2, 16, 16, None) == 1
    assert L.moe_route(None, None, 0, 8, 2, None, None, None) == 0      # T == 0 is a no-op
    assert L.moe_permute(16, 4, 2000, 2, 256, 256, 256, 256, 1 << 20, None) == 2
    assert L.moe_permute(16, 4, 8, 2, 256, 256, 256, None, 0, None) == 3


def test_forward_validation_happens_on_the_host():
    L = moe.lib()
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    ws = moe.moe_workspace_bytes(s, 4)
    args = lambda **kw: [ctypes.byref(kw.get("shape", s)), kw.get("x", 256), kw.get("T", 4), kw.get("r", 256),
                         None, kw.get("gu", 256), kw.get("dn", 256), kw.get("ws", 256), kw.get("wsb", ws),
                         kw.get("out", 256), None, None]
    assert L.moe_forward(*args(x=None)) == 1
    assert L.moe_forward(*args(x=8)) == 1                  # x not 16-byte aligned
    assert L.moe_forward(*args(gu=512 + 16)) == 1          # packed bank not 256-byte aligned
    assert L.moe_forward(*args(ws=None)) == 3
    assert L.moe_forward(*args(wsb=ws - 1)) == 3
    assert L.moe_forward(*args(T=-2)) == 1
    assert L.moe_forward(*args(shape=moe.make_shape(2048, 500, 256, 8, "int4_g128"))) == 2
    assert L.moe_forward(*args(shape=moe.make_shape(2048, 512, 256, 8, 4))) == 1   # unknown format
    assert L.moe_forward(*args(r=None)) == 1
    opts = moe.ForwardOpts()
    opts.path = 9
    a = args()
    a[10] = ctypes.byref(opts)
    assert L.moe_forward(*a) == 1
    # T == 0 is a valid no-op
    assert L.moe_forward(*args(T=0)) == 0
    assert moe.moe_forward_launch_count(s, 4, 3, False) == -1     # unknown path


def test_launch_counts_with_and_without_the_folded_shared_expert():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    dec, pre = moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL
    # decode: split-K routing GEMV + finalize, gate_up, down (with the combine)
    assert moe.moe_forward_launch_count(s, 4, dec, False) == 4
    # the shared expert rides those four kernels up to I_s = 512 on the decode path
    for T in (1, 4, 32):
        assert moe.moe_forward_shared_launch_count(s, 512, T, dec) == moe.moe_forward_launch_count(s, T, dec, False)
    assert moe.moe_forward_shared_launch_count(s, 448, 8, moe.MOE_PATH_AUTO) == 4
    # its own three kernels elsewhere: larger I_s, the grouped path, more than 32 tokens
    assert moe.moe_forward_shared_launch_count(s, 640, 4, dec) == 4 + 3
    assert (moe.moe_forward_shared_launch_count(s, 512, 16, pre)
            == moe.moe_forward_launch_count(s, 16, pre, False) + 3)
    assert (moe.moe_forward_shared_launch_count(s, 512, 64, moe.MOE_PATH_AUTO)
            == moe.moe_forward_launch_count(s, 64, moe.MOE_PATH_AUTO, False) + 3)
    assert moe.moe_forward_shared_launch_count(s, 96, 4, dec) == -1   # I_s not a multiple of 64
    assert moe.moe_forward_shared_launch_count(s, 512, 64, dec) == -1  # no decode path above 32 tokens


def test_shared_workspace_holds_the_folded_partials():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    for T in (1, 4, 32):
        extra = moe.moe_workspace_bytes_shared(s, 512, T) - moe.moe_workspace_bytes(s, T)
        # activation, gate and the routing GEMV's 8 split partials of 1,025 rows per token
        assert extra >= T * 512 * 2 + T * 4 + 8 * T * (2 * 512 + 1) * 4
        # and the own-kernel form's down product [T, H]
        assert extra >= T * 512 * 2 + T * 4 + T * 2048 * 4


def test_workspace_query_with_flags():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    base = moe.moe_workspace_bytes(s, 8192)
    assert moe.moe_workspace_bytes_flags(s, 8192, 0) == base
    assert moe.moe_workspace_bytes_flags(s, 8192, moe.MOE_FLAG_DETERMINISTIC) >= base + 8192 * 8 * 2048 * 4
    # the grouped path may be chosen at any T: the flag adds the per-row buffer at 32 tokens too
    assert (moe.moe_workspace_bytes_flags(s, 32, moe.MOE_FLAG_DETERMINISTIC)
            >= moe.moe_workspace_bytes(s, 32) + 32 * 8 * 2048 * 4)
    assert moe.moe_workspace_bytes_flags(s, 4, 2) == 0          # unknown flag
    assert moe.moe_workspace_bytes_host(s, 4) >= moe.moe_workspace_bytes(s, 4) + 2 * 4 * 2048 * 2


def test_partial_and_host_validation():
    L = moe.lib()
    s = moe.make_shape(256, 64, 8, 2, "int4_g128")
    wsb = moe.moe_workspace_bytes(s, 4)
    part = lambda b, n, **kw: L.moe_forward_partial(ctypes.byref(s), 256, 4, 256, None, b, n, 256, 256, 256, wsb,
                                                   kw.get("out", 256), None, None)
    assert part(6, 3) == 1           # the range leaves the layer's experts
    assert part(-1, 2) == 1
    assert part(2, 0) == 1
    assert part(0, 8, out=None) == 1
    assert L.moe_partial_to_bf16(None, 4, 256, 256, None) == 1
    assert L.moe_partial_to_bf16(256, 4, 250, 256, None) == 1   # H not a multiple of 4
    assert L.moe_partial_to_bf16(None, 0, 256, None, None) == 0
    assert L.moe_forward_host(ctypes.byref(s), None, 4, 256, None, 256, 256, 256, 1 << 20, 256, None, None) == 1
    assert L.moe_forward_host(ctypes.byref(s), 256, 4, 256, None, 256, 256, 256, 16, 256, None, None) == 3


def test_routed_forward_validation():
    L = moe.lib()
    s = moe.make_shape(256, 64, 8, 2, "mxfp4")
    ws = moe.moe_workspace_bytes(s, 16)
    assert L.moe_forward_routed(ctypes.byref(s), 256, 16, None, 256, 256, 256, 256, ws, 256, None, None) == 1


def test_workspace_status_validation():
    L = moe.lib()
    assert L.moe_workspace_status(None, 256, None) == 3
    assert L.moe_workspace_init(256, 100, None) == 3
    assert L.moe_selftest_bounded_wait(256, 256, 11 * 10**9, None) == 1
    assert L.moe_selftest_bounded_wait(None, 0, 11 * 10**9, None) == 1
    assert L.moe_selftest_bounded_wait(256, 100, 1000, None) == 3


def test_noalloc_validation_happens_before_anything_is_enqueued():
    """Argument errors of moe_forward_noalloc come back before it touches
    the device (no GPU here: a call that got past the checks would fail with
    MOE_ERR_CUDA instead)."""
    L = moe.lib()
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    args = lambda **kw: [ctypes.byref(kw.get("shape", s)), kw.get("x", 256), kw.get("T", 4), kw.get("r", 256),
                         kw.get("bias", None), kw.get("gu", 256), kw.get("dn", 256), kw.get("out", 256), None]
    assert L.moe_forward_noalloc(*args(x=None)) == 1
    assert L.moe_forward_noalloc(*args(x=8)) == 1
    assert L.moe_forward_noalloc(*args(r=None)) == 1
    assert L.moe_forward_noalloc(*args(bias=2)) == 1       # bias not 4-byte aligned
    assert L.moe_forward_noalloc(*args(gu=512 + 16)) == 1
    assert L.moe_forward_noalloc(*args(out=None)) == 1
    assert L.moe_forward_noalloc(*args(T=-1)) == 1
    assert L.moe_forward_noalloc(*args(shape=moe.make_shape(2048, 500, 256, 8, "int4_g128"))) == 2
    assert L.moe_forward_noalloc(*args(T=8192)) == 2       # workspace beyond the fixed scratch
    assert L.moe_forward_noalloc(*args(T=0)) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    w = moe_synth.gate_up_bank(moe_synth.TINY, seed=0)
    with pytest.raises(ValueError):
        moe.moe_pack_int4_g128(w, packed=torch.empty(10, dtype=torch.uint8))
