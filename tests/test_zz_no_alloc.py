"""The allocation-free forward entry point (collected last on purpose).

moe_forward_noalloc serves callers that may not allocate device memory while
they issue work: runtimes that reserve their whole memory budget at start-up,
plugins whose host framework owns the allocator, and code that records its
GPU work for later replay.  It runs the same layer on a fixed scratch array
inside the library.  These tests call it through the C ABI and check:
  * its output against the regular moe_forward (caller-provided workspace) on
    two calls in a row: bit-identical on the deterministic decode path, within
    the layer tolerance on the grouped path (its fp32 combine is order-
    dependent);
  * its output against the CPU oracle on the tiny layer;
  * that a bounded-wait timeout recorded in the array survives a later call
    and is reported (then cleared) by moe_noalloc_status;
  * that batches whose workspace exceeds the array are refused.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from oracle import moe_oracle as o
from parity_util import assert_out_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
PACK = {"int4_g128": moe.moe_pack_int4_g128, "mxfp4": moe.moe_pack_mxfp4, "nvfp4": moe.moe_pack_nvfp4}


def noalloc_call(shape, layer, gu, dn, out):
    """moe_forward_noalloc through the C ABI (ctypes, raw device pointers)."""
    T = layer.x.shape[0]
    return moe.lib().moe_forward_noalloc(ctypes.byref(shape), layer.x.data_ptr(), T, layer.router_w.data_ptr(),
                                         None if layer.bias is None else layer.bias.data_ptr(), gu.data_ptr(),
                                         dn.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def setup(fmt, T, seed, zipf=False, s=moe_synth.NEX):
    layer = moe_synth.make_layer(s, T=T, seed=seed, zipf=zipf, device=DEV)
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    gu, dn = PACK[fmt](layer.gate_up), PACK[fmt](layer.down)
    ws = moe.alloc_workspace(shape, T)
    ref = moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, ws, bias=layer.bias)
    torch.cuda.synchronize()
    return layer, shape, gu, dn, ref


@pytest.mark.parametrize("fmt,T,zipf", [("int4_g128", 4, False), ("mxfp4", 32, True), ("nvfp4", 1, False)])
def test_noalloc_decode_path_equals_workspace_forward_twice(fmt, T, zipf):
    layer, shape, gu, dn, ref = setup(fmt, T, 77 + T, zipf)
    assert moe.moe_workspace_bytes(shape, T) <= moe.moe_noalloc_scratch_bytes()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"no-alloc and workspace forward differ ({fmt}, T={T})"
    assert moe.moe_noalloc_status() == moe.MOE_OK


def test_noalloc_grouped_path_matches_workspace_forward_twice():
    """64 tokens take the grouped tcgen05 GEMMs; their workspace still fits the array."""
    T = 64
    layer, shape, gu, dn, ref = setup("int4_g128", T, 164)
    assert moe.moe_workspace_bytes(shape, T) <= moe.moe_noalloc_scratch_bytes()
    ref64 = ref.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK
        torch.cuda.synchronize()
        assert_out_close(out, ref64, "no-alloc vs workspace forward (grouped path, T=64)")
    assert moe.moe_noalloc_status() == moe.MOE_OK


def test_noalloc_tiny_layer_against_the_oracle():
    s = moe_synth.TINY
    layer, shape, gu, dn, _ = setup("int4_g128", 16, moe_synth.SEED_TINY, s=s)
    out = torch.full((16, s.hidden), float("nan"), dtype=torch.bfloat16, device=DEV)
    assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK
    torch.cuda.synchronize()
    ob = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(layer.gate_up.cpu()))
    db = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(layer.down.cpu()))
    r = o.forward(moe_synth.bf16_bits(layer.x), moe_synth.bf16_bits(layer.router_w), None, ob, db, s.top_k)
    assert_out_close(out, r["out"], "no-alloc vs oracle (tiny layer)")


def test_noalloc_refuses_batches_beyond_its_scratch():
    s = moe_synth.NEX
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "int4_g128")
    T = 8192
    assert moe.moe_workspace_bytes(shape, T) > moe.moe_noalloc_scratch_bytes()
    x = torch.zeros(T, s.hidden, dtype=torch.bfloat16, device=DEV)
    r = torch.zeros(s.num_experts, s.hidden, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros(T, s.hidden, dtype=torch.bfloat16, device=DEV)
    gu = torch.zeros(moe.moe_packed_bytes(shape, 0), dtype=torch.uint8, device=DEV)
    dn = torch.zeros(moe.moe_packed_bytes(shape, 1), dtype=torch.uint8, device=DEV)
    st = moe.lib().moe_forward_noalloc(ctypes.byref(shape), x.data_ptr(), T, r.data_ptr(), None, gu.data_ptr(),
                                       dn.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == moe.MOE_ERR_UNSUPPORTED
    assert torch.count_nonzero(out) == 0


def test_noalloc_timeout_survives_a_later_call_and_is_reported_once():
    layer, shape, gu, dn, ref = setup("int4_g128", 4, 81)
    out = torch.empty_like(ref)
    assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK   # the array is set up on this device
    moe.moe_selftest_bounded_wait(None, 20_000_000)                 # 20 ms wait on the array's status word
    assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK   # a later call does not erase it
    assert moe.moe_noalloc_status() == moe.MOE_ERR_TIMEOUT
    assert moe.moe_noalloc_status() == moe.MOE_OK                   # reading clears it
    out.fill_(float("nan"))
    assert noalloc_call(shape, layer, gu, dn, out) == moe.MOE_OK
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
