"""The allocation-free forward entry point (collected last on purpose).

moe_forward_noalloc serves callers that cannot allocate device memory, such
as work recorded ahead of time and replayed later (a captured CUDA graph or a
pre-built command buffer) and runtimes that reserve their memory budget up
front.  It runs the same layer on a fixed scratch array inside the library.
These tests call it through the C ABI and check that its output matches the
regular moe_forward (which uses a caller-provided workspace) within the layer
tolerance, on two calls in a row, and that oversized batches are refused.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from parity_util import assert_out_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("fmt,T,zipf", [("int4_g128", 4, False), ("mxfp4", 32, True)])
def test_noalloc_forward_matches_workspace_forward_twice(fmt, T, zipf):
    s = moe_synth.NEX
    layer = moe_synth.make_layer(s, T=T, seed=77 + T, zipf=zipf, device=DEV)
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    pack = moe.moe_pack_int4_g128 if fmt == "int4_g128" else moe.moe_pack_mxfp4
    gu, dn = pack(layer.gate_up), pack(layer.down)
    ws = moe.alloc_workspace(shape, T)
    ref = moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, ws, bias=layer.bias)
    torch.cuda.synchronize()
    ref64 = ref.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full((T, s.hidden), float("nan"), dtype=torch.bfloat16, device=DEV)
        st = moe.lib().moe_forward_noalloc(ctypes.byref(shape), layer.x.data_ptr(), T,
                                           layer.router_w.data_ptr(),
                                           None if layer.bias is None else layer.bias.data_ptr(),
                                           gu.data_ptr(), dn.data_ptr(), out.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
        assert st == moe.MOE_OK
        torch.cuda.synchronize()
        assert_out_close(out, ref64, f"no-alloc vs workspace forward ({fmt}, T={T})")


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
    assert st == 2  # MOE_ERR_UNSUPPORTED
    assert torch.count_nonzero(out) == 0
