"""The single-kernel decode layer (MOE_PATH_FUSED, T <= 8) against the CPU oracle, through the
C ABI (needs a B200): odd shapes, more experts than CTAs, every expert
selected, the given-routing entry point, and back-to-back launches that reuse
one workspace's device counters (eagerly and inside a replayed CUDA graph).
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from test_gpu_parity import DEV, check_layer, pack_gpu, run_forward

FMTS = ["int4_g128", "mxfp4"]  # NVFP4 banks run on the three-kernel decode path

pytestmark = pytest.mark.gpu


def shape_of(layer, fmt):
    s = layer.shape
    return moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)


FUSED = moe.MOE_PATH_FUSED


def test_single_kernel_path_launch_counts():
    s = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    for T in (1, 4, 8):
        assert moe.moe_forward_launch_count(s, T, FUSED, 0) == 1
        assert moe.moe_forward_launch_count(s, T, FUSED, 1) == 1
    assert moe.moe_forward_launch_count(s, 9, FUSED, 0) == -1   # above the path's token limit
    assert moe.moe_forward_launch_count(moe.make_shape(2048, 512, 256, 8, "nvfp4"), 4, FUSED, 0) == -1


def test_single_kernel_path_rejects_nvfp4():
    layer = moe_synth.make_layer(moe_synth.TINY, T=4, seed=3, device=DEV)
    with pytest.raises(moe.MoeError):
        run_forward(layer, "nvfp4", FUSED)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("T", [2, 8])
def test_fused_tiny_layer(fmt, T):
    layer = moe_synth.make_layer(moe_synth.TINY, T=T, seed=300 + T, device=DEV)
    check_layer(layer, fmt, FUSED)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("T", [5, 8])
def test_fused_odd_shape_partial_blocks(fmt, T):
    """H = 320 (2.5 k-blocks of 128, a last INT4 group of 64) and I = 192."""
    shape = moe_synth.LayerShape(hidden=320, inter=192, num_experts=6, top_k=3)
    layer = moe_synth.make_layer(shape, T=T, seed=310 + T, device=DEV)
    check_layer(layer, fmt, FUSED)


def test_fused_more_experts_than_ctas_and_top32():
    """E = 1024 (seven router experts per CTA), k = 32: up to 256 touched slots."""
    shape = moe_synth.LayerShape(hidden=256, inter=64, num_experts=1024, top_k=32)
    layer = moe_synth.make_layer(shape, T=8, seed=320, device=DEV)
    check_layer(layer, "int4_g128", FUSED)


def test_fused_every_expert_selected():
    """k = E: the softmax runs over all experts and every expert sees every token."""
    shape = moe_synth.LayerShape(hidden=128, inter=64, num_experts=4, top_k=4)
    layer = moe_synth.make_layer(shape, T=8, seed=330, device=DEV)
    check_layer(layer, "mxfp4", FUSED)


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_nex_t8(fmt):
    layer = moe_synth.make_layer(moe_synth.NEX, T=8, seed=340, zipf=True, device=DEV)
    check_layer(layer, fmt, FUSED)


def test_fused_routed_is_bit_identical_to_routing_in_kernel():
    layer = moe_synth.make_layer(moe_synth.NEX, T=4, seed=350, device=DEV)
    out, dbg = run_forward(layer, "int4_g128", FUSED)
    out2, dbg2 = run_forward(layer, "int4_g128", FUSED, routed=(dbg["topk_ids_out"], dbg["topk_w_out"]))
    assert torch.equal(out, out2)
    assert torch.equal(dbg["act_out"], dbg2["act_out"])
    assert torch.equal(dbg["sorted_rows_out"], dbg2["sorted_rows_out"])


def test_fused_back_to_back_launches_and_graph_replay():
    """Many launches on one workspace, without host synchronisation between
    them: every launch must leave the device counters at zero for the next."""
    layers = [moe_synth.make_layer(moe_synth.NEX, T=4, seed=360 + i, device=DEV) for i in range(3)]
    fmt = "int4_g128"
    shape = shape_of(layers[0], fmt)
    packed = [(pack_gpu(fmt, L.gate_up), pack_gpu(fmt, L.down)) for L in layers]
    ws = moe.alloc_workspace(shape, 4)
    ref = [moe.moe_forward(shape, L.x, L.router_w, gu, dn, ws, path=FUSED).clone()
           for L, (gu, dn) in zip(layers, packed)]
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    outs = [torch.empty_like(r) for r in ref]

    def seq():
        for _ in range(5):
            for i, (L, (gu, dn)) in enumerate(zip(layers, packed)):
                moe.moe_forward(shape, L.x, L.router_w, gu, dn, ws, out=outs[i], path=FUSED,
                                stream=torch.cuda.current_stream())

    seq()
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    for o_, r in zip(outs, ref):
        assert torch.equal(o_, r)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            seq()
    torch.cuda.current_stream().wait_stream(s)
    for o_ in outs:
        o_.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    for o_, r in zip(outs, ref):
        assert torch.equal(o_, r)
    # the outputs agree with the oracle (first layer)
    check_layer(layers[0], fmt, FUSED)
