"""Expert-parallel shards of the layer on one GPU (needs a B200).

moe_forward_partial computes, for a contiguous block of experts held in its
own packed banks, the fp32 contribution of those experts with the routing of
all E experts.  Here every shard of a partition of the experts runs on the
same GPU in turn (the ranks of an expert-parallel group, one after another),
the contributions are summed and rounded once by moe_partial_to_bf16, and the
result is checked against moe_forward on the whole banks and against the
pure oracle (test_gpu_parity's rule).  Both kernel paths, uneven blocks, a
shard that no token routes to, and every format.
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from oracle import moe_oracle as o
from parity_util import assert_out_close
from test_gpu_parity import DEV, PACKERS, run_forward, verify_layer
from weight_only_bit_router_b200.expert_parallel import expert_range

pytestmark = pytest.mark.gpu


def sharded_forward(layer, fmt, blocks, path=None, flags=0):
    """Sum of moe_forward_partial over the expert blocks [(begin, count)], rounded once."""
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    T = layer.x.shape[0]
    ws = moe.alloc_workspace(shape, T, flags=flags)
    total = torch.zeros(T, s.hidden, dtype=torch.float32, device=DEV)
    for begin, count in blocks:
        gu = PACKERS[fmt](layer.gate_up[begin:begin + count].contiguous())
        dn = PACKERS[fmt](layer.down[begin:begin + count].contiguous())
        part = moe.moe_forward_partial(shape, layer.x, layer.router_w, begin, count, gu, dn, ws, bias=layer.bias,
                                       path=path, flags=flags)
        assert moe.moe_workspace_status(ws) == moe.MOE_OK
        total += part
    return moe.moe_partial_to_bf16(total)


def check_sharded(layer, fmt, blocks, path=None, sample=None, name="", flags=0):
    ep = sharded_forward(layer, fmt, blocks, path, flags)
    full, dbg = run_forward(layer, fmt, path)
    # against moe_forward: the same kernels, only the fp32 summation order differs
    assert_out_close(ep, full.float().cpu().numpy().astype(np.float64), f"{name}: shards vs whole banks")
    # against the pure oracle, with moe_forward's routing and activations
    verify_layer(layer, fmt, ep, dbg, path, sample, name=name)


@pytest.mark.parametrize("fmt", ["int4_g128", "mxfp4", "nvfp4"])
def test_two_shards_decode_path(fmt):
    layer = moe_synth.make_layer(moe_synth.NEX, T=8, seed=2008, device=DEV)
    blocks = [expert_range(256, r, 2) for r in range(2)]
    check_sharded(layer, fmt, blocks, name=f"ep2_{fmt}_T8")


def test_uneven_shards_and_an_empty_one_decode_path():
    layer = moe_synth.make_layer(moe_synth.NEX, T=4, seed=2004, device=DEV)
    logits = o.router_logits(moe_synth.bf16_bits(layer.x), moe_synth.bf16_bits(layer.router_w))
    ids, _ = o.route(logits, None, 8)
    used = set(int(e) for e in ids.ravel())
    idle = next(e for e in range(256) if e not in used)     # an expert no token routes to
    blocks = [(0, idle), (idle, 1), (idle + 1, 256 - idle - 1)] if idle > 0 else [(0, 1), (1, 255)]
    blocks = [(b, n) for b, n in blocks if n > 0]
    check_sharded(layer, "int4_g128", blocks, name="ep_uneven_T4")


@pytest.mark.parametrize("world,flags", [(2, 0), (4, 0), (2, moe.MOE_FLAG_DETERMINISTIC)])
def test_shards_grouped_path(world, flags):
    layer = moe_synth.make_layer(moe_synth.NEX, T=300, seed=2300 + world, device=DEV)
    blocks = [expert_range(256, r, world) for r in range(world)]
    sample = np.random.default_rng(world).choice(300, 16, replace=False)
    check_sharded(layer, "int4_g128", blocks, moe.MOE_PATH_PREFILL, sample=sample, name=f"ep{world}_T300_f{flags}",
                  flags=flags)


def test_shards_tiny_layer_both_paths():
    layer = moe_synth.make_layer(moe_synth.TINY, T=16, seed=3, device=DEV)
    for path in (moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL):
        check_sharded(layer, "int4_g128", [(0, 3), (3, 5)], path, name=f"ep_tiny_path{path}")


def test_partial_rejects_ranges_outside_the_layer():
    layer = moe_synth.make_layer(moe_synth.TINY, T=4, seed=4, device=DEV)
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "int4_g128")
    gu = moe.moe_pack_int4_g128(layer.gate_up[6:].contiguous())
    dn = moe.moe_pack_int4_g128(layer.down[6:].contiguous())
    ws = moe.alloc_workspace(shape, 4)
    for begin, count in ((6, 3), (-1, 2), (2, 0)):
        with pytest.raises(moe.MoeError):
            moe.moe_forward_partial(shape, layer.x, layer.router_w, begin, count, gu, dn, ws)
