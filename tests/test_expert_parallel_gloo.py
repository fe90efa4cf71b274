"""Expert-parallel layer: the host-side exchange as CPU processes over gloo.

ExpertParallelLayer gathers the ranks' tokens, has every rank compute the
contribution of its own block of experts, and sums the contributions back to
the ranks that own the tokens.  Here the per-rank contribution is computed by
the CPU oracle (the layer with the weights of non-local slots set to zero),
so these tests check the partition of the experts and the movement of tokens
and partial sums; the kernels' own expert restriction is checked on the GPU
(test_gpu_expert_parallel.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import moe_synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_range_partitions_the_experts():
    from weight_only_bit_router_b200.expert_parallel import expert_range
    for E in (8, 256, 255, 1024, 3):
        for world in range(1, min(E, 9) + 1):
            ranges = [expert_range(E, r, world) for r in range(world)]
            assert ranges[0][0] == 0
            for (b0, n0), (b1, _) in zip(ranges, ranges[1:]):
                assert b0 + n0 == b1
            assert sum(n for _, n in ranges) == E
            assert max(n for _, n in ranges) - min(n for _, n in ranges) <= 1
    with pytest.raises(ValueError):
        expert_range(4, 0, 5)


def oracle_partial(layer, x_bits, begin, count):
    """The oracle's fp64 layer output restricted to experts [begin, begin + count)."""
    from oracle import moe_oracle as o
    s = layer.shape
    gu = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(layer.gate_up))
    dn = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(layer.down))
    logits = o.router_logits(x_bits, moe_synth.bf16_bits(layer.router_w))
    ids, w = o.route(logits, None, s.top_k)
    local = (ids >= begin) & (ids < begin + count)
    out, _ = o.forward_routed(x_bits, ids, np.where(local, w, 0.0), gu, dn, s.num_experts)
    return out


def _worker(rank, world, port, T_local, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import weight_only_bit_router_b200 as moe
        from oracle import moe_oracle as o
        from weight_only_bit_router_b200.expert_parallel import ExpertParallelLayer
        s = moe_synth.TINY
        layer = moe_synth.make_layer(s, T=world * T_local, seed=11)   # the same weights on every rank
        x_local = layer.x[rank * T_local:(rank + 1) * T_local]        # this rank's tokens
        shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "int4_g128")
        calls = []

        def partial_fn(x_all):
            calls.append(x_all.shape[0])
            part = oracle_partial(layer, moe_synth.bf16_bits(x_all), ep.expert_begin, ep.num_local)
            return torch.from_numpy(part.astype(np.float32))

        def finalize_fn(p):
            return torch.from_numpy(o.f64_to_bf16(p.numpy().astype(np.float64)).view(np.int16)).view(torch.bfloat16)

        ep = ExpertParallelLayer(shape, layer.router_w, None, None, partial_fn=partial_fn, finalize_fn=finalize_fn)
        out = ep.forward(x_local)
        ref = oracle_partial(layer, moe_synth.bf16_bits(layer.x), 0, s.num_experts)[rank * T_local:(rank + 1) * T_local]
        q.put((rank, ep.expert_begin, ep.num_local, calls, out.float().numpy().astype(np.float64), ref))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2])
def test_two_ranks_sum_to_the_full_layer(world):
    T_local = 5
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, T_local, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    covered = []
    for rank, begin, count, calls, out, ref in res:
        assert calls == [world * T_local]            # every rank routed all gathered tokens
        covered.extend(range(begin, begin + count))
        rms = np.sqrt(np.mean(ref ** 2))
        assert np.all(np.abs(out - ref) <= 1e-2 * np.abs(ref) + 1e-3 * rms), f"rank {rank}"
    assert covered == list(range(moe_synth.TINY.num_experts))   # the ranks' experts partition E
