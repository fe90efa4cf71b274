"""Multi-rank host logic of the benchmark on CPU: world_size 2 over gloo.

The layer forward shards by data parallelism only (each rank runs its own
replica on its own tokens); the one collective is the max-over-ranks of the
timed region.  These tests run that plumbing as two CPU processes.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    r, local, w = bench.dist_init("gloo")
    assert (r, local, w) == (rank, rank, world)
    # per-rank token seeds differ (weak scaling: each rank its own tokens)
    seeds = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    torch.distributed.all_gather(seeds, torch.tensor([bench.rank_token_seed(rank, 4)]))
    # the timed region is the slowest rank's
    m = bench.reduce_max(10.0 + 5.0 * rank, "cpu")
    bench.barrier()
    q.put((rank, m, [int(s) for s in seeds]))
    torch.distributed.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_and_distinct_token_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [m for _, m, _ in res] == [15.0, 15.0]
    seeds = res[0][2]
    assert len(set(seeds)) == world


def test_single_process_helpers_are_identities():
    import bench
    assert bench.reduce_max(3.5, "cpu") == 3.5
    bench.barrier()
    assert bench.dist_env() == (0, 0, 1) or "RANK" in os.environ
