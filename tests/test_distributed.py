"""Multi-rank plumbing of the benchmark on CPU (gloo, world size 2).

The decode path needs no collective: every transformer block is an
independent stream with its own code ("Dekompresi per transformer block"),
so ranks take disjoint blocks.  These tests cover the host-side pieces that
run on every rank: the block assignment and the max/sum/min reduction that
turns per-rank timings into the whole-job number.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_streaming_workload_blocks_partition(world):
    seen = []
    for r in range(world):
        seen += [b for _, b in bench.shard(5, r, world)]
    assert sorted(seen) == list(range(32))


@pytest.mark.parametrize("workload", [1, 2, 3, 4])
def test_weak_scaling_gives_each_rank_its_own_block(workload):
    blocks = [bench.shard(workload, r, 8) for r in range(8)]
    assert all(len(b) == 1 for b in blocks)
    assert len({b[0] for b in blocks}) == 8
    assert bench.scaling_kind(workload) == "weak"
    assert bench.scaling_kind(5) == "strong"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.0 + rank           # rank 1 is the slowest
        e2e = 10.0 - rank
        n = 100 * (rank + 1)
        good = rank == 0 or world == 1
        out = bench.reduce_over_ranks(ms, e2e, n, good, "cpu", world)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        ms, e2e, n, good = results[r]
        assert ms == 2.0          # max over ranks
        assert e2e == 10.0        # max over ranks
        assert n == 300.0         # sum over ranks
        assert good is False      # min: one rank was not exact


def test_reduce_single_rank_is_identity():
    assert bench.reduce_over_ranks(1.5, 2.5, 7, True, "cpu", 1) == (1.5, 2.5, 7.0, True)
