"""Multi-rank host logic on CPU (gloo, world size 2): the data-parallel
sharding of tokens, per-rank seeds, the max-over-ranks timing reduction and
the weak-scaling throughput formula that bench.py uses at N > 1."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_mixture_experts_histogram_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # max over ranks: each rank reports a different "time"
        m = bench.dist_max(10.0 + rank, world)
        # every rank draws its own seeded batch; gather a checksum of x
        wl = synth.Workload("dp", 64, 128, 4, 128, 2)
        inp = synth.make_inputs(wl, seed=synth.rank_seed(42, rank))
        chk = torch.tensor([float(inp["x"].float().sum())])
        out = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(out, chk)
        bench.barrier(world)
        q.put((rank, m, [float(o) for o in out]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_draw_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, sums in res:
        assert m == 11.0                      # slowest rank's time
        assert sums[0] != sums[1]             # independent replicas' batches


@pytest.mark.parametrize("T,world", [(8192, 8), (512, 3), (7, 4), (1, 2)])
def test_shard_tokens_partitions_the_batch(T, world):
    spans = [synth.shard_tokens(T, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == T
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0 and a0 <= a1
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_rank_seeds_are_distinct_and_weak_scaling_formula():
    import bench
    assert len({synth.rank_seed(42, r) for r in range(64)}) == 64
    # 8 ranks x 3072 tokens x 20 steps in 100 ms -> 4.9152e6 tokens/s
    assert bench.weak_scaling_value(8, 3072, 20, 100.0) == pytest.approx(8 * 3072 * 20 / 0.1)
