"""The multi-GPU path of bench.py on CPU ranks (gloo, world size 2): every rank
shards its own work (distinct seeds), the timing collective returns the slowest
rank's time on every rank, and the whole-job value counts all ranks' work."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        seed = bench.shard_seed(rank)
        # each rank draws its own shard
        x = synth.normal((4, 8), seed)
        elapsed = 10.0 + 5.0 * rank          # rank 1 is the slow one
        dist.barrier()
        t = bench.max_over_ranks(elapsed, world, "cpu")
        dist.barrier()
        v = bench.weak_scaling_value(world, 2e12, 10, t)
        q.put((rank, seed, float(x.sum()), t, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    (r0, s0, x0, t0, v0), (r1, s1, x1, t1, v1) = res
    assert s0 != s1 and x0 != x1                 # disjoint shards
    assert t0 == t1 == 15.0                      # both ranks see the slowest time
    assert v0 == v1 == pytest.approx(2 * 2e12 * 10 / 15e-3 / 1e12)
