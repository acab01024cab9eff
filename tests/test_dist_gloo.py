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


def _head_shard_worker(rank, world, port, q):
    """Each rank attends its share of the heads with the oracle (prefill and a
    short stream), then an all-gather over the head axis rebuilds the outputs."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import synth
        from oracle import attention as orc
        from streaming_frame_causal_b200 import head_shard
        F, P, H, D = 5, 40, 4, 32
        h0, hr = head_shard(rank, world, H)
        qq, kk, vv = synth.tiny_qkv(seed=31, F=F, P=P, H=H, D=D)
        part = orc.prefill(qq.numpy(), kk.numpy(), vv.numpy(), P=P, scale_frames=1, sliding_window_size=2,
                           heads=range(h0, h0 + hr))
        t = torch.from_numpy(np.ascontiguousarray(part))
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t)
        pre = torch.cat(parts, dim=2).numpy()
        # streaming: the rank's cache holds only its heads
        cache = orc.StreamCache(heads=hr, head_dim=D, P=P, scale_frames=1, window_frames=2, page_tokens=16)
        outs = []
        for i in range(F):
            fq, fk, fv = (x[0, i * P:(i + 1) * P] for x in (qq.numpy(), kk.numpy(), vv.numpy()))
            cache.append_evict(0, i, fk[:, h0:h0 + hr], fv[:, h0:h0 + hr])
            o = torch.from_numpy(np.ascontiguousarray(cache.attend(0, fq[:, h0:h0 + hr])))
            got = [torch.empty_like(o) for _ in range(world)]
            dist.all_gather(got, o)
            outs.append(torch.cat(got, dim=1).numpy())
        q.put((rank, (h0, hr), pre, np.stack(outs)))
    finally:
        dist.destroy_process_group()


def test_head_sharded_attention_gathers_to_the_single_rank_result():
    import numpy as np
    import synth
    from oracle import attention as orc
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(0, 2), (2, 2)]
    F, P, H, D = 5, 40, 4, 32
    qq, kk, vv = synth.tiny_qkv(seed=31, F=F, P=P, H=H, D=D)
    want = orc.prefill(qq.numpy(), kk.numpy(), vv.numpy(), P=P, scale_frames=1, sliding_window_size=2)
    cache = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=1, window_frames=2, page_tokens=16)
    want_s = []
    for i in range(F):
        fq, fk, fv = (x[0, i * P:(i + 1) * P] for x in (qq.numpy(), kk.numpy(), vv.numpy()))
        cache.append_evict(0, i, fk, fv)
        want_s.append(cache.attend(0, fq))
    for rank, _, pre, stream in res:
        np.testing.assert_array_equal(pre, want)          # every rank holds the whole gathered output
        np.testing.assert_array_equal(stream, np.stack(want_s))


def test_head_shard_plan():
    from streaming_frame_causal_b200 import head_shard
    for H, world in ((16, 2), (16, 3), (32, 8), (5, 5)):
        shards = [head_shard(r, world, H) for r in range(world)]
        assert shards[0][0] == 0 and sum(n for _, n in shards) == H
        assert all(a + n == b for (a, n), (b, _) in zip(shards, shards[1:]))
        assert max(n for _, n in shards) - min(n for _, n in shards) <= 1
    with pytest.raises(ValueError):
        head_shard(2, 2, 16)
