"""Multi-rank host logic on CPU (gloo, world size 2): the KV-group partition
covers every head exactly once, and timings aggregate as the max over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_prefill_last_b200 import shard


def test_partition_covers_every_group_once():
    for h_kv in (1, 4, 8, 7):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for r in range(world):
                lo, hi = shard.kv_group_range(h_kv, world, r)
                seen += list(range(lo, hi))
            assert seen == list(range(h_kv))
    assert shard.query_head_range(28, 4, 2, 1) == (14, 28)
    with pytest.raises(ValueError):
        shard.kv_group_range(8, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = shard.query_head_range(32, 8, world, rank)
        t = shard.max_over_ranks(10.0 + rank)
        obj = [None] * world
        dist.all_gather_object(obj, (lo, hi))
        q.put((rank, t, obj))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_partition():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, obj in res:
        assert t == 11.0
        assert obj == [(0, 16), (16, 32)]


def _slice_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist
    import crisp_synth as S
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank draws only its KV groups of one layer (the --shard heads
        # path of bench.py); gathered, the shards are the whole layer
        cfg = S.scaled("C_cliff", n=1024, h_q=8, h_kv=4)
        lo, hi = shard.kv_group_range(cfg.h_kv, world, rank)
        qs, ks, _ = S.generate_slice(cfg, lo, hi, threads=2, with_v=False)
        gq = [None] * world
        gk = [None] * world
        dist.all_gather_object(gq, qs)
        dist.all_gather_object(gk, ks)
        # timings aggregate as the slowest rank, counts add up
        t = torch.tensor([5.0 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        cnt = torch.tensor([float(hi - lo)], dtype=torch.float64)
        dist.all_reduce(cnt, op=dist.ReduceOp.SUM)
        if rank == 0:
            full = S.generate(cfg, with_v=False)
            ok = bool((np.concatenate(gq) == full.q).all() and (np.concatenate(gk) == full.k).all())
            q.put((ok, float(t.item()), float(cnt.item())))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_head_shards_rebuild_the_layer():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_slice_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok, t, cnt = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok and t == 6.0 and cnt == 4.0
