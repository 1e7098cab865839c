"""Multi-rank host logic on CPU: two gloo ranks, no GPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from virtual_imaging_b200.series import max_over_ranks, shard, sum_over_ranks


def test_shard_covers_and_balances():
    for n in range(0, 40):
        for world in range(1, 9):
            parts = [shard(n, world, r) for r in range(world)]
            flat = [i for p in parts for i in p]
            assert flat == list(range(n))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard(69, world, rank)                   # the pages' 69-acquisition series
        t = max_over_ranks(1.0 + rank)                  # per-rank timed region
        n = sum_over_ranks(len(mine))
        dist.barrier()
        q.put((rank, mine, t, n))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, t0, n0), (r1, m1, t1, n1) = out
    assert m0 + m1 == list(range(69)) and len(m0) == 35 and len(m1) == 34
    assert t0 == t1 == 2.0
    assert n0 == n1 == 69
