"""One acquisition split into contiguous block ranges over ranks (two gloo ranks on
CPU): each rank queries only its blocks and the gathered image equals the image of
the whole acquisition.  The per-rank query is the oracle's decode-based masked sum
over the rank's own oracle-encoded blocks, standing in for the rank's GPU resident;
the partition, the row counts and the all-gather are the library's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from virtual_imaging_b200.shard import ShardedQuery, block_ranges, check_stride, rows_of


def test_block_ranges_cover_align_balance():
    for n in range(0, 70):
        for world in range(1, 9):
            for g in (1, 2, 4, 16):
                rs = block_ranges(n, world, g)
                assert len(rs) == world and rs[0][0] == 0 and rs[-1][1] == n
                assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
                assert all(b0 % g == 0 or b0 == n for b0, _ in rs)
                units = [-(-(b1 - b0) // g) for b0, b1 in rs]
                assert max(units) - min(units) <= 1
                for k in (d for d in (1, 2, 4, 8, 16) if g % d == 0):
                    rows = sum(rows_of(b0, b1, k)[1] for b0, b1 in rs)
                    assert rows == -(-n // k)              # ceil(B/k) rows, each once
    assert block_ranges(512, 8, 16)[3] == (192, 256)
    with pytest.raises(ValueError):
        check_stride(16, 3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _acquisition():
    rng = np.random.default_rng(41)
    P, B = 10 * 13, 10
    lam = rng.uniform(0.0, 6.0, size=P)
    x = np.minimum(rng.poisson(np.broadcast_to(lam, (B * 512, P))), 255).astype(np.uint8)
    masks = [(rng.random(P) < f).astype(np.uint8) for f in (0.1, 0.5, 1.0)]
    return x, masks


def _worker(rank, world, port, q):
    import oracle as O

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, masks = _acquisition()
        B = x.shape[0] // 512
        sq = ShardedQuery(B, world, rank, granule=2)
        b0, b1 = sq.b0, sq.b1
        enc = O.encode(x[b0 * 512:b1 * 512], 8, threads=1)      # this rank's blocks only

        def local(mask, k):
            if b1 == b0:
                return torch.zeros((0, 512), dtype=torch.int64)
            return torch.from_numpy(O.resident_masked_sum(enc, mask, None, k, threads=1).astype(np.int64))

        out = []
        for m in masks:
            for k in (1, 2):
                out.append(sq.run(local, m, k).numpy())
        dist.barrier()
        q.put((rank, (b0, b1), out))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_full_image():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle as O

    x, masks = _acquisition()
    (r0, rng0, out0), (r1, rng1, out1) = got
    assert rng0 == (0, 6) and rng1 == (6, 10)                  # 5 units of 2 blocks: 3 + 2
    i = 0
    for m in masks:
        for k in (1, 2):
            want = O.dense_masked_sum(x, m, None, k).astype(np.int64)
            assert out0[i].shape == want.shape and (out0[i] == want).all(), (i, k)
            assert (out1[i] == want).all(), (i, k)
            i += 1
