"""One acquisition over several GPUs: contiguous block ranges, one per rank.

Page "Paired-count resident layout", "Operation pipeline" step 4: the 512-scan
blocks are independent work items and ``block_stride=k`` touches blocks 0, k,
2k, ...  So an acquisition splits into contiguous block ranges, one per GPU:
each rank encodes and holds its own range (its own resident, its own delta
baselines) and a query runs on every rank over its range.  The only exchange
is the result: every rank owns a disjoint, ordered run of image rows, and one
all-gather (NCCL over NVLink between GPUs, gloo on CPU) assembles the full
``[ceil(B/k)][512]`` image on every rank.  No kernel reads another GPU's
memory.

A rank's range starts at a multiple of ``granule`` blocks; a query's stride
must divide the granule, so that the blocks a rank touches (global b with
b % k == 0) are its local blocks 0, k, 2k, ...  (the library's strided query
starts at a resident's first block).
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist


def block_ranges(n_blocks: int, world: int, granule: int = 1) -> list[tuple[int, int]]:
    """Contiguous, balanced split of blocks 0..n_blocks-1 over `world` ranks, in units of
    `granule` blocks (the last unit may be short): [(b0, b1), ...] in rank order, every b0
    a multiple of `granule`.  Lower ranks take the extra units; a rank may get none."""
    if world < 1 or granule < 1 or n_blocks < 0:
        raise ValueError("bad block_ranges arguments")
    units = math.ceil(n_blocks / granule)
    base, extra = divmod(units, world)
    out = []
    u0 = 0
    for r in range(world):
        u1 = u0 + base + (1 if r < extra else 0)
        out.append((min(n_blocks, u0 * granule), min(n_blocks, u1 * granule)))
        u0 = u1
    return out


def rows_of(b0: int, b1: int, k: int) -> tuple[int, int]:
    """The global image rows of blocks [b0, b1) at stride k: rows r with r*k in [b0, b1),
    as (first row, row count)."""
    first = -(-b0 // k)
    end = -(-b1 // k)
    return first, max(0, end - first)


def check_stride(granule: int, k: int) -> None:
    if k < 1 or granule % k:
        raise ValueError(f"block_stride {k} must divide the shard granule {granule}")


def gather_rows(local: torch.Tensor, counts: list[int], group=None) -> torch.Tensor:
    """All-gather of each rank's image rows ([counts[rank]][512], any integer dtype)
    into the full image [sum(counts)][512], in rank order, on every rank.  Uneven
    counts are padded to the largest for the collective and trimmed after it."""
    world = len(counts)
    if world == 1:
        return local
    width = local.shape[1]
    most = max(counts)
    pad = torch.zeros((most, width), dtype=local.dtype, device=local.device)
    pad[: local.shape[0]] = local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    return torch.cat([bufs[r][: counts[r]] for r in range(world)], dim=0)


class ShardedQuery:
    """The full image of a strided masked sum over an acquisition split by block_ranges.

    `local_query(mask, k)` runs the query over this rank's resident and returns its
    rows ([rows][512]; [0][512] when the rank holds no blocks); `run` assembles every
    rank's rows.  With the library's resident:
    ``lambda m, k: res.masked_sum(m, block_stride=k)``."""

    def __init__(self, n_blocks: int, world: int, rank: int, granule: int, group=None):
        self.n_blocks, self.world, self.rank, self.granule, self.group = n_blocks, world, rank, granule, group
        self.ranges = block_ranges(n_blocks, world, granule)
        self.b0, self.b1 = self.ranges[rank]

    def counts(self, k: int) -> list[int]:
        check_stride(self.granule, k)
        return [rows_of(b0, b1, k)[1] for b0, b1 in self.ranges]

    def run(self, local_query, mask, k: int) -> torch.Tensor:
        counts = self.counts(k)
        mine = local_query(mask, k)
        if mine.shape != (counts[self.rank], 512):
            raise ValueError(f"rank {self.rank}: local image {tuple(mine.shape)}, expected "
                             f"({counts[self.rank]}, 512)")
        return gather_rows(mine, counts, self.group)
