"""Several acquisitions over several GPUs: one process per GPU, each holding its
own residents; no data crosses between ranks (page "Paired-count resident
layout": a series is a list of independent acquisitions, each its own
source).  Only timing and counts are reduced across ranks, on the host side
of torch.distributed (NCCL between GPUs, gloo on CPU)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard(n_sources: int, world: int, rank: int) -> list[int]:
    """Contiguous, balanced split of source indices 0..n_sources-1: rank r gets
    floor or ceil of n_sources/world sources, lower ranks take the extra ones."""
    if world < 1 or not 0 <= rank < world or n_sources < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n_sources, world)
    start = rank * base + min(rank, extra)
    return list(range(start, start + base + (1 if rank < extra else 0)))


def _reduce(value: float, op, device=None) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (a timed region's duration)."""
    return _reduce(value, dist.ReduceOp.MAX, device)


def sum_over_ranks(value: float, device=None) -> float:
    """The total over all ranks (units of work processed)."""
    return _reduce(value, dist.ReduceOp.SUM, device)
