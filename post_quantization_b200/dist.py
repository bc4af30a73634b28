"""Multi-GPU plumbing of the KronQ path (torch.distributed; one process per GPU).

The path shards without a data-path exchange: each rank quantizes its own blocks, and a
layer's statistics, factor and solve never leave the GPU that computes them. What crosses
ranks is host-sized: the step time (max over ranks) and, for a mixed-precision stack, the two
traces per sublayer that the bit allocation needs on every rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    """(rank, world size); (0, 1) when torch.distributed is not initialised."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def shard(n_items: int, rank: int, world_size: int) -> list[int]:
    """Contiguous, balanced split of item indices 0..n_items-1 (sizes differ by at most one)."""
    base, extra = divmod(n_items, world_size)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return list(range(start, stop))


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the step time every rank reports)."""
    rank, ws = world()
    if ws == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_traces(local: dict[int, tuple[float, float]], n_items: int,
                  device=None) -> list[tuple[float, float]]:
    """Every rank's (tr H_X, tr H_G) per sublayer, assembled in sublayer order on all ranks.

    local maps global sublayer index -> traces for the sublayers this rank processed; each
    sublayer must be owned by exactly one rank.
    """
    rank, ws = world()
    buf = torch.zeros(n_items, 3, dtype=torch.float64, device=device)
    for i, (a, b) in local.items():
        buf[i, 0] = a
        buf[i, 1] = b
        buf[i, 2] = 1.0
    if ws > 1:
        dist.all_reduce(buf, op=dist.ReduceOp.SUM)
    if not torch.all(buf[:, 2] == 1.0):
        raise RuntimeError("every sublayer must be owned by exactly one rank")
    return [(float(buf[i, 0]), float(buf[i, 1])) for i in range(n_items)]
