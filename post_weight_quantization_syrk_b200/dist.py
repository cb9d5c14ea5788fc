"""Rank plumbing for running the path on several GPUs, one process per GPU.

The path shards without a data-path collective: layers (or whole decoder
blocks) are independent problems, so each rank takes its own.  The one real
exchange is the bit allocation of a whole model, which needs every linear's
trace sensitivity (KronQ paper page, Abstract: sensitivity-guided mixed
precision): the per-rank tables of scores are summed across ranks (each entry
comes from exactly one rank, the others contribute zero, so the sum is exact)
and every rank then runs the same deterministic allocation.
"""
from __future__ import annotations

import os

import torch


def rank_env():
    """(rank, world, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def shard(n: int, rank: int, world: int):
    """Indices 0..n-1 owned by `rank`: strided, so that consecutive blocks
    (similar cost) spread over the ranks."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside world {world}")
    return list(range(rank, n, world))


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def all_max(value: float, device) -> float:
    """Maximum of a per-rank scalar over all ranks (the job's time is the
    slowest rank's)."""
    dist = _dist()
    if dist is None or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def merge_table(table: torch.Tensor) -> torch.Tensor:
    """In place: every rank ends with the full table, given that each entry
    was filled by exactly one rank and is zero elsewhere."""
    dist = _dist()
    if dist is not None and dist.get_world_size() > 1:
        dist.all_reduce(table, op=dist.ReduceOp.SUM)
    return table
