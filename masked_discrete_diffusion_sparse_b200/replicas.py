"""Replica sharding for N > 1 processes, one per GPU.

The sampling path has no exchange step: a run of one sequence never needs data from another, so
N GPUs run N independent replicas of the same model, each on its own sequences.  Nothing crosses
ranks on the data path; only the timing is combined (the job ends with its slowest replica).
"""
from __future__ import annotations


def replica_sequence_ids(rank: int, batch: int) -> list[int]:
    """Global indices of this rank's sequences (they seed its prompts and decoding orders):
    rank * batch .. rank * batch + batch - 1, so the ranks' sequence sets are disjoint."""
    if rank < 0 or batch < 1:
        raise ValueError("rank must be >= 0 and batch >= 1")
    return [rank * batch + s for s in range(batch)]


def slowest_time_ms(ms: float, world: int, dist=None, device=None) -> float:
    """Maximum over ranks of a per-rank time in milliseconds (all_reduce MAX when world > 1)."""
    if world <= 1:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed divided by the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / (ms_max / 1e3)
