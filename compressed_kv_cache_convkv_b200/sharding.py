"""Work split across GPUs for the ConvKV step.

The step shards with no exchange: independent layer / denoising-step states,
and the heads inside one state, never read each other's K/V (per-head conv
weights, per-head attention).  A rank therefore owns a contiguous range of
units (states or heads) and runs its own handle on its own GPU; the only
cross-rank operation is the reduction of the device timing (the maximum over
ranks), done with torch.distributed.
"""
from __future__ import annotations


def shard(units: int, world: int, rank: int) -> range:
    """Contiguous range of `units` owned by `rank` of `world` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world or units < 0:
        raise ValueError(f"bad shard request: units={units} world={world} rank={rank}")
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist=None, device=None) -> float:
    """Sum of a per-rank float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
