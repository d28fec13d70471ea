"""Replica bookkeeping for one process per GPU.

The hot path shards without any exchange: sequences, query blocks and receiver layers are
independent units, so each rank owns whole requests (its own maps, BSR, V and O) and runs
compression and retrieval on them alone.  The only collectives are the ones of the
measurement: a barrier before timing and the maximum of the ranks' times (a job takes as long
as its slowest rank).
"""
from typing import List

import torch
import torch.distributed as dist


def owned(n_units: int, world: int, rank: int) -> range:
    """The contiguous share of `n_units` independent units (requests, layers) owned by `rank`:
    sizes differ by at most one, earlier ranks take the extra ones."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(seconds: float, device=None) -> float:
    """The largest of the ranks' values (every rank gets it); the value itself without a
    process group."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(seconds)
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(count: int, device=None) -> int:
    """Total of an integer over the ranks (units processed by the whole job)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return int(count)
    t = torch.tensor([count], dtype=torch.int64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return int(t.item())


def job_throughput(units_all_ranks: int, slowest_seconds: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    if slowest_seconds <= 0:
        raise ValueError("non-positive time")
    return units_all_ranks / slowest_seconds


def shares(n_units: int, world: int) -> List[range]:
    return [owned(n_units, world, r) for r in range(world)]
