"""Host-side plumbing for running the path on several GPUs of one node.

The path splits into independent problems -- (batch, KV head) units with no
exchange between them -- so N GPUs run N replicas, each on its own sequences.
There is no collective on the data path; torch.distributed is only used to
line the ranks up and to take the slowest rank's time.
"""
from __future__ import annotations

from typing import Sequence

import torch


def rank_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own sequences."""
    return int(base_seed) + 1000 * int(rank)


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous share of n_units for `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(int(n_units), world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job finishes with its slowest rank)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank: Sequence[float], slowest_seconds: float) -> float:
    """Whole-job throughput: all ranks' work over the slowest rank's time."""
    if slowest_seconds <= 0:
        raise ValueError("time must be positive")
    return float(sum(work_per_rank)) / slowest_seconds
