"""Host-side plumbing for running the path on several GPUs of one node.

The path splits into independent problems -- (batch, KV head) units with no
exchange between them -- so N GPUs run N replicas, each on its own sequences
(the benchmark's weak scaling); torch.distributed only lines the ranks up and
takes the slowest rank's time.

decode_kv_parallel is the other split, by cache rows (the NVIDIA attention
page, "Parameter four: parallelism"): every rank holds a contiguous share of
each sequence's cached rows, computes attention over it (attn_decode_partial),
the partial results are all-gathered, and attn_decode_merge combines them.
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


def kv_shard_rows(Lmax: int, rank: int, world: int) -> range:
    """The cache rows rank `rank` holds when Lmax rows are split over `world` ranks."""
    return shard(Lmax, rank, world)


def shard_seqlens(seqlens: torch.Tensor, rows: range) -> torch.Tensor:
    """Per-sequence valid rows inside the shard `rows` (a sequence of length n holds rows 0..n-1)."""
    return (seqlens.to(torch.int64) - rows.start).clamp(0, len(rows)).to(torch.int32)


def decode_kv_parallel(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, seqlens_shard: torch.Tensor,
                       group=None, partial_fn=None, merge_fn=None):
    """One new token per sequence against a cache split by rows over the ranks of `group`.

    q [B,Hq,D] (the same on every rank); k_shard / v_shard [B,Hkv,rows,D] this rank's rows;
    seqlens_shard int32 [B] the valid rows of each sequence in this shard (shard_seqlens).
    Every rank returns the full result (out [B,Hq,D] bf16, lse [B,Hq]).  partial_fn / merge_fn
    default to the library's attn_decode_partial / attn_decode_merge.
    """
    import torch.distributed as dist
    from . import decode_merge, decode_partial
    o, lse = (partial_fn or decode_partial)(q, k_shard, v_shard, seqlens_shard)
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o) for _ in range(world)]
    l_all = [torch.empty_like(lse) for _ in range(world)]
    dist.all_gather(o_all, o.contiguous(), group=group)
    dist.all_gather(l_all, lse.contiguous(), group=group)
    return (merge_fn or decode_merge)(torch.stack(o_all), torch.stack(l_all))
