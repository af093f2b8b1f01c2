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


class KVParallelDecode:
    """Decode with the cache split by rows over the ranks of `group` (KV parallelism).

    Every rank holds a contiguous share of each sequence's cached rows
    (kv_shard_rows / shard_seqlens) and the same query rows.  One step:
      1. attention over this rank's rows (attn_decode_partial), written straight
         into this rank's slice of the exchange buffers;
      2. an all-gather of the fp32 partials (B * Hq * (D + 1) * 4 bytes per rank);
      3. the log-sum-exp merge of all ranks' partials (attn_decode_merge).
    Every rank ends with the full result.  The buffers are allocated once, so a
    step allocates nothing and every rank makes the same collective calls in the
    same order.  partial_fn(q, k, v, seqlens, o_out, lse_out) and
    merge_fn(o_all, lse_all, out, lse) default to the library's kernels; the
    tests substitute the fp64 oracle to check the exchange on CPU ranks.
    """

    def __init__(self, q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, seqlens_shard: torch.Tensor,
                 *, scale=None, group=None, partial_fn=None, merge_fn=None, workspace=None):
        import torch.distributed as dist
        B, Hq, D = q.shape
        self.q, self.k, self.v, self.sl = q, k_shard, v_shard, seqlens_shard
        self.scale, self.group = scale, group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if self.distributed else 1
        self.rank = dist.get_rank(group) if self.distributed else 0
        self.o_all = torch.empty((self.world, B, Hq, D), dtype=torch.float32, device=q.device)
        self.lse_all = torch.empty((self.world, B, Hq), dtype=torch.float32, device=q.device)
        self.out = torch.empty((B, Hq, D), dtype=q.dtype, device=q.device)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        self.workspace = workspace
        self._partial = partial_fn or self._library_partial
        self._merge = merge_fn or self._library_merge

    def _library_partial(self, q, k, v, sl, o_out, lse_out):
        from . import decode_partial
        decode_partial(q, k, v, sl, scale=self.scale, o_part=o_out, lse_part=lse_out, workspace=self.workspace)

    def _library_merge(self, o_all, lse_all, out, lse):
        from . import decode_merge
        decode_merge(o_all, lse_all, out=out, lse=lse)

    def step(self):
        """One decode step; returns (out [B,Hq,D], lse [B,Hq]) -- buffers reused by the next step."""
        import torch.distributed as dist
        self._partial(self.q, self.k, self.v, self.sl, self.o_all[self.rank], self.lse_all[self.rank])
        if self.world > 1:
            dist.all_gather(list(self.o_all.unbind(0)), self.o_all[self.rank], group=self.group)
            dist.all_gather(list(self.lse_all.unbind(0)), self.lse_all[self.rank], group=self.group)
        self._merge(self.o_all, self.lse_all, self.out, self.lse)
        return self.out, self.lse


def decode_kv_parallel(q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, seqlens_shard: torch.Tensor,
                       group=None, partial_fn=None, merge_fn=None, scale=None):
    """One new token per sequence against a cache split by rows over the ranks of `group`:
    one KVParallelDecode step.  q [B,Hq,D] (the same on every rank); k_shard / v_shard
    [B,Hkv,rows,D] this rank's rows; seqlens_shard int32 [B] the valid rows of each sequence
    in this shard (shard_seqlens).  Every rank returns the full result (out, lse)."""
    return KVParallelDecode(q, k_shard, v_shard, seqlens_shard, scale=scale, group=group, partial_fn=partial_fn,
                            merge_fn=merge_fn).step()
