"""Host-side plumbing for running the path on several GPUs of one node.

The path splits into independent problems -- (batch, KV head) units with no
exchange between them -- so N GPUs run N replicas, each on its own sequences
(the benchmark's weak scaling); torch.distributed only lines the ranks up and
takes the slowest rank's time.

KVParallelDecode is the other split, by cache rows (the NVIDIA attention
page, "Parameter four: parallelism"): every rank holds a contiguous share of
each sequence's cached rows, computes attention over it (attn_decode_partial),
and the partial results are merged by their log-sum-exps -- after an
all-gather (attn_decode_merge), or in place across GPUs with the exchange
fused into the merge (attn_decode_merge_peers).
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


def _align(x: int, a: int = 256) -> int:
    return (x + a - 1) // a * a


class PartBuffers:
    """One rank's exchange buffer for the fused KV-parallel merge, and every rank's
    buffer as this process reaches it.

    Each rank's buffer holds, in order: its O part [rows, D] fp32, its LSE part
    [rows] fp32, and two flag arrays of `world` uint32 (ready, consumed), each
    section 256-byte aligned.  base_ptrs[r] is rank r's buffer address as seen
    from this process: this GPU's own memory for r == rank, a peer's mapped here
    otherwise (or, when one GPU stands in for every rank, another local buffer).
    The flags must be zero before the first step."""

    @staticmethod
    def nbytes(rows: int, D: int, world: int) -> int:
        return _align(rows * D * 4) + _align(rows * 4) + 2 * _align(world * 4)

    def __init__(self, local: torch.Tensor, base_ptrs: Sequence[int], rank: int, rows: int, D: int):
        world = len(base_ptrs)
        if local.dtype != torch.uint8 or local.numel() < self.nbytes(rows, D, world):
            raise ValueError("local buffer too small")
        self.rank, self.world, self.rows, self.D = rank, world, rows, D
        o_off, lse_off = 0, _align(rows * D * 4)
        ready_off = lse_off + _align(rows * 4)
        cons_off = ready_off + _align(world * 4)
        dev = local.device
        self.local = local
        self.o_part = local[o_off:o_off + rows * D * 4].view(torch.float32)
        self.lse_part = local[lse_off:lse_off + rows * 4].view(torch.float32)
        self.ready = local[ready_off:ready_off + world * 4].view(torch.int32)
        self.consumed = local[cons_off:cons_off + world * 4].view(torch.int32)
        as_dev = lambda xs: torch.tensor(list(xs), dtype=torch.int64, device=dev)
        self.o_ptrs = as_dev(b + o_off for b in base_ptrs)
        self.lse_ptrs = as_dev(b + lse_off for b in base_ptrs)
        # where this rank signals: its slot in every rank's ready / consumed array
        self.ready_slots = as_dev(b + ready_off + 4 * rank for b in base_ptrs)
        self.consumed_slots = as_dev(b + cons_off + 4 * rank for b in base_ptrs)


def symmetric_part_buffers(rows: int, D: int, group=None, device=None) -> PartBuffers:
    """This rank's PartBuffers in symmetric memory shared by the ranks of `group`
    (torch.distributed._symmetric_memory): peers' buffers are mapped into this
    process, so the merge reads them with plain loads over NVLink."""
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    buf = symm_mem.empty(PartBuffers.nbytes(rows, D, world), dtype=torch.uint8, device=device)
    buf.zero_()
    handle = symm_mem.rendezvous(buf, group if group is not None else dist.group.WORLD)
    torch.cuda.synchronize(buf.device)
    dist.barrier(group)
    return PartBuffers(buf, [int(p) for p in handle.buffer_ptrs], rank, rows, D)


def local_part_buffers(rows: int, D: int, world: int, device) -> list:
    """`world` ranks' PartBuffers all in one GPU's memory, for one process that
    runs every rank's share in turn (to check the fused merge on one GPU)."""
    bufs = [torch.zeros(PartBuffers.nbytes(rows, D, world), dtype=torch.uint8, device=device) for _ in range(world)]
    ptrs = [b.data_ptr() for b in bufs]
    return [PartBuffers(bufs[r], ptrs, r, rows, D) for r in range(world)]


class KVParallelDecode:
    """Decode with the cache split by rows over the ranks of `group` (KV parallelism).

    Every rank holds a contiguous share of each sequence's cached rows
    (kv_shard_rows / shard_seqlens) and the same query rows.  One step:
      1. attention over this rank's rows (attn_decode_partial), written straight
         into this rank's part buffers;
      2. the exchange, and 3. the log-sum-exp merge of all ranks' parts:
         - default: an all-gather of the fp32 partials (B * Hq * (D + 1) * 4
           bytes per rank) into preallocated buffers, then attn_decode_merge;
         - fused=True: no copy -- every rank's merge reads all parts where they
           were written (attn_decode_merge_peers, plain loads over NVLink),
           ordered by epoch flags (attn_kvp_signal / attn_kvp_wait); the parts
           live in `parts` (PartBuffers; symmetric memory by default).
    Every rank ends with the full result.  Buffers are allocated once, so a step
    allocates nothing, and every rank makes the same calls in the same order.
    partial_fn(q, k, v, seqlens, o_out, lse_out) and merge_fn(o_all, lse_all, out,
    lse) replace the library's kernels in the all-gather form (the tests use the
    fp64 oracle to check the exchange on CPU ranks).
    """

    def __init__(self, q: torch.Tensor, k_shard: torch.Tensor, v_shard: torch.Tensor, seqlens_shard: torch.Tensor,
                 *, scale=None, group=None, partial_fn=None, merge_fn=None, workspace=None, fused=False,
                 parts: PartBuffers = None, rank=None, world=None):
        import torch.distributed as dist
        B, Hq, D = q.shape
        self.q, self.k, self.v, self.sl = q, k_shard, v_shard, seqlens_shard
        self.scale, self.group = scale, group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.world = world if world is not None else (dist.get_world_size(group) if self.distributed else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if self.distributed else 0)
        self.out = torch.empty((B, Hq, D), dtype=q.dtype, device=q.device)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        self.workspace = workspace
        self.fused = fused
        if fused:
            self.parts = parts if parts is not None else symmetric_part_buffers(B * Hq, D, group, q.device)
            if (self.parts.world, self.parts.rank) != (self.world, self.rank):
                raise ValueError("part buffers laid out for another rank or world size")
            self.epoch = 0
        else:
            self.o_all = torch.empty((self.world, B, Hq, D), dtype=torch.float32, device=q.device)
            self.lse_all = torch.empty((self.world, B, Hq), dtype=torch.float32, device=q.device)
        self._partial = partial_fn or self._library_partial
        self._merge = merge_fn or self._library_merge

    def _library_partial(self, q, k, v, sl, o_out, lse_out):
        from . import decode_partial
        decode_partial(q, k, v, sl, scale=self.scale, o_part=o_out, lse_part=lse_out, workspace=self.workspace)

    def _library_merge(self, o_all, lse_all, out, lse):
        from . import decode_merge
        decode_merge(o_all, lse_all, out=out, lse=lse)

    def produce(self):
        """Fused form, first half of a step: this rank's part, then its ready signal."""
        from . import kvp_signal, kvp_wait
        P = self.parts
        e = self.epoch + 1
        if e > 1:   # every rank has read this rank's previous part
            kvp_wait(P.consumed, e - 1)
        B, Hq, D = self.q.shape
        self._library_partial(self.q, self.k, self.v, self.sl, P.o_part.view(B, Hq, D), P.lse_part.view(B, Hq))
        kvp_signal(P.ready_slots, e)

    def consume(self):
        """Fused form, second half: merge every rank's part in place, then tell every rank it was read."""
        from . import decode_merge_peers, kvp_signal
        P = self.parts
        e = self.epoch + 1
        B, Hq, D = self.q.shape
        decode_merge_peers(P.o_ptrs, P.lse_ptrs, P.ready, e, B * Hq, D, out=self.out, lse=self.lse)
        kvp_signal(P.consumed_slots, e)
        self.epoch = e
        return self.out, self.lse

    def step(self):
        """One decode step; returns (out [B,Hq,D], lse [B,Hq]) -- buffers reused by the next step."""
        if self.fused:
            self.produce()
            return self.consume()
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
