"""Multi-rank host logic on CPU with gloo (world size 2): sharding covers every
unit once, the slowest rank's time is what every rank reports, and the whole-job
rate sums all ranks' work.  No GPU involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from exact_tiled_attention_gqa_b200.multigpu import job_rate, rank_seed, shard


def test_shard_covers_units_once():
    for n in (0, 1, 7, 64, 513):
        for world in (1, 2, 3, 8):
            seen = [u for r in range(world) for u in shard(n, r, world)]
            assert seen == list(range(n))
            sizes = [len(shard(n, r, world)) for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def test_rank_seeds_differ():
    assert len({rank_seed(0, r) for r in range(8)}) == 8


def test_job_rate():
    assert job_rate([2.0, 2.0], 0.5) == 8.0
    with pytest.raises(ValueError):
        job_rate([1.0], 0.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    from exact_tiled_attention_gqa_b200.multigpu import max_over_ranks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_time = [3.0, 5.0][rank]
        out[rank] = max_over_ranks(local_time)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 5.0, 1: 5.0}


def _kv_parallel_worker(rank, world, port, out):
    """Each rank holds a contiguous share of every sequence's cache rows, computes
    its partial with the fp64 oracle, the partials are all-gathered over gloo, and
    a plain log-sum-exp merge must give the oracle's decode over all rows."""
    import datetime
    import math

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from exact_tiled_attention_gqa_b200.multigpu import decode_kv_parallel, kv_shard_rows, shard_seqlens
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        g = torch.Generator().manual_seed(7)
        B, Hq, Hkv, L, D = 3, 4, 2, 50, 16
        q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
        k = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)
        v = torch.randn(B, Hkv, L, D, generator=g).to(torch.bfloat16)
        sl = torch.tensor([50, 7, 0], dtype=torch.int32)
        rows = kv_shard_rows(L, rank, world)
        ks = k[:, :, rows.start:rows.stop].contiguous()
        vs = v[:, :, rows.start:rows.stop].contiguous()
        sls = shard_seqlens(sl, rows)

        def partial(q_, k_, v_, s_, o_out, l_out):
            o, l = oracle.attention_decode(q_, k_, v_, s_.numpy(), 1 / math.sqrt(D))
            o_out.copy_(torch.from_numpy(o))
            l_out.copy_(torch.from_numpy(l))

        def merge(o_all, l_all, out, lse):
            o_all, l_all = o_all.double(), l_all.double()
            m = l_all.max(0).values
            w = torch.where(torch.isinf(l_all), torch.zeros_like(l_all), torch.exp(l_all - m))
            tot = w.sum(0)
            o = (w[..., None] * o_all).sum(0) / torch.where(tot > 0, tot, torch.ones_like(tot))[..., None]
            out.copy_(o)
            lse.copy_(torch.where(tot > 0, m + torch.log(tot), torch.full_like(m, -math.inf)))

        o, l = decode_kv_parallel(q, ks, vs, sls, partial_fn=partial, merge_fn=merge)
        o, l = o.double(), l.double()
        ref_o, ref_l = oracle.attention_decode(q, k, v, sl.numpy(), 1 / math.sqrt(D))
        ok_rows = np.isfinite(ref_l)
        out[rank] = (float(np.abs(o.numpy() - ref_o).max()),
                     float(np.abs(l.numpy()[ok_rows] - ref_l[ok_rows]).max()),
                     bool(np.all(np.isneginf(l.numpy()[~ok_rows]))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_kv_parallel_decode_gloo(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_kv_parallel_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(world):
        err_o, err_l, empty_ok = out[r]
        # the exchange carries fp32 partials and the result is bf16-shaped: fp32-level agreement
        assert err_o < 2e-2 and err_l < 1e-5 and empty_ok


def test_shard_seqlens():
    import torch
    from exact_tiled_attention_gqa_b200.multigpu import kv_shard_rows, shard_seqlens
    sl = torch.tensor([0, 5, 10, 17], dtype=torch.int32)
    parts = [shard_seqlens(sl, kv_shard_rows(17, r, 3)) for r in range(3)]
    assert torch.equal(sum(p.to(torch.int64) for p in parts), sl.to(torch.int64))
    assert [len(kv_shard_rows(17, r, 3)) for r in range(3)] == [6, 6, 5]
