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
