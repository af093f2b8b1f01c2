"""KV-parallel decode with the exchange fused into the merge, on one GPU.

Each rank leaves its attn_decode_partial results in its own buffer and every
rank's merge (attn_decode_merge_peers) reads all parts where they lie, ordered
by epoch flags (attn_kvp_signal / attn_kvp_wait).  Across GPUs the buffers are
peers' memory reached over NVLink; here one GPU stands in for N ranks: each
rank's buffer is a separate allocation, and one process runs every rank's first
half (wait for the previous epoch's readers, partial, ready signal) and then
every rank's second half (merge, consumed signal) in stream order, so each wait
is met by work enqueued before it.  Three epochs in a row must each equal the
whole-cache decode (and the oracle), with the device error word clear.
"""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_gqa_b200 as attn
from exact_tiled_attention_gqa_b200 import _native
from exact_tiled_attention_gqa_b200.multigpu import KVParallelDecode, kv_shard_rows, local_part_buffers, shard_seqlens
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    attn.device_error(reset=True)
    yield
    attn.device_error(reset=True)


@pytest.mark.parametrize("N,D", [(2, 128), (3, 64), (4, 256), (1, 128)])
def test_fused_merge_equals_whole_cache_decode(oracle_mod, N, D):
    B, Hq, Hkv, Lmax = 6, 16, 2, 5000
    seqlens = [5000, 4097, 1, 0, 2500, 700]
    g = torch.Generator().manual_seed(N * 100 + D)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16).cuda()
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    q = torch.empty(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    bufs = local_part_buffers(B * Hq, D, N, q.device)
    ranks = []
    for r in range(N):
        rows = kv_shard_rows(Lmax, r, N)
        ranks.append(KVParallelDecode(q, k[:, :, rows.start:rows.stop].contiguous(),
                                      v[:, :, rows.start:rows.stop].contiguous(), shard_seqlens(sl, rows),
                                      scale=1 / math.sqrt(D), fused=True, parts=bufs[r], rank=r, world=N))
    for epoch in range(3):
        q.copy_(torch.randn(B, Hq, D, generator=g).to(torch.bfloat16))
        for r in ranks:
            r.produce()
        outs = [tuple(t.clone() for t in r.consume()) for r in ranks]
        want_o, want_l = attn.decode(q, k, v, sl, scale=1 / math.sqrt(D))
        torch.cuda.synchronize()
        assert attn.device_error(reset=True) == 0
        for o, l in outs:
            assert (o.float() - want_o.float()).abs().max().item() <= 2e-2
            fin = torch.isfinite(want_l)
            assert torch.equal(torch.isneginf(l), torch.isneginf(want_l))
            assert (l[fin] - want_l[fin]).abs().max().item() <= 1e-3
        if epoch == 0:
            ref_o, ref_l = oracle_mod.attention_decode(q.cpu(), k.cpu(), v.cpu(), np.array(seqlens, np.int32),
                                                       1 / math.sqrt(D))
            assert_close(outs[0][0], outs[0][1], ref_o, ref_l, f"fused kv-parallel x{N} D{D}")


def test_waits_on_a_flag_nothing_sets_give_up():
    """A flag that never reaches its epoch: the wait and the merge each give up
    after their time limit with ATTN_DEVERR_TIMEOUT, and the context stays usable."""
    attn.device_error(reset=True)
    flags = torch.zeros(2, dtype=torch.int32, device="cuda")
    attn.kvp_wait(flags, 5)
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == _native.ATTN_DEVERR_TIMEOUT
    rows, D = 8, 64
    part = torch.zeros(rows * D + rows, dtype=torch.float32, device="cuda")
    o_ptrs = torch.tensor([part.data_ptr()], dtype=torch.int64, device="cuda")
    l_ptrs = torch.tensor([part.data_ptr() + rows * D * 4], dtype=torch.int64, device="cuda")
    out = torch.full((rows, D), 7.0, dtype=torch.bfloat16, device="cuda")
    attn.decode_merge_peers(o_ptrs, l_ptrs, flags[:1], 1, rows, D, out=out)
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == _native.ATTN_DEVERR_TIMEOUT
    assert torch.all(out == 7.0)   # left unwritten
    # signalled, the same merge runs
    attn.kvp_signal(torch.tensor([flags.data_ptr()], dtype=torch.int64, device="cuda"), 1)
    attn.decode_merge_peers(o_ptrs, l_ptrs, flags[:1], 1, rows, D, out=out)
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == 0
    assert torch.all(out == 0.0)
