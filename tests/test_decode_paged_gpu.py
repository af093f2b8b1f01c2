"""GPU parity for attn_decode_paged (through the C ABI): the paged cache is
gathered back to contiguous rows on the host and the fp64 oracle runs on that.
Pages are handed out in a shuffled order, and pages no sequence uses (and rows
past each sequence's length) hold NaN, so a wrong page or row shows up."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode_mq, decode_paged, device_error
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    device_error(reset=True)
    yield
    assert device_error(reset=True) == 0


def _paged_inputs(seqlens, Hq, Hkv, Lq, D, page_size, seed, spare_pages=3):
    g = torch.Generator().manual_seed(seed)
    B = len(seqlens)
    pages_per = [max(1, -(-n // page_size)) for n in seqlens]
    max_pages = max(pages_per) + 1
    n_pages = sum(pages_per) + spare_pages
    order = torch.randperm(n_pages, generator=g)
    k_pages = torch.full((n_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16)
    v_pages = torch.full((n_pages, Hkv, page_size, D), float("nan"), dtype=torch.bfloat16)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)   # unused entries: never read
    k_cont = torch.full((B, Hkv, max_pages * page_size, D), float("nan"), dtype=torch.bfloat16)
    v_cont = torch.full_like(k_cont, float("nan"))
    nxt = 0
    for b, n in enumerate(seqlens):
        for i in range(pages_per[b]):
            pg = int(order[nxt]); nxt += 1
            table[b, i] = pg
            rows = min(page_size, n - i * page_size)
            if rows <= 0:
                continue
            kk = torch.randn(Hkv, rows, D, generator=g).to(torch.bfloat16)
            vv = torch.randn(Hkv, rows, D, generator=g).to(torch.bfloat16)
            k_pages[pg, :, :rows] = kk
            v_pages[pg, :, :rows] = vv
            k_cont[b, :, i * page_size:i * page_size + rows] = kk
            v_cont[b, :, i * page_size:i * page_size + rows] = vv
    q = torch.randn(B, Hq, Lq, D, generator=g).to(torch.bfloat16)
    return q, k_pages, v_pages, table, torch.tensor(seqlens, dtype=torch.int32), k_cont, v_cont


@pytest.mark.parametrize("page_size", [64, 128, 256])
@pytest.mark.parametrize("G,Lq,D", [(4, 1, 128), (4, 4, 128), (8, 2, 64), (1, 1, 128), (16, 4, 128), (4, 2, 256),
                                    (32, 1, 256)])
def test_paged_against_oracle(oracle_mod, page_size, G, Lq, D):
    Hkv = 2
    seqlens = [1000, 1, 0, 257, 64, 3000]
    q, kp, vp, table, sl, kc, vc = _paged_inputs(seqlens, G * Hkv, Hkv, Lq, D, page_size, seed=page_size + G + Lq)
    scale = 1 / math.sqrt(D)
    out, lse = decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    outs, lses = [], []
    for b, n in enumerate(seqlens):
        o, l = oracle_mod.attention_prefill(q[b:b + 1], kc[b:b + 1, :, :n], vc[b:b + 1, :, :n], scale, True)
        outs.append(o[0]); lses.append(l[0])
    assert_close(out, lse, np.stack(outs), np.stack(lses), f"paged ps{page_size} G{G} Lq{Lq} D{D}")
    # the same rows read contiguously give the same answer
    mo, ml = decode_mq(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert (mo.float() - out.float()).abs().max().item() <= 2e-2


def test_bad_page_is_flagged_not_read_out_of_bounds():
    """A block-table entry outside the pool is replaced by page 0 and flagged, never dereferenced."""
    q, kp, vp, table, sl, kc, vc = _paged_inputs([300], 4, 1, 1, 128, 128, seed=1)
    table[0, 1] = 10_000
    out, _ = decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), sl.cuda())
    torch.cuda.synchronize()
    assert device_error(reset=True) & 0x4
