"""GPU parity for attn_decode_mq (Lq new tokens per sequence, bottom-right
causal against the cache) through the C ABI, against the fp64 oracle: for
each sequence, the oracle's causal prefill of the Lq new rows onto that
sequence's seqlens[b] cached rows (the chunked-prefill reading the oracle pins
against the guide's L = 2 demonstration)."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode, decode_mq, device_error, prefill
from exact_tiled_attention_gqa_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    device_error(reset=True)
    yield
    assert device_error(reset=True) == 0


def _inputs(B, Hq, Hkv, Lq, Lmax, D, seqlens, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    for b, n in enumerate(seqlens):
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    return q, k, v, torch.tensor(seqlens, dtype=torch.int32)


def _oracle(oracle_mod, q, k, v, seqlens, scale):
    B, Hq, Lq, D = q.shape
    outs, lses = [], []
    for b in range(B):
        n = int(seqlens[b])
        o, l = oracle_mod.attention_prefill(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], scale, True)
        outs.append(o[0])
        lses.append(l[0])
    return np.stack(outs), np.stack(lses)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G,Lq", [(4, 1), (4, 2), (4, 4), (4, 8), (4, 16), (1, 16), (8, 8), (2, 5), (3, 7), (16, 4),
                                  (32, 2), (64, 1), (4, 32), (8, 16), (64, 2), (3, 40)])
def test_multi_query_against_oracle(oracle_mod, D, G, Lq):
    Hkv = 2
    seqlens = [700, Lq, 1, 333, 65, 4100]
    seqlens = [s for s in seqlens]
    Lmax = max(seqlens)
    q, k, v, sl = _inputs(len(seqlens), G * Hkv, Hkv, Lq, Lmax, D, seqlens, seed=G * 100 + Lq + D)
    scale = 1 / math.sqrt(D)
    out, lse = decode_mq(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = _oracle(oracle_mod, q, k, v, sl, scale)
    assert_close(out, lse, ref_o, ref_l, f"G{G} Lq{Lq} D{D}")


def test_lq1_is_decode():
    q, k, v, sl = _inputs(3, 8, 2, 1, 900, 128, [900, 17, 450], seed=5)
    q, k, v, sl = q.cuda(), k.cuda(), v.cuda(), sl.cuda()
    a, la = decode_mq(q, k, v, sl)
    b, lb = decode(q[:, :, 0].contiguous(), k, v, sl)
    torch.cuda.synchronize()
    assert torch.equal(a[:, :, 0], b) and torch.equal(la[:, :, 0], lb)


def test_verify_matches_chunked_prefill():
    """With equal lengths, Lq new tokens against the cache = the last Lq rows of a causal prefill."""
    B, Hq, Hkv, L, D, Lq = 2, 8, 2, 777, 128, 6
    q, k, v = (t.cuda() for t in W.prefill_inputs(B, Hq, Hkv, L, L, D, seed=3))
    po, pl = prefill(q, k, v, is_causal=True)
    mo, ml = decode_mq(q[:, :, -Lq:].contiguous(), k, v, torch.full((B,), L, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert (po[:, :, -Lq:].float() - mo.float()).abs().max().item() <= 2e-2
    assert (pl[:, :, -Lq:] - ml).abs().max().item() <= 1e-3


def test_too_many_rows_rejected():
    from exact_tiled_attention_gqa_b200 import AttnError
    q = torch.zeros(1, 8, 17, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(AttnError, match="G \\* Lq"):
        decode_mq(q, k, k, torch.tensor([64], dtype=torch.int32, device="cuda"))
