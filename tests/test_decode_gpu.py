"""GPU parity for attn_decode (through the C ABI) against the fp64 oracle.

Cache rows at or beyond seqlens[b] are filled with NaN to show they are never
used.  Every case compares every (batch, head) row, the full-size Qwen3-8B
decode batch and the whole group-size sweep included.
"""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode, device_error
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


def _inputs(B, Hq, Hkv, Lmax, D, seqlens, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    for b, n in enumerate(seqlens):
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    return q, k, v, sl


def _check(oracle_mod, q, k, v, sl, what):
    D = q.shape[-1]
    out, lse = decode(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), scale=1 / math.sqrt(D))
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_decode(q, k, v, sl, 1 / math.sqrt(D))
    return assert_close(out, lse, ref_o, ref_l, what)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32, 64, 128, 3, 12, 17, 24, 48, 96])
def test_group_sizes(oracle_mod, D, G):
    Hkv = 2 if G <= 64 else 1
    seqlens = [700, 1, 333, 64, 65, 129, 128, 127]
    q, k, v, sl = _inputs(len(seqlens), G * Hkv, Hkv, 700, D, seqlens, seed=G * 10 + D)
    _check(oracle_mod, q, k, v, sl, f"G{G} D{D}")


@pytest.mark.parametrize("Lmax,seqlens", [(5000, [5000, 4097, 4096, 4095, 1, 2500]), (64, [64, 63]),
                                          (1, [1, 1]), (9000, [0, 9000])])
def test_split_edges(oracle_mod, Lmax, seqlens):
    q, k, v, sl = _inputs(len(seqlens), 8, 2, Lmax, 128, seqlens, seed=Lmax)
    _check(oracle_mod, q, k, v, sl, f"Lmax{Lmax}")


@pytest.mark.parametrize("Lmax,seqlens", [(5000, [5000, 4097, 4096, 4095, 1, 2500]), (9000, [0, 9000, 2049])])
def test_split_edges_d256(oracle_mod, Lmax, seqlens):
    q, k, v, sl = _inputs(len(seqlens), 8, 2, Lmax, 256, seqlens, seed=Lmax + 1)
    _check(oracle_mod, q, k, v, sl, f"D256 Lmax{Lmax}")


def test_zero_length_sequence(oracle_mod):
    q, k, v, sl = _inputs(2, 4, 1, 100, 128, [0, 50], seed=1)
    out, lse = decode(q.cuda(), k.cuda(), v.cuda(), sl.cuda())
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))


def test_decode_matches_prefill_last_row(oracle_mod):
    from exact_tiled_attention_gqa_b200 import prefill
    B, Hq, Hkv, L, D = 2, 8, 2, 400, 128
    q, k, v = (t.cuda() for t in W.prefill_inputs(B, Hq, Hkv, L, L, D, seed=9))
    po, pl = prefill(q, k, v, is_causal=True)
    do, dl = decode(q[:, :, -1].contiguous(), k, v, torch.full((B,), L, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert (po[:, :, -1].float() - do.float()).abs().max().item() <= 2e-2
    assert (pl[:, :, -1] - dl).abs().max().item() <= 1e-3


def _full_check(oracle_mod, shape, seed, fill_nan):
    """Every (batch, head) row of a full-size decode against the oracle, streamed
    one slab of at most 8 KV heads (and their query heads) of one sequence at a time."""
    q, k, v, sl = W.decode_inputs_for(shape, seed=seed, device="cuda", fill_beyond=float("nan") if fill_nan else None)
    out, lse = decode(q, k, v, sl)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    G = shape.G
    out_h, lse_h, q_h = out.cpu(), lse.cpu(), q.cpu()
    for b in range(shape.B):
        n = int(sl[b])
        for g0 in range(0, shape.Hkv, 8):
            g1 = min(shape.Hkv, g0 + 8)
            kb = k[b:b + 1, g0:g1, :n].cpu()
            vb = v[b:b + 1, g0:g1, :n].cpu()
            qb = q_h[b:b + 1, g0 * G:g1 * G]
            ref_o, ref_l = oracle_mod.attention_decode(qb, kb, vb, np.array([n], np.int32), shape.scale)
            assert_close(out_h[b:b + 1, g0 * G:g1 * G], lse_h[b:b + 1, g0 * G:g1 * G], ref_o, ref_l,
                         f"{shape.name} b{b} kv heads {g0}..{g1 - 1}")


@pytest.mark.slow
def test_qwen_decode_full_size_every_row(oracle_mod):
    _full_check(oracle_mod, W.QWEN_DECODE, seed=0, fill_nan=True)


@pytest.mark.slow
@pytest.mark.parametrize("G", W.GROUP_SWEEP)
def test_group_sweep_full_size_every_row(oracle_mod, G):
    _full_check(oracle_mod, W.group_sweep_decode(G), seed=G, fill_nan=False)


@pytest.mark.parametrize("n_parts,D", [(2, 128), (3, 64), (4, 256), (1, 128)])
def test_partial_and_merge_equal_full_decode(oracle_mod, n_parts, D):
    """KV parallelism on one GPU: the cache split by rows into n_parts shards, each
    decoded with decode_partial, merged with decode_merge, equals the whole decode."""
    from exact_tiled_attention_gqa_b200 import decode_merge, decode_partial
    from exact_tiled_attention_gqa_b200.multigpu import kv_shard_rows, shard_seqlens
    seqlens = [5000, 4097, 1, 0, 2500, 700]
    Lmax = 5000
    q, k, v, sl = _inputs(len(seqlens), 16, 2, Lmax, D, seqlens, seed=n_parts * 10 + D)
    qd, kd, vd, sld = q.cuda(), k.cuda(), v.cuda(), sl.cuda()
    os_, ls_ = [], []
    for r in range(n_parts):
        rows = kv_shard_rows(Lmax, r, n_parts)
        o, l = decode_partial(qd, kd[:, :, rows.start:rows.stop].contiguous(), vd[:, :, rows.start:rows.stop].contiguous(),
                              shard_seqlens(sld, rows), scale=1 / math.sqrt(D))
        os_.append(o)
        ls_.append(l)
    out, lse = decode_merge(torch.stack(os_), torch.stack(ls_))
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_decode(q, k, v, sl, 1 / math.sqrt(D))
    assert_close(out, lse, ref_o, ref_l, f"kv-parallel x{n_parts} D{D}")
