"""Seeded random shapes through prefill and decode, every output element against
the fp64 oracle.

The cases are drawn once from a fixed numpy seed (the list is the same on every
run): batch, heads and group size (including group sizes that do not divide
the 128-row tile), query and key lengths from 1 to a few tiles on either side of
a tile boundary, head dims 64 / 128 / 256, causal and full attention; decode
with cache lengths from 0 to Lmax, one to sixteen new rows per sequence, bf16 and
8-bit caches; and prefills of 149 to 591 long work units, whose part-filled last
wave is cut into key runs and merged.  They complement the hand-picked edge cases
of the other parity files with combinations nobody chose.
"""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode, decode_kv8, decode_mq, device_error, prefill, prefill_workspace_size
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


def _near_tile(rng, hi):
    """A length in [1, hi], often within a few of a multiple of 128."""
    if rng.random() < 0.5:
        return int(rng.integers(1, hi + 1))
    base = 128 * int(rng.integers(1, max(2, hi // 128 + 1)))
    return int(min(hi, max(1, base + int(rng.integers(-2, 3)))))


def _prefill_cases(n=64, seed=20251203):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        D = int(rng.choice([64, 128, 256]))
        G = int(rng.choice([1, 2, 3, 4, 5, 6, 8, 16, 32]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 3))
        Lk = _near_tile(rng, 700)
        Lq = Lk if rng.random() < 0.5 else _near_tile(rng, 700)
        causal = bool(rng.random() < 0.75)
        cases.append((B, G * Hkv, Hkv, Lq, Lk, D, causal, seed + i))
    return cases


def _decode_cases(n=48, seed=20251204):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        D = int(rng.choice([64, 128, 256]))
        G = int(rng.choice([1, 2, 4, 5, 8, 12, 16, 24, 32, 64]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 5))
        Lmax = _near_tile(rng, 3000)
        seqlens = [int(x) for x in rng.integers(0, Lmax + 1, size=B)]
        seqlens[int(rng.integers(0, B))] = Lmax   # one full-length sequence per case
        cases.append((B, G * Hkv, Hkv, Lmax, D, seqlens, seed + i))
    return cases


def _key_split_cases(n=6, seed=20251207):
    """Launches of 149 .. 591 units, all of at least 8 key tiles, and not a whole number
    of 148-unit waves: the shapes whose last wave is cut into key runs."""
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        D = int(rng.choice([64, 128]))
        G = int(rng.choice([1, 2, 4, 8]))
        P = 128 // G
        Hkv = int(rng.choice([1, 2, 4, 8]))
        B = int(rng.integers(1, 3))
        n_mblk = -(-int(rng.integers(160, 580)) // (B * Hkv))
        Lq = n_mblk * 2 * P - int(rng.integers(0, 2 * P))
        causal = bool(rng.random() < 0.7)
        Lk = Lq + int(rng.integers(1024, 3000)) if causal else int(rng.integers(1024, 5000))
        units = B * Hkv * -(-Lq // (2 * P))
        if 148 < units < 592 and units % 148 and B * G * Hkv * Lq * Lk <= 3e8:
            cases.append((B, G * Hkv, Hkv, Lq, Lk, D, causal, seed + len(cases)))
    return cases


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,seed", _key_split_cases())
def test_random_prefill_key_split(oracle_mod, B, Hq, Hkv, Lq, Lk, D, causal, seed):
    assert prefill_workspace_size(B, Hq, Hkv, Lq, Lk, D, causal) > 0, "the key split should apply"
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=seed)
    scale = 1.0 / math.sqrt(D)
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, is_causal=causal)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, causal)
    assert_close(out, lse, ref_o, ref_l, f"key split B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} Lk{Lk} D{D} causal{causal}")


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,seed", _prefill_cases())
def test_random_prefill(oracle_mod, B, Hq, Hkv, Lq, Lk, D, causal, seed):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=seed)
    scale = 1.0 / math.sqrt(D)
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, is_causal=causal)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, causal)
    assert_close(out, lse, ref_o, ref_l, f"B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} Lk{Lk} D{D} causal{causal}")


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,D,seqlens,seed", _decode_cases())
def test_random_decode(oracle_mod, B, Hq, Hkv, Lmax, D, seqlens, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    for b, n in enumerate(seqlens):   # rows past a sequence's length are never read
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    sl = torch.tensor(seqlens, dtype=torch.int32)
    scale = 1.0 / math.sqrt(D)
    out, lse = decode(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_decode(q, k, v, sl, scale)
    assert_close(out, lse, ref_o, ref_l, f"B{B} Hq{Hq} Hkv{Hkv} Lmax{Lmax} D{D} seqlens{seqlens}")


def _mq_cases(n=32, seed=20251205):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        D = int(rng.choice([64, 128, 256]))
        Lq = int(rng.choice([1, 2, 3, 4, 6, 8, 16]))
        G = int(rng.choice([g for g in (1, 2, 3, 4, 5, 8, 16, 32, 64) if g * Lq <= 128]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 5))
        Lmax = _near_tile(rng, 2500)
        seqlens = [int(x) for x in rng.integers(0, Lmax + 1, size=B)]
        seqlens[int(rng.integers(0, B))] = Lmax
        cases.append((B, G * Hkv, Hkv, Lq, Lmax, D, seqlens, seed + i))
    return cases


def _kv8_cases(n=32, seed=20251206):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        fmt = str(rng.choice([W.KV_E4M3, W.KV_Q8_0]))
        D = int(rng.choice([64, 128]))
        Lq = int(rng.choice([1, 1, 2, 4]))
        G = int(rng.choice([g for g in (1, 2, 3, 4, 5, 8, 12, 16, 32, 64) if g * Lq <= 64]))
        Hkv = int(rng.integers(1, 4))
        B = int(rng.integers(1, 5))
        Lmax = _near_tile(rng, 2500)
        if fmt == W.KV_Q8_0:   # the q8_0 scale plane needs Lmax % 4 == 0 (16-byte rows for TMA)
            Lmax = max(4, Lmax - Lmax % 4)
        seqlens = [int(x) for x in rng.integers(0, Lmax + 1, size=B)]
        seqlens[int(rng.integers(0, B))] = Lmax
        cases.append((fmt, B, G * Hkv, Hkv, Lq, Lmax, D, seqlens, seed + i))
    return cases


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lmax,D,seqlens,seed", _mq_cases())
def test_random_decode_mq(oracle_mod, B, Hq, Hkv, Lq, Lmax, D, seqlens, seed):
    """Lq new rows per sequence, bottom-right against seqlens[b] cached rows: the oracle is
    the causal prefill of those rows onto that sequence's rows."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    for b, n in enumerate(seqlens):
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    sl = torch.tensor(seqlens, dtype=torch.int32)
    scale = 1.0 / math.sqrt(D)
    out, lse = decode_mq(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    outs, lses = [], []
    for b in range(B):
        n = seqlens[b]
        o, l = oracle_mod.attention_prefill(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], scale, True)
        outs.append(o[0])
        lses.append(l[0])
    assert_close(out, lse, np.stack(outs), np.stack(lses), f"B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} D{D} seqlens{seqlens}")


@pytest.mark.parametrize("fmt,B,Hq,Hkv,Lq,Lmax,D,seqlens,seed", _kv8_cases())
def test_random_decode_kv8(oracle_mod, fmt, B, Hq, Hkv, Lq, Lmax, D, seqlens, seed):
    """8-bit caches with NaN codes (E4M3) or NaN / inf scales (q8_0) past every length; the
    oracle dequantises exactly."""
    q, k, v, ks, vs, _ = W.decode_inputs_kv8(B, Hq, Hkv, Lmax, D, 1, Lmax, fmt, seed=seed, Lq=Lq)
    for b, n in enumerate(seqlens):
        if fmt == W.KV_E4M3:
            k[b, :, n:].view(torch.uint8).fill_(0x7F)
            v[b, :, n:].view(torch.uint8).fill_(0xFF)
        else:
            ks[b, :, n:] = float("nan")
            vs[b, :, n:] = float("inf")
    sl = torch.tensor(seqlens, dtype=torch.int32)
    scale = 1.0 / math.sqrt(D)
    out, lse = decode_kv8(q.cuda(), k.cuda(), v.cuda(), ks.cuda(), vs.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ofmt = oracle_mod.KV_E4M3 if fmt == W.KV_E4M3 else oracle_mod.KV_Q8_0
    ref_o, ref_l = oracle_mod.attention_decode_kv8(q, k, v, ofmt, ks, vs, sl, scale)
    assert_close(out, lse, ref_o, ref_l, f"{fmt} B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} D{D} seqlens{seqlens}")
