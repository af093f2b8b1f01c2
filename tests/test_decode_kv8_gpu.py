"""GPU parity for attn_decode_kv8 (8-bit KV cache, through the C ABI) against
the fp64 oracle, which dequantises the codes exactly and runs the pinned
eager attention.  Rows past each sequence's length hold NaN codes (E4M3) or
NaN scales (q8_0), to show they are never used."""
import ctypes
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import _native, decode_kv8, decode_mq, device_error
from exact_tiled_attention_gqa_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu

FMTS = {W.KV_E4M3: 1, W.KV_Q8_0: 2}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    device_error(reset=True)
    yield
    assert device_error(reset=True) == 0


def _oracle_fmt(oracle_mod, fmt):
    return oracle_mod.KV_E4M3 if fmt == W.KV_E4M3 else oracle_mod.KV_Q8_0


def test_code_conversion_matches_torch():
    """Every pair of codes, as the kernel converts them for its f16 MMAs."""
    codes = torch.from_numpy(np.arange(65536, dtype=np.uint16).view(np.int16)).cuda()
    out = torch.empty(65536, dtype=torch.int32, device="cuda")
    for fmt, code in FMTS.items():
        st = _native.lib().attn_selftest_kv8_convert(ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                                     65536, code, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0
        torch.cuda.synchronize()
        got = out.cpu().view(torch.float16).view(65536, 2).double()
        b = torch.arange(65536, dtype=torch.int32)
        lo, hi = (b & 0xFF).to(torch.uint8), ((b >> 8) & 0xFF).to(torch.uint8)
        if fmt == W.KV_E4M3:
            want = torch.stack([lo.view(torch.float8_e4m3fn).double(), hi.view(torch.float8_e4m3fn).double()], 1)
        else:
            want = torch.stack([lo.view(torch.int8).double(), hi.view(torch.int8).double()], 1)
        nan = torch.isnan(want)
        assert torch.equal(torch.isnan(got), nan), fmt
        assert torch.equal(got[~nan], want[~nan]), fmt


def _run(oracle_mod, fmt, B_seqlens, Hq, Hkv, Lq, Lmax, D, seed):
    B = len(B_seqlens)
    q, k, v, ks, vs, _ = W.decode_inputs_kv8(B, Hq, Hkv, Lmax, D, 1, Lmax, fmt, seed=seed, Lq=Lq)
    sl = torch.tensor(B_seqlens, dtype=torch.int32)
    # rows past each length: NaN codes / scales (never used)
    for b, n in enumerate(B_seqlens):
        if fmt == W.KV_E4M3:
            k[b, :, n:].view(torch.uint8).fill_(0x7F)
            v[b, :, n:].view(torch.uint8).fill_(0xFF)
        else:
            k[b, :, n:] = -128
            v[b, :, n:] = 127
            ks[b, :, n:] = float("nan")
            vs[b, :, n:] = float("inf")
    scale = 1.0 / math.sqrt(D)
    out, lse = decode_kv8(q.cuda(), k.cuda(), v.cuda(), ks.cuda(), vs.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_decode_kv8(q, k, v, _oracle_fmt(oracle_mod, fmt), ks, vs, sl, scale)
    return assert_close(out, lse, ref_o, ref_l, f"{fmt} G{Hq // Hkv} Lq{Lq} D{D}")


@pytest.mark.parametrize("fmt", [W.KV_E4M3, W.KV_Q8_0])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G,Lq", [(1, 1), (4, 1), (8, 1), (16, 1), (3, 1), (4, 4), (2, 5), (32, 1), (8, 8), (64, 1),
                                  (12, 3)])
def test_kv8_against_oracle(oracle_mod, fmt, D, G, Lq):
    Hkv = 2
    seqlens = [700, max(Lq, 1), 333, 64, 65, 1300]
    _run(oracle_mod, fmt, seqlens, G * Hkv, Hkv, Lq, 1300, D, seed=G * 10 + Lq + D)


@pytest.mark.parametrize("fmt", [W.KV_E4M3, W.KV_Q8_0])
def test_kv8_split_edges(oracle_mod, fmt):
    """Lengths on and around the split and tile boundaries, a zero length, a full cache."""
    _run(oracle_mod, fmt, [5000, 4097, 4096, 4095, 0, 2500, 1, 63], 8, 2, 1, 5000, 128, seed=7)


def test_kv8_e4m3_equals_bf16_decode_on_same_values(oracle_mod):
    """With a power-of-two scale the E4M3 elements are exact in bf16: the bf16 decode on
    those elements agrees (to the bf16 output rounding)."""
    B, Hq, Hkv, L, D = 3, 8, 2, 900, 128
    q, k, v, _, _, sl = W.decode_inputs_kv8(B, Hq, Hkv, L, D, 100, L, W.KV_E4M3, seed=3)
    s = torch.full((Hkv,), 2.0 ** -6, dtype=torch.float32)
    a, la = decode_kv8(q.cuda(), k.cuda(), v.cuda(), s.cuda(), s.cuda(), sl.cuda())
    kb = (k.to(torch.float32) * 2.0 ** -6).to(torch.bfloat16)
    vb = (v.to(torch.float32) * 2.0 ** -6).to(torch.bfloat16)
    assert torch.equal(kb.float(), k.to(torch.float32) * 2.0 ** -6)
    b, lb = decode_mq(q.cuda(), kb.cuda(), vb.cuda(), sl.cuda())
    torch.cuda.synchronize()
    assert (a.float() - b.float()).abs().max().item() <= 2e-2
    assert (la - lb).abs().max().item() <= 1e-3


def test_kv8_large_query_values(oracle_mod):
    """Query rows with |q| far beyond f16 range: the per-row power-of-two rescale keeps them exact."""
    B, Hq, Hkv, L, D = 2, 4, 1, 300, 64
    q, k, v, ks, vs, sl = W.decode_inputs_kv8(B, Hq, Hkv, L, D, 50, L, W.KV_Q8_0, seed=9)
    q = (q.float() * torch.tensor([1e6, 1e-7, 3e4, 1.0]).view(1, Hq, 1, 1)).to(torch.bfloat16)
    scale = 1e-6
    out, lse = decode_kv8(q.cuda(), k.cuda(), v.cuda(), ks.cuda(), vs.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_mod.attention_decode_kv8(q, k, v, oracle_mod.KV_Q8_0, ks, vs, sl, scale)
    assert_close(out, lse, ref_o, ref_l, "large q")


@pytest.mark.slow
@pytest.mark.parametrize("fmt", [W.KV_E4M3, W.KV_Q8_0])
def test_kv8_full_size_every_row(oracle_mod, fmt):
    """The Qwen3-8B decode batch (B 64, 32 768 cached rows) with an 8-bit cache, every
    (b, head) row; the oracle dequantises and runs one sequence at a time."""
    shape = W.QWEN_DECODE_E4M3 if fmt == W.KV_E4M3 else W.QWEN_DECODE_Q8_0
    q, k, v, ks, vs, sl = W.decode_inputs_kv8(shape.B, shape.Hq, shape.Hkv, shape.Lmax, shape.D, shape.seqlen_lo,
                                              shape.seqlen_hi, fmt, seed=1, device="cuda", fill_beyond=True)
    out, lse = decode_kv8(q, k, v, ks, vs, sl, scale=shape.scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    out, lse, q_h = out.cpu(), lse.cpu(), q.cpu()
    for b in range(shape.B):
        n = int(sl[b])
        ksl = ks.cpu() if fmt == W.KV_E4M3 else ks[b:b + 1, :, :n].cpu()
        vsl = vs.cpu() if fmt == W.KV_E4M3 else vs[b:b + 1, :, :n].cpu()
        ref_o, ref_l = oracle_mod.attention_decode_kv8(q_h[b:b + 1], k[b:b + 1, :, :n].cpu(), v[b:b + 1, :, :n].cpu(),
                                                       _oracle_fmt(oracle_mod, fmt), ksl, vsl, np.array([n]),
                                                       shape.scale)
        assert_close(out[b:b + 1], lse[b:b + 1], ref_o, ref_l, f"{shape.name} b{b}")


def _paged_kv8(fmt, seqlens, Hq, Hkv, Lq, D, page_size, seed, spare_pages=2):
    """Contiguous 8-bit inputs, then the same rows scattered into shuffled pages
    (unused pages and rows hold NaN codes / NaN scales)."""
    B = len(seqlens)
    Lmax = max(64, -(-max(seqlens) // page_size) * page_size)
    q, k, v, ks, vs, _ = W.decode_inputs_kv8(B, Hq, Hkv, Lmax, D, 1, Lmax, fmt, seed=seed, Lq=Lq)
    pages_per = [max(1, -(-n // page_size)) for n in seqlens]
    max_pages = max(pages_per) + 1
    n_pages = sum(pages_per) + spare_pages
    order = torch.randperm(n_pages, generator=torch.Generator().manual_seed(seed))
    kp = torch.empty((n_pages, Hkv, page_size, D), dtype=k.dtype)
    vp = torch.empty_like(kp)
    kp.view(torch.uint8).fill_(0x7F if fmt == W.KV_E4M3 else 0x80)
    vp.view(torch.uint8).fill_(0x7F if fmt == W.KV_E4M3 else 0x80)
    if fmt == W.KV_Q8_0:
        ksp = torch.full((n_pages, Hkv, page_size, D // 32), float("nan"), dtype=torch.float16)
        vsp = torch.full_like(ksp, float("nan"))
    else:
        ksp, vsp = ks, vs
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(seqlens):
        for i in range(pages_per[b]):
            pg = int(order[nxt]); nxt += 1
            table[b, i] = pg
            rows = min(page_size, n - i * page_size)
            if rows <= 0:
                continue
            sl = slice(i * page_size, i * page_size + rows)
            kp[pg, :, :rows] = k[b, :, sl]
            vp[pg, :, :rows] = v[b, :, sl]
            if fmt == W.KV_Q8_0:
                ksp[pg, :, :rows] = ks[b, :, sl]
                vsp[pg, :, :rows] = vs[b, :, sl]
    return q, k, v, ks, vs, kp, vp, ksp, vsp, table


@pytest.mark.parametrize("fmt", [W.KV_E4M3, W.KV_Q8_0])
@pytest.mark.parametrize("page_size", [64, 128, 256])
@pytest.mark.parametrize("G,Lq,D", [(4, 1, 128), (8, 2, 64), (1, 1, 128), (32, 1, 128)])
def test_kv8_paged_against_oracle(oracle_mod, fmt, page_size, G, Lq, D):
    from exact_tiled_attention_gqa_b200 import decode_kv8_paged
    Hkv = 2
    seqlens = [1000, 1, 0, 257, 64, 2100]
    q, k, v, ks, vs, kp, vp, ksp, vsp, table = _paged_kv8(fmt, seqlens, G * Hkv, Hkv, Lq, D, page_size,
                                                           seed=page_size + G + Lq + D)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    scale = 1 / math.sqrt(D)
    out, lse = decode_kv8_paged(q.cuda(), kp.cuda(), vp.cuda(), ksp.cuda(), vsp.cuda(), table.cuda(), sl.cuda(),
                                scale=scale)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_decode_kv8(q, k, v, _oracle_fmt(oracle_mod, fmt), ks, vs, sl, scale)
    assert_close(out, lse, ref_o, ref_l, f"paged {fmt} ps{page_size} G{G} Lq{Lq} D{D}")
    # the same rows read contiguously give the same answer
    mo, ml = decode_kv8(q.cuda(), k.cuda(), v.cuda(), ks.cuda(), vs.cuda(), sl.cuda(), scale=scale)
    torch.cuda.synchronize()
    assert (mo.float() - out.float()).abs().max().item() <= 2e-2


def test_kv8_paged_bad_page_is_flagged():
    from exact_tiled_attention_gqa_b200 import decode_kv8_paged
    q, k, v, ks, vs, kp, vp, ksp, vsp, table = _paged_kv8(W.KV_E4M3, [300], 4, 1, 1, 128, 128, seed=1)
    table[0, 1] = 10_000
    decode_kv8_paged(q.cuda(), kp.cuda(), vp.cuda(), ksp.cuda(), vsp.cuda(), table.cuda(),
                     torch.tensor([300], dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert device_error(reset=True) & 0x4
