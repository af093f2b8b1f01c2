"""attn_decode_host (q, seqlens in and out, lse back in host memory; the KV
cache on the device) against the device-buffer attn_decode and the fp64
oracle.  The call runs the same kernels on device copies of its inputs, so
its results must equal attn_decode's bit for bit."""
import math

import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode, decode_host, decode_host_workspace_size, device_error
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
    for b, n in enumerate(seqlens):   # rows past a sequence's length are never read
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    return q, k, v, torch.tensor(seqlens, dtype=torch.int32)


@pytest.mark.parametrize("B,Hq,Hkv,Lmax,D,seqlens", [
    (3, 8, 2, 700, 128, [700, 1, 333]), (2, 32, 1, 2100, 128, [2100, 64]), (4, 16, 4, 300, 64, [0, 299, 5, 300]),
    (2, 16, 2, 1500, 256, [1500, 777])])
def test_host_equals_device_and_oracle(oracle_mod, B, Hq, Hkv, Lmax, D, seqlens):
    q, k, v, sl = _inputs(B, Hq, Hkv, Lmax, D, seqlens, seed=B * 10 + Hq + D)
    kd, vd = k.cuda(), v.cuda()
    ref_o, ref_l = decode(q.cuda(), kd, vd, sl.cuda())
    stream = torch.cuda.Stream()
    out, lse = decode_host(q.pin_memory(), kd, vd, sl.pin_memory(), stream=stream)
    stream.synchronize()
    assert device_error(reset=True) == 0
    assert torch.equal(out, ref_o.cpu()) and torch.equal(lse, ref_l.cpu())
    o64, l64 = oracle_mod.attention_decode(q, k, v, sl, 1 / math.sqrt(D))
    assert_close(out, lse, o64, l64, f"decode_host D{D}")


def test_host_pageable_no_lse_and_workspace_reuse():
    """Pageable host memory, no LSE, one workspace for two calls with new queries."""
    B, Hq, Hkv, Lmax, D = 4, 32, 8, 1024, 128
    q, k, v, sl = _inputs(B, Hq, Hkv, Lmax, D, [1024, 17, 512, 900], seed=3)
    kd, vd = k.cuda(), v.cuda()
    ws = torch.empty(decode_host_workspace_size(B, Hq, Hkv, Lmax, D), dtype=torch.uint8, device="cuda")
    out1, lse1 = decode_host(q, kd, vd, sl, want_lse=False, workspace=ws)
    q2 = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    out2, _ = decode_host(q2, kd, vd, sl, workspace=ws)
    torch.cuda.synchronize()
    assert lse1 is None
    assert torch.equal(out1, decode(q.cuda(), kd, vd, sl.cuda())[0].cpu())
    assert torch.equal(out2, decode(q2.cuda(), kd, vd, sl.cuda())[0].cpu())


def test_host_qwen_batch(oracle_mod):
    """The Qwen3-8B decode batch (B 64, lengths up to 32768) through the host call, every row
    against attn_decode and a sample of rows against the oracle."""
    s = W.QWEN_DECODE
    q, k, v, sl = W.decode_inputs_for(s, seed=0, device="cuda")
    ref_o, ref_l = decode(q, k, v, sl)
    out, lse = decode_host(q.cpu().pin_memory(), k, v, sl.cpu().pin_memory())
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o.cpu()) and torch.equal(lse, ref_l.cpu())
    for b in (0, 31, 63):
        n = int(sl[b])
        o64, l64 = oracle_mod.attention_decode(q[b:b + 1].cpu(), k[b:b + 1, :, :n].cpu(), v[b:b + 1, :, :n].cpu(),
                                               torch.tensor([n], dtype=torch.int32), s.scale)
        assert_close(out[b:b + 1], lse[b:b + 1], o64, l64, f"decode_host qwen b{b}")
