"""attn_prefill_host (host buffers in and out, copies overlapped with the
kernels by the library) against the device-buffer attn_prefill, which the
oracle parity tests cover: the per-unit kernels compute each row exactly as
the whole-batch kernel does, so the results must be bit-identical."""
import math

import pytest
import torch

from exact_tiled_attention_gqa_b200 import device_error, prefill, prefill_host, prefill_host_scratch_size
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


def _pin(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal", [
    (2, 8, 2, 300, 300, 128, True), (3, 32, 8, 1024, 1024, 128, True), (2, 16, 2, 500, 1300, 64, True),
    (1, 8, 8, 257, 257, 256, False), (4, 4, 1, 2048, 2048, 128, True), (2, 128, 1, 40, 300, 128, True)])
def test_host_equals_device(B, Hq, Hkv, Lq, Lk, D, causal):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=B * 100 + Hq + Lq)
    ref_o, ref_l = prefill(q.cuda(), k.cuda(), v.cuda(), is_causal=causal)
    stream = torch.cuda.Stream()
    out, lse = prefill_host(_pin(q), _pin(k), _pin(v), is_causal=causal, stream=stream)
    stream.synchronize()
    assert device_error(reset=True) == 0
    assert torch.equal(out, ref_o.cpu()) and torch.equal(lse, ref_l.cpu())


def test_host_pageable_no_lse_and_reuse(oracle_mod):
    """Pageable host memory, no LSE, and one scratch reused by two calls in a row."""
    B, Hq, Hkv, L, D = 2, 8, 2, 700, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, L, L, D, seed=5)
    scratch = torch.empty(prefill_host_scratch_size(B, Hq, Hkv, L, L, D), dtype=torch.uint8, device="cuda")
    out1, lse1 = prefill_host(q, k, v, want_lse=False, scratch=scratch)
    out2, lse2 = prefill_host(_pin(q), _pin(k), _pin(v), scratch=scratch)
    torch.cuda.synchronize()
    assert lse1 is None and torch.equal(out1, out2)
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, 1 / math.sqrt(D), True)
    assert_close(out2, lse2, ref_o, ref_l, "prefill_host")


def test_host_no_keys():
    q = torch.randn(1, 4, 5, 128).to(torch.bfloat16)
    e = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16)
    out, lse = prefill_host(q, e, e)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
