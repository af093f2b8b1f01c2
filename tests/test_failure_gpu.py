"""Failure behaviour on the GPU, without faulting it.

Every pipeline wait in the kernels is bounded: it gives up after a time limit,
records ATTN_DEVERR_TIMEOUT in the device error word and raises the CTA's abort
flag, so the CTA's other waits end as well and the kernel returns.  Here a
diagnostic kernel makes such a wait run out on purpose -- a barrier that is
announced but never completed, with a 1 ms limit -- and the test checks that

  * the call completes, the consumer's wait reports failure after about its
    limit, and the producer's wait (whose own limit is 2 s) ends through the
    abort flag within milliseconds;
  * the error word holds exactly ATTN_DEVERR_TIMEOUT, and clearing it works;
  * the context stays usable: prefill and decode right afterwards still match
    the fp64 oracle with a clean error word;
  * the persistent prefill's scheduling counters are all back at zero.
"""
import ctypes
import math

import pytest
import torch

import exact_tiled_attention_gqa_b200 as attn
from exact_tiled_attention_gqa_b200 import _native
from exact_tiled_attention_gqa_b200 import workloads as W
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    attn.device_error(reset=True)
    yield
    assert attn.device_error(reset=True) == 0


def _sched_busy():
    n = ctypes.c_int(-1)
    _native.check(_native.lib().attn_prefill_sched_busy(ctypes.byref(n)), "attn_prefill_sched_busy")
    return n.value


def _wait_selftest(limit_ns):
    res = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    st = _native.lib().attn_selftest_wait(limit_ns, ctypes.c_void_p(res.data_ptr()),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    _native.check(st, "attn_selftest_wait")
    torch.cuda.synchronize()
    return res.cpu().tolist()


@pytest.mark.parametrize("limit_ms", [1, 20])
def test_wait_runs_out_and_unwinds(oracle_mod, limit_ms):
    assert attn.device_error(reset=True) == 0
    prod_ok, prod_us, cons_ok, cons_us = _wait_selftest(limit_ms * 1_000_000)
    assert cons_ok == 0 and prod_ok == 0
    # the consumer gave up after its own limit (checked every 64 spins, so a little later)
    assert limit_ms * 1000 <= cons_us < limit_ms * 1000 + 50_000, cons_us
    # the producer's 2 s wait ended through the abort flag, not its own limit
    assert prod_us < limit_ms * 1000 + 50_000, prod_us
    assert attn.device_error(reset=True) == _native.ATTN_DEVERR_TIMEOUT
    assert attn.device_error(reset=True) == 0

    # the context is still good: exact results right after
    q, k, v = W.prefill_inputs(2, 16, 4, 700, 700, 128, seed=5)
    out, lse = attn.prefill(q.cuda(), k.cuda(), v.cuda(), is_causal=True)
    seqlens = [700, 1, 333, 0]
    dq = torch.randn(4, 16, 128, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    dout, dlse = attn.decode(dq.cuda(), k[:1].expand(4, -1, -1, -1).contiguous().cuda(),
                             v[:1].expand(4, -1, -1, -1).contiguous().cuda(),
                             torch.tensor(seqlens, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, 1 / math.sqrt(128), True)
    assert_close(out, lse, ref_o, ref_l, "prefill after a timed-out wait")
    kc = k[:1].expand(4, -1, -1, -1).contiguous()
    vc = v[:1].expand(4, -1, -1, -1).contiguous()
    ref_o, ref_l = oracle_mod.attention_decode(dq, kc, vc, seqlens, 1 / math.sqrt(128))
    assert_close(dout, dlse, ref_o, ref_l, "decode after a timed-out wait")
    assert _sched_busy() == 0


def test_sched_counters_zero_between_launches():
    """Every persistent launch leaves its counters at zero, at D = 64 and 128, for
    unit counts below, at and above the SM count."""
    for D, B, L in ((64, 1, 300), (128, 4, 2000), (128, 1, 8192)):
        q, k, v = (t.cuda() for t in W.prefill_inputs(B, 32, 8, L, L, D, seed=D + L))
        for _ in range(3):
            attn.prefill(q, k, v, is_causal=True)
        assert _sched_busy() == 0, (D, B, L)
    assert attn.device_error(reset=True) == 0
