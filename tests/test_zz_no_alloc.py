"""attn_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers own no device memory of their own to lend -- an inference engine
that reserves nearly all of HBM for its pool up front, or a hot loop that must
not call cudaMalloc because it can synchronise the device.  For them the
library keeps the decode split partials in a fixed scratch array of its own.

This file checks, through the C ABI (and once through the Python wrapper):
  * two calls in a row give the same result as attn_decode with a caller
    workspace, within the parity tolerances, for each decode kernel family
    (the mma.sync split kernel, the tcgen05 kernel at G = 32, and D = 256);
  * one case against the fp64 oracle on sampled (batch, head) rows;
  * a second call with fewer splits than the first, so the scratch still holds
    the first call's extra partials, which must not leak into the result;
  * sizes beyond the scratch are refused.
It is named to run last, so a failure here stops a `-x` run only after every
other test has run.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import _native, decode, decode_noalloc, decode_workspace_size, device_error
from parity import LSE_MAX_ABS, O_MAX_ABS, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return _native.lib()


def _inputs(B, Hq, Hkv, Lmax, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    sl = torch.randint(0, Lmax + 1, (B,), generator=g, dtype=torch.int32)
    sl[0] = Lmax
    return q, k, v, sl


def _call_noalloc(lib, q, k, v, sl, out, lse):
    B, Hq, D = q.shape
    Hkv, Lmax = k.shape[1], k.shape[2]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.attn_decode_noalloc(p(q), p(k), p(v), p(sl), p(out), p(lse), B, Hq, Hkv, Lmax, D,
                                   1.0 / math.sqrt(D), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same_as_decode(out, lse, ref_o, ref_l):
    assert (out.float() - ref_o.float()).abs().max().item() <= O_MAX_ABS
    fin = torch.isfinite(ref_l)
    assert torch.equal(torch.isneginf(lse), torch.isneginf(ref_l))
    assert (lse[fin] - ref_l[fin]).abs().max().item() <= LSE_MAX_ABS


@pytest.mark.parametrize("shape", [(6, 32, 8, 3000, 128), (3, 16, 1, 9000, 64), (2, 64, 2, 4000, 128),
                                   (2, 32, 2, 2000, 256)],
                         ids=["split-G4", "split-G16-D64", "tcgen05-G32", "D256"])
def test_two_calls_match_attn_decode(lib, shape):
    B, Hq, Hkv, Lmax, D = shape
    assert decode_workspace_size(B, Hq, Hkv, Lmax, D) <= _native.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    device_error(reset=True)
    for seed in (1, 2):   # two calls in a row, different inputs: no state carries over
        q, k, v, sl = (t.cuda() for t in _inputs(B, Hq, Hkv, Lmax, D, seed + D))
        ref_o, ref_l = decode(q, k, v, sl)
        out = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        assert _call_noalloc(lib, q, k, v, sl, out, lse) == 0, lib.attn_last_error()
        torch.cuda.synchronize()
        _same_as_decode(out, lse, ref_o, ref_l)
    assert device_error(reset=True) == 0


def test_fewer_splits_after_more_against_the_oracle(lib, oracle_mod):
    """A long call fills many splits of the scratch; a shorter one right after
    uses fewer, through the Python wrapper, and is checked against the oracle."""
    device_error(reset=True)
    qa, ka, va, sla = (t.cuda() for t in _inputs(4, 32, 8, 20000, 128, 7))
    out_a = torch.empty_like(qa)
    lse_a = torch.empty(4, 32, dtype=torch.float32, device="cuda")
    decode_noalloc(qa, ka, va, sla, out=out_a, lse=lse_a)
    q, k, v, sl = _inputs(4, 32, 8, 2500, 128, 8)
    assert decode_workspace_size(4, 32, 8, 2500, 128) < decode_workspace_size(4, 32, 8, 20000, 128)
    out = torch.empty(4, 32, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(4, 32, dtype=torch.float32, device="cuda")
    decode_noalloc(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), out=out, lse=lse)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    rng = np.random.default_rng(3)
    pairs = [(0, 0), (3, 31)] + [(int(rng.integers(4)), int(rng.integers(32))) for _ in range(10)]
    for b, h in pairs:
        g = h // 4
        n = int(sl[b])
        ref_o, ref_l = oracle_mod.attention_decode(q[b:b + 1, h:h + 1], k[b:b + 1, g:g + 1, :n],
                                                   v[b:b + 1, g:g + 1, :n], np.array([n], np.int32),
                                                   1 / math.sqrt(128))
        assert_close(out[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], ref_o, ref_l, f"noalloc b{b} h{h}")
    ref_o, ref_l = decode(qa, ka, va, sla)
    torch.cuda.synchronize()
    _same_as_decode(out_a, lse_a, ref_o, ref_l)


def test_oversize_is_refused(lib):
    # Hq=64, Lmax=131072 at B=64 needs far more partials than the 16 MiB scratch
    B, Hq, Hkv, Lmax, D = 64, 64, 8, 131072, 128
    assert decode_workspace_size(B, Hq, Hkv, Lmax, D) > _native.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    st = lib.attn_decode_noalloc(a, a, a, a, a, None, B, Hq, Hkv, Lmax, D, 0.1, None)
    assert st == _native.ATTN_ERR_WORKSPACE
    assert b"static scratch" in lib.attn_last_error()
