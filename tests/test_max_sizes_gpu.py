"""Large-size edge cases, checked on sampled rows the oracle computes one by one:
a cache of 2^20 rows for one sequence (256 splits), a batch of 1024 short
sequences (one split each, many rows of zero length), and a 65536-token causal
prefill (the longest the guide's tables reach)."""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import decode, device_error, prefill
from exact_tiled_attention_gqa_b200 import workloads as W
from parity import assert_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    device_error(reset=True)
    yield
    assert device_error(reset=True) == 0


def _check_decode_rows(oracle_mod, q, k, v, sl, out, lse, pairs, scale):
    G = q.shape[1] // k.shape[1]
    for b, h in pairs:
        n = int(sl[b])
        g = h // G
        ref_o, ref_l = oracle_mod.attention_decode(q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, g:g + 1, :n].cpu(),
                                                   v[b:b + 1, g:g + 1, :n].cpu(), np.array([n], np.int32), scale)
        assert_close(out[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1], ref_o, ref_l, f"b{b} h{h} n{n}")


def test_decode_one_million_rows(oracle_mod):
    q, k, v, sl = W.decode_inputs(1, 8, 1, 1 << 20, 128, (1 << 20) - 3, (1 << 20) - 3, seed=1, device="cuda")
    out, lse = decode(q, k, v, sl)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    _check_decode_rows(oracle_mod, q, k, v, sl, out, lse, [(0, 0), (0, 5), (0, 7)], 1 / math.sqrt(128))


def test_decode_many_short_sequences(oracle_mod):
    q, k, v, sl = W.decode_inputs(1024, 16, 2, 96, 64, 0, 96, seed=2, device="cuda", fill_beyond=float("nan"))
    out, lse = decode(q, k, v, sl)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    empty = (sl == 0).nonzero().flatten().tolist()
    for b in empty[:8]:
        assert torch.all(out[b] == 0) and torch.all(torch.isneginf(lse[b]))
    rng = np.random.default_rng(2)
    pairs = [(int(rng.integers(1024)), int(rng.integers(16))) for _ in range(24)]
    _check_decode_rows(oracle_mod, q, k, v, sl, out, lse, [p for p in pairs if int(sl[p[0]]) > 0], 1 / math.sqrt(64))


def test_prefill_64k_tokens(oracle_mod):
    L = 65536
    q, k, v = (t.cuda() for t in W.prefill_inputs(1, 8, 1, L, L, 128, seed=3))
    out, lse = prefill(q, k, v, is_causal=True)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    rows = [0, 1, 127, 128, 4095, 32767, 32768, L - 129, L - 2, L - 1]
    ref_o, ref_l = oracle_mod.attention_prefill(q.cpu(), k.cpu(), v.cpu(), 1 / math.sqrt(128), True, rows=rows)
    assert_close(out[:, :, rows], lse[:, :, rows], ref_o, ref_l, "L65536")
