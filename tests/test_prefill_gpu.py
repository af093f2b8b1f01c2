"""GPU parity for attn_prefill (through the C ABI) against the fp64 oracle.

Every case compares every output element, the full-size Qwen3-8B-shaped and
chunked workloads included.
"""
import math

import numpy as np
import pytest
import torch

from exact_tiled_attention_gqa_b200 import device_error, prefill, prefill_workspace_size
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


def _run(oracle_mod, B, Hq, Hkv, Lq, Lk, D, causal, seed=0, spike=0, rows=None):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=seed, spike_every=spike)
    scale = 1.0 / math.sqrt(D)
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, is_causal=causal)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, causal, rows=rows)
    if rows is not None:
        out, lse = out[:, :, rows], lse[:, :, rows]
    assert device_error(reset=True) == 0
    return assert_close(out, lse, ref_o, ref_l, f"B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} Lk{Lk} D{D} causal{causal}")


def test_tiny_config(oracle_mod):
    s = W.TINY_PREFILL
    _run(oracle_mod, s.B, s.Hq, s.Hkv, s.Lq, s.Lk, s.D, True)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (6, 2), (32, 1), (5, 5)])
def test_ragged_multi_tile(oracle_mod, D, causal, Hq, Hkv):
    _run(oracle_mod, 2, Hq, Hkv, 300, 300, D, causal, seed=Hq * 7 + Hkv)


@pytest.mark.parametrize("Lq,Lk", [(77, 500), (1, 500), (2, 257), (128, 640), (250, 129), (129, 128), (1, 1),
                                   (3, 1), (200, 130), (513, 513)])
def test_chunked_bottom_right(oracle_mod, Lq, Lk):
    _run(oracle_mod, 1, 8, 2, Lq, Lk, 128, True, seed=Lq + Lk, spike=97)


def test_group_of_128_and_64(oracle_mod):
    _run(oracle_mod, 1, 128, 1, 40, 300, 128, True, seed=5)
    _run(oracle_mod, 1, 64, 1, 70, 200, 64, True, seed=6)
    _run(oracle_mod, 1, 128, 1, 20, 300, 256, True, seed=7)


@pytest.mark.parametrize("Lq,Lk", [(77, 500), (1, 500), (128, 640), (250, 129), (1, 1), (200, 130), (513, 513),
                                   (1000, 1700)])
def test_d256_chunked_and_long(oracle_mod, Lq, Lk):
    """D = 256 runs one Q tile per CTA with two S buffers in TMEM and a ring of
    half tiles; these cover 1 to 14 key tiles, so the ring and the buffers wrap."""
    _run(oracle_mod, 1, 8, 2, Lq, Lk, 256, True, seed=Lq + 3 * Lk, spike=97)


@pytest.mark.parametrize("D", [128, 256])
def test_rescale_on_every_tile(oracle_mod, D):
    """Keys whose scores climb by more than 2^8 (log2) per 128-key tile: the
    running max moves on every tile, so O is rescaled in TMEM each time (at
    D = 256 while the previous P.V product may still be in flight)."""
    B, Hq, Hkv, L = 1, 8, 2, 1400
    q, k, v = W.prefill_inputs(B, Hq, Hkv, L, L, D, seed=21)
    # q ~ ones / sqrt(D), k_j = noise + r_j ones: score * scale * log2 e ~ r_j log2 e,
    # with r_j stepping by 12 / log2 e per tile (a rise of about 2^12 per tile)
    ramp = (torch.arange(L, dtype=torch.float32) // 128) * (12.0 / math.log2(math.e))
    q = (1.0 / math.sqrt(D) + 0.1 * q.float()).to(torch.bfloat16)
    k = (0.5 * k.float() + ramp[None, None, :, None]).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(D)
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=scale, is_causal=True)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, True)
    assert device_error(reset=True) == 0
    assert_close(out, lse, ref_o, ref_l, f"rescale D{D}")


def test_no_keys_and_empty(oracle_mod):
    q = torch.randn(1, 4, 5, 128).to(torch.bfloat16).cuda()
    e = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    out, lse = prefill(q, e, e, is_causal=True)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    q0 = torch.empty(1, 4, 0, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(1, 2, 9, 128).to(torch.bfloat16).cuda()
    out0, lse0 = prefill(q0, k, k)
    assert out0.numel() == 0 and lse0.numel() == 0


def test_large_scores_stay_finite(oracle_mod):
    """Scores in the hundreds (inputs scaled by 8 and 4): the online max keeps exponentials bounded."""
    q, k, v = W.prefill_inputs(1, 8, 2, 256, 256, 128, seed=11)
    q, k = q * 8, k * 4
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=1 / math.sqrt(128), is_causal=True)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, 1 / math.sqrt(128), True)
    assert_close(out, lse, ref_o, ref_l, "large scores")


def test_deterministic(oracle_mod):
    q, k, v = (t.cuda() for t in W.prefill_inputs(2, 8, 2, 333, 333, 128, seed=3))
    a, la = prefill(q, k, v)
    b, lb = prefill(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("D", [64, 128])
def test_persistent_counters_reused_and_concurrent(oracle_mod, D):
    """For D <= 128 one CTA per SM takes work units from a per-launch counter
    (256 counters in turn, each put back to zero by its launch's last CTA).
    With 168 units (more than the SMs, so CTAs take several), 600 launches in a
    row use every counter twice or more, then two streams run launches on
    different inputs at the same time: every result must equal the first one,
    which matches the oracle."""
    B, Hq, Hkv, L = 2, 16, 4, 1300
    ins = [tuple(t.cuda() for t in W.prefill_inputs(B, Hq, Hkv, L, L, D, seed=40 + i)) for i in range(2)]
    scale = 1.0 / math.sqrt(D)
    first = [prefill(*x, scale=scale) for x in ins]
    torch.cuda.synchronize()
    q, k, v = (t.cpu() for t in ins[0])
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, True)
    assert_close(first[0][0], first[0][1], ref_o, ref_l, f"persistent D{D}")
    out = torch.empty_like(ins[0][0])
    for _ in range(600):
        prefill(*ins[0], scale=scale, out=out, want_lse=False)
    torch.cuda.synchronize()
    assert torch.equal(out, first[0][0])
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(x[0]) for x in ins]
    bad = 0
    for _ in range(20):
        for i in range(2):
            with torch.cuda.stream(streams[i]):
                prefill(*ins[i], scale=scale, out=outs[i], want_lse=False, stream=streams[i])
        for i in range(2):
            streams[i].synchronize()
            bad += int(not torch.equal(outs[i], first[i][0]))
    assert bad == 0
    assert device_error(reset=True) == 0


@pytest.mark.parametrize("D,Hq,Hkv,causal", [(128, 12, 4, True), (64, 24, 4, True), (128, 12, 4, False),
                                              (128, 40, 8, True)])
def test_persistent_many_units_ragged_groups(oracle_mod, D, Hq, Hkv, causal):
    """G = 3, 6, 5 (the Q tile has padding rows and its TMA box is G x P rows)
    with several hundred work units, so each persistent CTA runs many units in a
    row through the same Q tiles and staging block; sampled rows across tiles."""
    B, L = 4, 2000
    rows = sorted({0, 1, 41, 42, 43, 83, 84, 85, 127, 128, 255, 256, 1000, 1023, 1024, 1998, 1999})
    _run(oracle_mod, B, Hq, Hkv, L, L, D, causal, seed=Hq + D, spike=97, rows=rows)


@pytest.mark.slow
@pytest.mark.parametrize("shape", [W.QWEN_PREFILL_4K, W.QWEN_PREFILL_8K_B4, W.CHUNKED_16K, W.CHUNKED_32K],
                         ids=lambda s: s.name)
def test_full_size_every_row(oracle_mod, shape):
    """The full-size workloads in the launch configuration the benchmark times,
    every output element against the oracle.  These are the sizes at which the
    persistent scheduler runs its banded unit order (B4 L8192: bands of 3 KV
    groups and a last band of 2; the chunked shapes: bands of 1), so every unit
    of every band is checked.  The oracle runs per sequence to bound host memory."""
    q, k, v = W.prefill_inputs_for(shape, seed=0)
    out, lse = prefill(q.cuda(), k.cuda(), v.cuda(), scale=shape.scale, is_causal=shape.is_causal)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    out, lse = out.cpu(), lse.cpu()
    for b in range(shape.B):
        ref_o, ref_l = oracle_mod.attention_prefill(q[b:b + 1], k[b:b + 1], v[b:b + 1], shape.scale, shape.is_causal)
        assert_close(out[b:b + 1], lse[b:b + 1], ref_o, ref_l, f"{shape.name} b{b}")
        del ref_o, ref_l


@pytest.mark.parametrize("D,Lq,Lk,causal", [(128, 2048, 4096, True), (64, 2048, 3000, True), (128, 2048, 1500, False)])
def test_key_split_tail(oracle_mod, D, Lq, Lk, causal):
    """256 near-equal work units on 148 SMs: the 108 units of the part-filled second
    wave are cut into 4 runs of key tiles, written as fp32 partials and merged.  Every
    element against the oracle, and against the unsplit launch within rounding."""
    B, Hq, Hkv = 1, 32, 8
    need = prefill_workspace_size(B, Hq, Hkv, Lq, Lk, D, causal)
    assert need > 0, "the key split should apply to this launch"
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=Lq + Lk + D, spike_every=97)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    scale = 1.0 / math.sqrt(D)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out, lse = prefill(qd, kd, vd, scale=scale, is_causal=causal, workspace=ws)
    plain_o, plain_l = prefill(qd, kd, vd, scale=scale, is_causal=causal, split=False)
    torch.cuda.synchronize()
    assert device_error(reset=True) == 0
    ref_o, ref_l = oracle_mod.attention_prefill(q, k, v, scale, causal)
    assert_close(out, lse, ref_o, ref_l, f"key split D{D} Lq{Lq} Lk{Lk} causal{causal}")
    assert (out.float() - plain_o.float()).abs().max().item() <= 2e-2
    assert (lse - plain_l).abs().max().item() <= 1e-3
