"""Pins for the fp64 oracle: values the pages print, closed forms, brute force.

Each test ties the oracle to something other than itself, so that a dropped
term, a wrong sign, a wrong index or a transposed operand in ``attn_oracle.c``
fails at least one of them:

* the printed weights of the numpy mask demonstration on the SDPA /
  FlashAttention selection guide (section on the is_causal alignment trap),
  stored in ``tests/golden/mask_alignment_demo.txt``;
* closed forms: weights sum to 1, constant V, causal row 0, two keys, a
  dominant key, scale folding, key permutation;
* structure the pages state: a group of G query heads reads one KV head (GQA
  equals MHA with K/V repeated); decode is the last row of a causal prefill;
  chunked prefill is the tail of a full causal prefill;
* LSE against scipy's logsumexp, and the whole result against an independent
  numpy brute force on tiny shapes.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mask_alignment_demo.txt")


def _read_golden():
    rows = []
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            rows.append((int(parts[0]), parts[1], np.array([float(x) for x in parts[2:7]]),
                         parts[7] == "True"))
    return rows


def _page_demo_inputs():
    # The demonstration's inputs, drawn as it describes them.
    rng = np.random.default_rng(1)
    S, d = 5, 8
    q_all, k, v = (rng.standard_normal((S, d)) for _ in range(3))
    return q_all, k, v, S, d


def _bhld(x):
    return np.ascontiguousarray(x[None, None])


def test_page_mask_demo_weights(oracle_mod):
    """Bottom-right and upper-left weights of the last query row, as printed."""
    q_all, k, v, S, d = _page_demo_inputs()
    scale = 1.0 / math.sqrt(d)
    full, _ = oracle_mod.attention_prefill(_bhld(q_all), _bhld(k), _bhld(v), scale, True)
    golden = _read_golden()
    assert len(golden) == 4
    for L, align, w_printed, matches in golden:
        q = q_all[-L:]
        if align == "bottom-right":
            out, _, w = oracle_mod.attention_prefill(_bhld(q), _bhld(k), _bhld(v), scale, True,
                                                     want_probs=True)
            w_last = w[0, 0, -1]
        else:
            # upper-left keeps j <= i, i.e. the causal result over the first L keys only
            out, _, w = oracle_mod.attention_prefill(_bhld(q), _bhld(k[:L]), _bhld(v[:L]), scale,
                                                     True, want_probs=True)
            w_last = np.concatenate([w[0, 0, -1], np.zeros(S - L)])
        assert np.array_equal(np.round(w_last, 2), w_printed), (L, align, w_last)
        assert np.allclose(out[0, 0], full[0, 0, -L:]) == matches, (L, align)


def test_square_alignments_agree(oracle_mod):
    """For Lq == Lk both alignments keep the lower triangle (the demo's full run)."""
    q_all, k, v, S, d = _page_demo_inputs()
    _, _, w = oracle_mod.attention_prefill(_bhld(q_all), _bhld(k), _bhld(v), 1 / math.sqrt(d),
                                           True, want_probs=True)
    w = w[0, 0]
    assert np.all(w[np.triu_indices(S, 1)] == 0.0)
    assert np.all(w[np.tril_indices(S)] > 0.0)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_weights_sum_to_one_and_log_weights(oracle_mod):
    q, k, v = _rand((2, 6, 7, 16), 1), _rand((2, 3, 11, 16), 2), _rand((2, 3, 11, 16), 3)
    scale = 0.3
    for causal in (False, True):
        out, lse, w = oracle_mod.attention_prefill(q, k, v, scale, causal, want_probs=True)
        assert np.allclose(w.sum(-1), 1.0, atol=1e-13)
        # log w_ij = s_ij - LSE_i on visible cells, with s recomputed here
        kk = np.repeat(k, 2, axis=1)
        s = np.einsum("bhid,bhjd->bhij", q, kk) * scale
        vis = w > 0
        assert np.allclose(np.log(w[vis]), (s - lse[..., None])[vis], atol=1e-12)
        if causal:  # masked cells are exactly the upper triangle shifted by Lk - Lq = 4
            keep = np.tril(np.ones((7, 11), bool), k=4)
            assert np.array_equal(vis[0, 0], keep)


def test_constant_v_returns_v(oracle_mod):
    q, k = _rand((1, 4, 9, 8), 4), _rand((1, 2, 13, 8), 5)
    row = _rand((8,), 6)
    v = np.broadcast_to(row, (1, 2, 13, 8)).copy()
    for causal in (False, True):
        out, _ = oracle_mod.attention_prefill(q, k, v, 0.7, causal)
        assert np.allclose(out, row, atol=1e-13)


def test_causal_row0_is_v0(oracle_mod):
    """With Lq == Lk, causal row 0 sees key 0 only: O = v_0, LSE = scale * q_0 . k_0."""
    q, k, v = _rand((1, 2, 6, 8), 7), _rand((1, 2, 6, 8), 8), _rand((1, 2, 6, 8), 9)
    out, lse = oracle_mod.attention_prefill(q, k, v, 0.25, True)
    for h in range(2):
        assert np.array_equal(out[0, h, 0], v[0, h, 0])
        assert lse[0, h, 0] == pytest.approx(0.25 * float(np.dot(q[0, h, 0], k[0, h, 0])), abs=1e-14)


def test_two_keys_closed_form(oracle_mod):
    """Row 1 of a causal square problem: O = v0 + sigmoid(s1 - s0) (v1 - v0)."""
    q, k, v = _rand((1, 1, 4, 8), 10), _rand((1, 1, 4, 8), 11), _rand((1, 1, 4, 8), 12)
    scale = 0.4
    out, lse = oracle_mod.attention_prefill(q, k, v, scale, True)
    s0 = scale * float(np.dot(q[0, 0, 1], k[0, 0, 0]))
    s1 = scale * float(np.dot(q[0, 0, 1], k[0, 0, 1]))
    sig = 1.0 / (1.0 + math.exp(-(s1 - s0)))
    assert np.allclose(out[0, 0, 1], v[0, 0, 0] + sig * (v[0, 0, 1] - v[0, 0, 0]), atol=1e-14)
    assert lse[0, 0, 1] == pytest.approx(max(s0, s1) + math.log1p(math.exp(-abs(s1 - s0))), abs=1e-14)


def test_dominant_key_is_stable(oracle_mod):
    """Scores near 1e3 must not overflow; with gaps of 100 the output is the top key's value."""
    D = 8
    q = np.zeros((1, 1, 1, D)); q[0, 0, 0, 0] = 1.0
    k = np.zeros((1, 1, 5, D)); k[0, 0, :, 0] = [1000.0, 900.0, 1200.0, 1100.0, 0.0]
    v = _rand((1, 1, 5, D), 13)
    out, lse = oracle_mod.attention_prefill(q, k, v, 1.0, False)
    assert np.all(np.isfinite(out))
    assert np.allclose(out[0, 0, 0], v[0, 0, 2], atol=1e-12)
    assert lse[0, 0, 0] == pytest.approx(1200.0, abs=1e-12)


def test_scale_folds_into_q(oracle_mod):
    q, k, v = _rand((1, 2, 5, 8), 14), _rand((1, 1, 5, 8), 15), _rand((1, 1, 5, 8), 16)
    a, la = oracle_mod.attention_prefill(q, k, v, 0.5, True)
    b, lb = oracle_mod.attention_prefill(q * 0.5, k, v, 1.0, True)
    assert np.allclose(a, b, atol=1e-14) and np.allclose(la, lb, atol=1e-14)


def test_key_permutation_invariance(oracle_mod):
    q, k, v = _rand((1, 2, 3, 8), 17), _rand((1, 1, 9, 8), 18), _rand((1, 1, 9, 8), 19)
    perm = np.random.default_rng(20).permutation(9)
    a, la = oracle_mod.attention_prefill(q, k, v, 0.3, False)
    b, lb = oracle_mod.attention_prefill(q, k[:, :, perm], v[:, :, perm], 0.3, False)
    assert np.allclose(a, b, atol=1e-13) and np.allclose(la, lb, atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv(oracle_mod):
    """Query head h reads KV head h // G: same as MHA on K/V repeated G times per head."""
    G = 3
    q, k, v = _rand((2, 6, 5, 8), 21), _rand((2, 2, 7, 8), 22), _rand((2, 2, 7, 8), 23)
    for causal in (False, True):
        a, la = oracle_mod.attention_prefill(q, k, v, 0.35, causal)
        b, lb = oracle_mod.attention_prefill(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1),
                                             0.35, causal)
        assert np.array_equal(a, b) and np.array_equal(la, lb)
        # and not the interleaved mapping h % Hkv
        c, _ = oracle_mod.attention_prefill(q, np.tile(k, (1, G, 1, 1)), np.tile(v, (1, G, 1, 1)),
                                            0.35, causal)
        assert not np.allclose(a, c)


def test_g1_is_per_head_mha(oracle_mod):
    q, k, v = _rand((1, 3, 4, 8), 24), _rand((1, 3, 6, 8), 25), _rand((1, 3, 6, 8), 26)
    a, la = oracle_mod.attention_prefill(q, k, v, 0.3, True)
    for h in range(3):
        b, lb = oracle_mod.attention_prefill(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], 0.3, True)
        assert np.array_equal(a[:, h], b[:, 0]) and np.array_equal(la[:, h], lb[:, 0])


def test_chunked_prefill_is_tail_of_full(oracle_mod):
    """Lq < Lk with bottom-right alignment equals the last Lq rows of the full causal run."""
    q, k, v = _rand((1, 4, 12, 8), 27), _rand((1, 2, 12, 8), 28), _rand((1, 2, 12, 8), 29)
    full, lf = oracle_mod.attention_prefill(q, k, v, 0.3, True)
    for Lq in (1, 2, 5, 12):
        part, lp = oracle_mod.attention_prefill(q[:, :, -Lq:], k, v, 0.3, True)
        assert np.allclose(part, full[:, :, -Lq:], atol=1e-14)
        assert np.allclose(lp, lf[:, :, -Lq:], atol=1e-14)


def test_row_subset_matches_full(oracle_mod):
    q, k, v = _rand((2, 4, 10, 8), 30), _rand((2, 2, 14, 8), 31), _rand((2, 2, 14, 8), 32)
    full, lf = oracle_mod.attention_prefill(q, k, v, 0.3, True)
    rows = [9, 0, 4, 4]
    part, lp = oracle_mod.attention_prefill(q, k, v, 0.3, True, rows=rows)
    assert np.array_equal(part, full[:, :, rows]) and np.array_equal(lp, lf[:, :, rows])


def test_rows_without_visible_keys(oracle_mod):
    """Lq > Lk causal: rows i < Lq - Lk see nothing -> O = 0, LSE = -inf; Lk = 0 likewise."""
    q, k, v = _rand((1, 2, 6, 8), 33), _rand((1, 1, 4, 8), 34), _rand((1, 1, 4, 8), 35)
    out, lse = oracle_mod.attention_prefill(q, k, v, 0.3, True)
    assert np.all(out[:, :, :2] == 0.0) and np.all(np.isneginf(lse[:, :, :2]))
    assert np.all(np.isfinite(lse[:, :, 2:]))
    # row 2 sees key 0 only
    assert np.array_equal(out[0, 0, 2], v[0, 0, 0])
    e = np.zeros((1, 1, 0, 8))
    out0, lse0 = oracle_mod.attention_prefill(q, e, e, 0.3, False)
    assert np.all(out0 == 0.0) and np.all(np.isneginf(lse0))


def test_lse_matches_scipy_logsumexp(oracle_mod):
    q, k, v = _rand((1, 4, 6, 16), 36), _rand((1, 2, 9, 16), 37), _rand((1, 2, 9, 16), 38)
    _, lse = oracle_mod.attention_prefill(q, k, v, 0.2, True)
    s = np.einsum("bhid,bhjd->bhij", q, np.repeat(k, 2, axis=1)) * 0.2
    keep = np.tril(np.ones((6, 9), bool), k=3)
    ref = logsumexp(np.where(keep, s, -np.inf), axis=-1)
    assert np.allclose(lse, ref, atol=1e-13)


def _numpy_brute_force(q, k, v, scale, causal):
    """Independent numpy attention in the style of the page's demonstration."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    kk, vv = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    s = (q @ np.swapaxes(kk, -1, -2)) * scale
    if causal:
        s = np.where(np.tril(np.ones((Lq, Lk), bool), k=Lk - Lq), s, -np.inf)
    w = np.exp(s - s.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    return w @ vv, logsumexp(s, axis=-1)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny_shapes(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    Hkv = int(rng.integers(1, 4))
    G = int(rng.integers(1, 5))
    B, D = int(rng.integers(1, 3)), int(rng.choice([4, 8, 16]))
    Lk = int(rng.integers(1, 40))
    Lq = int(rng.integers(1, Lk + 1))
    q = rng.standard_normal((B, Hkv * G, Lq, D))
    k = rng.standard_normal((B, Hkv, Lk, D))
    v = rng.standard_normal((B, Hkv, Lk, D))
    for causal in (False, True):
        a, la = oracle_mod.attention_prefill(q, k, v, 1 / math.sqrt(D), causal)
        b, lb = _numpy_brute_force(q, k, v, 1 / math.sqrt(D), causal)
        assert np.allclose(a, b, atol=1e-12) and np.allclose(la, lb, atol=1e-12)


def test_decode_is_last_row_of_causal_prefill(oracle_mod):
    """One new token against the cache = the last row of a causal prefill of that length."""
    B, Hq, Hkv, Lmax, D = 3, 4, 2, 10, 8
    q = _rand((B, Hq, D), 40)
    kc, vc = _rand((B, Hkv, Lmax, D), 41), _rand((B, Hkv, Lmax, D), 42)
    seqlens = np.array([10, 1, 6], dtype=np.int32)
    out, lse = oracle_mod.attention_decode(q, kc, vc, seqlens, 0.3)
    for b in range(B):
        n = int(seqlens[b])
        qp = np.zeros((1, Hq, n, D)); qp[0, :, -1] = q[b]
        ref, lref = oracle_mod.attention_prefill(qp, kc[b:b + 1, :, :n], vc[b:b + 1, :, :n], 0.3, True)
        assert np.allclose(out[b], ref[0, :, -1], atol=1e-14)
        assert np.allclose(lse[b], lref[0, :, -1], atol=1e-14)


def test_decode_ignores_rows_beyond_seqlen(oracle_mod):
    B, Hq, Hkv, Lmax, D = 2, 2, 1, 9, 8
    q = _rand((B, Hq, D), 43)
    kc, vc = _rand((B, Hkv, Lmax, D), 44), _rand((B, Hkv, Lmax, D), 45)
    seqlens = np.array([4, 0], dtype=np.int32)
    a, la = oracle_mod.attention_decode(q, kc, vc, seqlens, 0.3)
    kn, vn = kc.copy(), vc.copy()
    kn[0, :, 4:] = np.nan; vn[0, :, 4:] = np.nan; kn[1] = np.nan; vn[1] = np.nan
    b, lb = oracle_mod.attention_decode(q, kn, vn, seqlens, 0.3)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    assert np.all(b[1] == 0.0) and np.all(np.isneginf(lb[1]))


def test_bf16_bits_widen_exactly(oracle_mod):
    """bf16 inputs are read as the exact values they hold (compared with torch's widening)."""
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 2, 5, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, 7, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 1, 7, 8, generator=g).to(torch.bfloat16)
    a, la = oracle_mod.attention_prefill(q, k, v, 0.3, True)
    b, lb = oracle_mod.attention_prefill(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                         0.3, True)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
    c, lc = oracle_mod.attention_prefill(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                         0.3, True)
    assert np.array_equal(a, c) and np.array_equal(la, lc)


# ---------------------------------------------------------------------------
# 8-bit caches: the element decoders against library routines and closed
# forms, the scale indexing against a structured input, and the attention
# against the pinned bf16 oracle on inputs both can represent.
# ---------------------------------------------------------------------------
def test_e4m3_values_match_torch_for_all_codes(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ours = np.array([oracle_mod.e4m3_value(c) for c in codes])
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    assert np.array_equal(ours[~np.isnan(ours)], lib[~np.isnan(lib)])
    assert np.isnan(ours).sum() == 2          # S.1111.111 only: no infinities
    # closed forms from the format definition
    assert oracle_mod.e4m3_value(0x38) == 1.0
    assert oracle_mod.e4m3_value(0x7E) == 448.0 and oracle_mod.e4m3_value(0xFE) == -448.0
    assert oracle_mod.e4m3_value(0x01) == 2.0 ** -9 and oracle_mod.e4m3_value(0x08) == 2.0 ** -6
    assert oracle_mod.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert math.copysign(1.0, oracle_mod.e4m3_value(0x80)) == -1.0 and oracle_mod.e4m3_value(0x80) == 0.0


def test_f16_values_match_numpy_for_all_patterns(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = np.array([oracle_mod.f16_value(b) for b in bits[::7]] + [oracle_mod.f16_value(b) for b in
                                                                      (0x0001, 0x03FF, 0x0400, 0x7BFF, 0x7C00)])
    lib = np.concatenate([bits[::7], np.array([0x0001, 0x03FF, 0x0400, 0x7BFF, 0x7C00], np.uint16)])
    lib = lib.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], lib[ok])
    assert oracle_mod.f16_value(0x0001) == 2.0 ** -24 and oracle_mod.f16_value(0x7BFF) == 65504.0


def test_q8_0_scale_indexing(oracle_mod):
    """Each scale is a distinct integer naming (b, g, r, block) (exact in fp16); code 1
    everywhere shows which scale every element used, and code -3 checks the int8 sign."""
    B, Hkv, L, D = 2, 3, 5, 64
    name = np.zeros((B, Hkv, L, D // 32), dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            for r in range(L):
                for c in range(D // 32):
                    name[b, g, r, c] = 1 + ((b * Hkv + g) * L + r) * 2 + c
    scales = name.astype(np.float16)
    codes = np.ones((B, Hkv, L, D), dtype=np.uint8)
    codes[..., 5] = np.uint8(256 - 3)
    out = oracle_mod.dequantize_kv8(codes, oracle_mod.KV_Q8_0, scales)
    for d in (0, 5, 31, 32, 63):
        want = name[..., d // 32].astype(np.float64) * (-3 if d == 5 else 1)
        assert np.array_equal(out[..., d], want), d


def test_e4m3_per_head_scale(oracle_mod):
    codes = np.full((2, 3, 4, 32), 0x38, dtype=np.uint8)     # value 1.0
    scales = np.array([0.5, 2.0, -4.0], dtype=np.float32)
    out = oracle_mod.dequantize_kv8(codes, oracle_mod.KV_E4M3, scales)
    for g in range(3):
        assert np.all(out[:, g] == scales[g])


def test_kv8_attention_equals_bf16_oracle_on_shared_values(oracle_mod):
    """Unit scales and codes whose values are exact in bf16: the 8-bit oracle must
    equal the pinned bf16 decode oracle (last row of a causal prefill) on the same values."""
    rng = np.random.default_rng(4)
    B, Hq, Hkv, L, D = 2, 4, 2, 40, 64
    q = torch.randn(B, Hq, 1, D, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    seqlens = np.array([40, 17])
    for fmt in (oracle_mod.KV_E4M3, oracle_mod.KV_Q8_0):
        if fmt == oracle_mod.KV_E4M3:
            pool = np.array([c for c in range(256) if abs(oracle_mod.e4m3_value(c)) <= 4.0], dtype=np.uint8)
            kc = rng.choice(pool, size=(B, Hkv, L, D)).astype(np.uint8)
            vc = rng.choice(pool, size=(B, Hkv, L, D)).astype(np.uint8)
            ks = vs = np.ones(Hkv, np.float32)
        else:
            kc = rng.integers(-4, 5, size=(B, Hkv, L, D)).astype(np.int8).view(np.uint8)
            vc = rng.integers(-4, 5, size=(B, Hkv, L, D)).astype(np.int8).view(np.uint8)
            ks = vs = np.ones((B, Hkv, L, D // 32), np.float16)
        o8, l8 = oracle_mod.attention_decode_kv8(q, kc, vc, fmt, ks, vs, seqlens, 0.125)
        kf = torch.from_numpy(oracle_mod.dequantize_kv8(kc, fmt, ks)).to(torch.bfloat16)
        vf = torch.from_numpy(oracle_mod.dequantize_kv8(vc, fmt, vs)).to(torch.bfloat16)
        assert torch.equal(kf.double(), torch.from_numpy(oracle_mod.dequantize_kv8(kc, fmt, ks)))  # exact in bf16
        ob, lb = oracle_mod.attention_decode(q[:, :, 0], kf, vf, seqlens.astype(np.int32), 0.125)
        assert np.allclose(o8[:, :, 0], ob, rtol=0, atol=1e-12) and np.allclose(l8[:, :, 0], lb, rtol=0, atol=1e-12)
