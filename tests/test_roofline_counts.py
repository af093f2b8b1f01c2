"""The work counts used for the roofline, checked against closed forms and the
figures the SDPA / FlashAttention selection guide prints for Qwen3-8B."""

import pytest

from exact_tiled_attention_gqa_b200.roofline import decode_bytes, prefill_flops, visible_pairs


def _brute_pairs(Lq, Lk, causal):
    return sum(1 for i in range(Lq) for j in range(Lk) if (not causal or j <= i + Lk - Lq))


@pytest.mark.parametrize("Lq,Lk", [(1, 1), (5, 5), (3, 7), (7, 3), (128, 128), (100, 1000), (10, 0), (0, 4)])
def test_visible_pairs_brute_force(Lq, Lk):
    for causal in (False, True):
        assert visible_pairs(Lq, Lk, causal) == _brute_pairs(Lq, Lk, causal)


def test_square_causal_is_triangle():
    assert visible_pairs(4096, 4096, True) == 4096 * 4097 // 2


def test_per_token_attention_flops_match_page_table():
    # "share of attention compute": per prefill token, 36 layers x 4 x 32 heads x 128 x (L/2)
    per_layer = lambda L: 4 * 32 * 128 * (L / 2)
    printed = {2048: 0.6, 4096: 1.2, 8192: 2.4, 16384: 4.8, 32768: 9.7}
    for L, gflop in printed.items():
        assert round(36 * per_layer(L) / 1e9, 1) == gflop
    # and our count for one layer, whole prompt, agrees with that per-token mean up to the diagonal
    L = 4096
    assert prefill_flops(1, 32, L, L, 128, True) == pytest.approx(L * per_layer(L), rel=1 / L + 1e-12)


def test_score_table_and_kv_bytes_match_page_table():
    # "eager attention memory": bf16 table + fp32 softmax = 6 bytes per cell, 32 heads, B=1
    for L, gib in {4096: 3, 8192: 12, 16384: 48, 32768: 192}.items():
        assert 32 * L * L * 6 / 2**30 == gib
    # KV cache per token: 36 layers x 8 KV heads x 128 x (K and V) x 2 bytes = 144 KiB
    assert 36 * 8 * 128 * 2 * 2 == 144 * 1024
    assert 36 * 32 * 128 * 2 * 2 == 576 * 1024   # if all 32 heads kept K/V


def test_decode_bytes():
    assert decode_bytes([10, 0, 3], 3, 8, 2, 128) == 13 * 2 * 128 * 4 + 3 * 8 * 128 * 4 + 3 * 8 * 4
