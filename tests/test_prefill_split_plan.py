"""The key-split plan of attn_prefill_ws, on the host (no GPU).

A persistent prefill launch (head dim 64 / 128) hands its work units (batch b,
KV head g, 2 x P query positions with P = 128 / G) to one CTA per SM.  When the
unit count U lies strictly between one and four waves and is not a whole number
of waves, and the last U mod n_sm units of the launch order each see at least 8
key tiles, those units are cut into 4 runs of key tiles.  The workspace then
holds, per cut unit, 4 x 256 rows of fp32 O (D floats each) and one fp32
log2-sum-exp per row, each array rounded up to 256 bytes.  The expected values
below are worked out from that rule by hand, not by the library.
"""
import ctypes

import pytest

from exact_tiled_attention_gqa_b200 import _native


def _align256(n):
    return (n + 255) // 256 * 256


def _plan(B, Hq, Hkv, Lq, Lk, D, causal, n_sm):
    n_full, n_items = ctypes.c_int(-7), ctypes.c_int(-7)
    size = _native.lib().attn_prefill_split_plan(B, Hq, Hkv, Lq, Lk, D, int(causal), n_sm, ctypes.byref(n_full),
                                                 ctypes.byref(n_items))
    return int(size), n_full.value, n_items.value


def _bytes(cut_units, D):
    rows = cut_units * 4 * 2 * 128
    return _align256(rows * D * 4) + _align256(rows * 4)


@pytest.mark.parametrize("Lk", [16384, 32768])
def test_chunked_prefill_cuts_its_last_wave(Lk):
    # 2048 rows x 8 KV heads in blocks of 64 positions (G = 4, P = 32): 256 units,
    # every one seeing at least 14336 keys; 256 - 148 = 108 units cut
    assert _plan(1, 32, 8, 2048, Lk, 128, True, 148) == (_bytes(108, 128), 148, 148 + 4 * 108)


def test_head_dim_64_and_a_smaller_sm_count():
    # Lk - Lq = 952: the earliest block's last row sees 952 + 64 keys = 8 tiles
    assert _plan(1, 32, 8, 2048, 3000, 64, True, 148) == (_bytes(108, 64), 148, 580)
    # 256 units on 100 SMs: 2 whole waves, 56 units cut
    assert _plan(1, 32, 8, 2048, 16384, 128, True, 100) == (_bytes(56, 128), 200, 200 + 4 * 56)


def test_no_cut_when_the_waves_are_full_or_many():
    assert _plan(1, 32, 8, 2048, 16384, 128, True, 256) == (0, 256, 256)   # one wave
    assert _plan(1, 32, 8, 2048, 16384, 128, True, 128) == (0, 256, 256)   # two whole waves
    # Qwen3-8B B4 L8192: 4 x 8 x 128 = 4096 units, more than 4 waves
    assert _plan(4, 32, 8, 8192, 8192, 128, True, 148) == (0, 4096, 4096)


def test_no_cut_when_the_last_units_are_short():
    # causal B1 L4096: 512 units, the lightest (1 .. 8 key tiles) handed out last
    assert _plan(1, 32, 8, 4096, 4096, 128, True, 148) == (0, 512, 512)
    # full attention over 896 keys is 7 tiles per unit; 897 keys make 8
    assert _plan(1, 32, 8, 2048, 896, 128, False, 148) == (0, 256, 256)
    assert _plan(1, 32, 8, 2048, 897, 128, False, 148) == (_bytes(108, 128), 148, 580)


def test_head_dim_256_and_invalid_arguments():
    assert _plan(1, 32, 8, 2048, 16384, 256, True, 148) == (0, 0, 0)
    assert _plan(1, 30, 8, 2048, 16384, 128, True, 148) == (0, 0, 0)   # Hq % Hkv != 0
    assert _plan(1, 32, 8, 2048, 16384, 128, True, 0) == (0, 0, 0)
    assert _native.lib().attn_prefill_split_plan(1, 32, 8, 2048, 16384, 128, 1, 148, None, None) == _bytes(108, 128)
