"""Parity cases run against the bounds-checking build of the library.

Run as a script in a process whose environment has ATTN_GQA_DEBUG_BOUNDS=1, so
the package loads libattn_gqa_sm100_debug_bounds.so (the same sources built with
-DATTN_DEBUG_BOUNDS=1).  In that build every kernel checks, where it turns work
units, ring positions and tile indices into addresses, that the result lies in
its tensor, and sets ATTN_DEVERR_BOUNDS otherwise.  Each case must match the
oracle and leave the device error word at zero.  Exits 0 when all pass.
"""
import math
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import exact_tiled_attention_gqa_b200 as attn  # noqa: E402
from exact_tiled_attention_gqa_b200 import _native  # noqa: E402
from exact_tiled_attention_gqa_b200 import workloads as W  # noqa: E402
from parity import assert_close  # noqa: E402

import oracle  # noqa: E402


def check_error(what):
    err = attn.device_error(reset=True)
    assert err == 0, f"{what}: device error word {err:#x}"


def prefill_case(B, Hq, Hkv, Lq, Lk, D, causal, seed, spike=0):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=seed, spike_every=spike)
    out, lse = attn.prefill(q.cuda(), k.cuda(), v.cuda(), scale=1 / math.sqrt(D), is_causal=causal)
    torch.cuda.synchronize()
    what = f"prefill B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} Lk{Lk} D{D} causal{causal}"
    check_error(what)
    ref_o, ref_l = oracle.attention_prefill(q, k, v, 1 / math.sqrt(D), causal)
    assert_close(out, lse, ref_o, ref_l, what)


def decode_case(B, Hq, Hkv, Lmax, D, seqlens, seed, Lq=1):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Lq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    out, lse = attn.decode_mq(q.cuda(), k.cuda(), v.cuda(), sl.cuda(), scale=1 / math.sqrt(D))
    torch.cuda.synchronize()
    what = f"decode B{B} Hq{Hq} Hkv{Hkv} Lq{Lq} Lmax{Lmax} D{D}"
    check_error(what)
    ro, rl = [], []
    for b in range(B):
        n = seqlens[b]
        o, l = oracle.attention_prefill(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], 1 / math.sqrt(D), True)
        ro.append(o)
        rl.append(l)
    import numpy as np
    assert_close(out, lse, np.concatenate(ro), np.concatenate(rl), what)


def kv8_case(fmt):
    B, Hq, Hkv, Lmax, D = 3, 16, 2, 700, 128
    q, k, v, ks, vs, sl = W.decode_inputs_kv8(B, Hq, Hkv, Lmax, D, 1, Lmax, fmt, seed=5, fill_beyond=True)
    out, lse = attn.decode_kv8(q.cuda(), k.cuda(), v.cuda(), ks.cuda(), vs.cuda(), sl.cuda(), scale=1 / math.sqrt(D))
    torch.cuda.synchronize()
    check_error(f"decode_kv8 {fmt}")
    ofmt = oracle.KV_E4M3 if fmt == W.KV_E4M3 else oracle.KV_Q8_0
    ro, rl = oracle.attention_decode_kv8(q, k, v, ofmt, ks, vs, sl, 1 / math.sqrt(D))
    assert_close(out, lse, ro, rl, f"decode_kv8 {fmt}")


def main():
    assert _native.LIB_PATH.endswith("_debug_bounds.so"), _native.LIB_PATH
    attn.device_error(reset=True)
    for D in (64, 128, 256):
        for Hq, Hkv in ((4, 4), (16, 4), (12, 2)):
            prefill_case(2, Hq, Hkv, 300, 300, D, True, seed=D + Hq)
        prefill_case(1, 8, 2, 77, 500, D, True, seed=D, spike=97)
        prefill_case(1, 8, 2, 300, 300, D, False, seed=D + 1)
    # the persistent scheduler's banded unit order: K/V of all groups above half
    # the L2, so units run in bands (1 group per band at Lk 16384, 3 per band
    # with a partial last band at Lk 10000 over 16 groups)
    prefill_case(1, 32, 8, 256, 16384, 128, True, seed=3, spike=97)
    prefill_case(2, 32, 8, 300, 10000, 128, True, seed=4)
    prefill_case(2, 32, 8, 300, 10000, 64, True, seed=5)
    # the key-split tail: 256 near-equal units, the last 108 cut into key runs
    for D, Lk in ((128, 4096), (64, 3000)):
        assert attn.prefill_workspace_size(1, 32, 8, 2048, Lk, D, True) > 0
        prefill_case(1, 32, 8, 2048, Lk, D, True, seed=6 + D)
    for G, D in ((4, 128), (16, 64), (32, 128), (64, 128), (4, 256)):
        decode_case(3, 2 * G, 2, 5000, D, [5000, 1, 2500], seed=G + D)
    decode_case(2, 8, 2, 900, 128, [900, 3], seed=9, Lq=4)
    kv8_case(W.KV_E4M3)
    kv8_case(W.KV_Q8_0)
    print("debug-bounds cases passed")


if __name__ == "__main__":
    main()
