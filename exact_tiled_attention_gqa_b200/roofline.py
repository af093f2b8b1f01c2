"""Algorithmic work and roofline denominators for the two calls.

Only counting, no attention arithmetic: how many multiply-adds the exact
result needs (masked pairs are never credited) and how many bytes a decode
step must read at least.

Prefill FLOPs = 4 * D * (visible query/key pairs) * B * Hq -- two GEMM-shaped
products (Q K^T and P V) of 2 * D flops per visible pair, the count the SDPA /
FlashAttention selection guide uses for its per-token attention cost ("share
of attention compute in long inputs": 4 x query heads x head dim x t per layer).

Decode bytes = every valid K and V cache row once (2 * D * 2 bytes per row per
KV head) plus q, out and lse.  Split-KV partials are overhead and not credited.
"""
from __future__ import annotations

import glob
import hashlib
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def visible_pairs(Lq: int, Lk: int, is_causal: bool) -> int:
    """Number of (i, j) with j visible from row i under the bottom-right causal mask."""
    if not is_causal:
        return Lq * Lk
    off = Lk - Lq
    total = 0
    # row i sees min(Lk, max(0, i + off + 1)) keys; sum in closed form over the three ranges
    lo = max(0, -off)               # first row with >= 1 key
    hi = min(Lq, Lk - off)          # rows < hi see fewer than Lk keys
    if hi > lo:
        a, b = lo + off + 1, hi - 1 + off + 1
        total += (a + b) * (hi - lo) // 2
    if Lq > max(hi, lo):
        total += (Lq - max(hi, lo)) * Lk
    return total


def prefill_flops(B: int, Hq: int, Lq: int, Lk: int, D: int, is_causal: bool) -> int:
    return 4 * D * visible_pairs(Lq, Lk, is_causal) * B * Hq


def decode_bytes(seqlens, B: int, Hq: int, Hkv: int, D: int) -> int:
    kv = sum(int(s) for s in seqlens) * Hkv * D * 2 * 2
    return kv + B * Hq * D * 2 * 2 + B * Hq * 4


def decode_kv8_bytes(seqlens, B: int, Hq: int, Hkv: int, D: int, q8_0: bool, Lq: int = 1) -> int:
    """Algorithmic bytes of an 8-bit-cache decode: every valid K and V row once
    (one byte per element, plus one fp16 scale per 32 values for q8_0), q, out, lse."""
    per_row = D + (D // 32) * 2 if q8_0 else D
    kv = sum(int(s) for s in seqlens) * Hkv * per_row * 2
    return kv + B * Hq * Lq * (D * 2 * 2 + 4)


def measured_peaks() -> dict:
    """MEASURED_PEAKS.json if present, else the pool's earlier measurement."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash() -> str:
    """Hash of the CUDA sources; a DRAM-traffic figure is only valid for the hash it was taken at."""
    h = hashlib.sha256()
    for path in sorted(glob.glob(os.path.join(ROOT, "exact_tiled_attention_gqa_b200", "csrc", "*"))):
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic() -> dict:
    """Per-launch DRAM bytes from profiles/traffic.json, only if taken at the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return {}
    return d.get("bytes_per_launch", {})
