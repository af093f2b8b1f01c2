"""Seeded synthetic inputs and the workload table.

This module only draws random tensors and names shapes: it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed from
it.  Every tensor is drawn as fp32 N(0, 1) from a seeded ``torch.Generator``
and rounded to bf16, which is the precision both sides then read.

Shapes are Qwen3-8B's attention (32 query heads, 8 KV heads, head dim 128, as
the SDPA / FlashAttention selection guide lists them under "eager attention
memory") and the group-size sweep of the NVIDIA attention-optimisation page
("Parameter one: group size").  There are no model weights and no dataset.

Draw order (fixed, so a seed names one input set):
  prefill: q, k, v; then K rows j with j % spike_every == 0 are multiplied by
           spike_scale (exact in bf16 for a power of two).
  decode : seqlens (int32, uniform in [lo, hi]), then q, k_cache, v_cache;
           cache rows at or beyond seqlens[b] are then overwritten with
           ``fill_beyond`` (NaN in tests, to show they are never used).
Large decode caches are drawn on the GPU with a CUDA generator, one
(batch, KV head) slab at a time so the fp32 staging stays small.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    D: int
    is_causal: bool = True
    spike_every: int = 0      # 0 = no spiked keys
    spike_scale: float = 8.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lmax: int
    D: int
    seqlen_lo: int
    seqlen_hi: int

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five workloads, named by what they are.
TINY_PREFILL = PrefillShape("tiny causal GQA prefill B1 Hq4 Hkv1 L128 D64", 1, 4, 1, 128, 128, 64)
QWEN_PREFILL_4K = PrefillShape("Qwen3-8B causal prefill B1 L4096", 1, 32, 8, 4096, 4096, 128)
QWEN_PREFILL_8K_B4 = PrefillShape("Qwen3-8B causal prefill B4 L8192", 4, 32, 8, 8192, 8192, 128)
CHUNKED_16K = PrefillShape("chunked prefill Lq2048 onto Lk16384 (bottom-right)", 1, 32, 8, 2048, 16384,
                           128, True, 97, 8.0)
CHUNKED_32K = PrefillShape("chunked prefill Lq2048 onto Lk32768 (bottom-right)", 1, 32, 8, 2048, 32768,
                           128, True, 97, 8.0)
QWEN_DECODE = DecodeShape("Qwen3-8B decode B64 seqlen U[1024,32768]", 64, 32, 8, 32768, 128, 1024, 32768)
# The Qwen3-8B decode batch with an 8-bit cache (E4M3 with per-KV-head scales, or
# q8_0 int8 codes with an fp16 scale per 32 values).
QWEN_DECODE_E4M3 = DecodeShape("Qwen3-8B decode B64 seqlen U[1024,32768], E4M3 KV cache", 64, 32, 8, 32768, 128,
                               1024, 32768)
QWEN_DECODE_Q8_0 = DecodeShape("Qwen3-8B decode B64 seqlen U[1024,32768], q8_0 KV cache", 64, 32, 8, 32768, 128,
                               1024, 32768)
# Head dim 64: the NVIDIA page ("Parameter two: head dimension") has it paying for a
# 128-wide tile, while the softmax cost does not shrink with D.
HD64_PREFILL = PrefillShape("head-dim-64 causal prefill B4 Hq32 Hkv8 L8192 D64", 4, 32, 8, 8192, 8192, 64)
# Head dim 256, the other width the NVIDIA attention page recommends ("Parameter
# two: head dimension"), at group size 8.
HD256_PREFILL = PrefillShape("head-dim-256 causal prefill B2 Hq16 Hkv2 L8192 D256", 2, 16, 2, 8192, 8192, 256)
HD256_DECODE = DecodeShape("head-dim-256 decode B32 Hq16 Hkv2 seqlen U[1024,32768] D256", 32, 16, 2, 32768, 256,
                           1024, 32768)


def group_sweep_decode(G: int) -> DecodeShape:
    """Decode at Hq=64, D=128, batch 8, 131072 cached keys per sequence, Hkv = 64 / G."""
    if 64 % G:
        raise ValueError("G must divide 64")
    return DecodeShape(f"group sweep decode G{G} B8 L131072", 8, 64, 64 // G, 131072, 128, 131072, 131072)


GROUP_SWEEP = (1, 2, 4, 8, 16, 32, 64)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn_bf16(shape, g: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def prefill_inputs(B: int, Hq: int, Hkv: int, Lq: int, Lk: int, D: int, seed: int = 0,
                   spike_every: int = 0, spike_scale: float = 8.0, device="cpu"):
    """(q [B,Hq,Lq,D], k [B,Hkv,Lk,D], v [B,Hkv,Lk,D]) bf16, i.i.d. N(0,1)."""
    g = _gen(seed, device)
    q = _randn_bf16((B, Hq, Lq, D), g, device)
    k = _randn_bf16((B, Hkv, Lk, D), g, device)
    v = _randn_bf16((B, Hkv, Lk, D), g, device)
    if spike_every:
        k[:, :, ::spike_every, :] *= spike_scale
    return q, k, v


def prefill_inputs_for(shape: PrefillShape, seed: int = 0, device="cpu"):
    return prefill_inputs(shape.B, shape.Hq, shape.Hkv, shape.Lq, shape.Lk, shape.D, seed,
                          shape.spike_every, shape.spike_scale, device)


def decode_inputs(B: int, Hq: int, Hkv: int, Lmax: int, D: int, seqlen_lo: int, seqlen_hi: int,
                  seed: int = 0, device="cpu", fill_beyond: Optional[float] = None):
    """(q [B,Hq,D], k_cache, v_cache [B,Hkv,Lmax,D] bf16, seqlens int32 [B] on ``device``).

    seqlens are drawn on the CPU generator (so they do not depend on the
    device); the tensors on ``device``'s generator.
    """
    gcpu = _gen(seed, "cpu")
    seqlens = torch.randint(seqlen_lo, seqlen_hi + 1, (B,), generator=gcpu, dtype=torch.int64)
    seqlens = seqlens.to(torch.int32)
    g = gcpu if torch.device(device).type == "cpu" else _gen(seed, device)
    q = _randn_bf16((B, Hq, D), g, device)
    k = torch.empty((B, Hkv, Lmax, D), dtype=torch.bfloat16, device=device)
    v = torch.empty((B, Hkv, Lmax, D), dtype=torch.bfloat16, device=device)
    for cache in (k, v):
        for b in range(B):
            for h in range(Hkv):
                cache[b, h].copy_(_randn_bf16((Lmax, D), g, device))
    if fill_beyond is not None:
        for b in range(B):
            n = int(seqlens[b])
            if n < Lmax:
                k[b, :, n:, :] = fill_beyond
                v[b, :, n:, :] = fill_beyond
    return q, k, v, seqlens.to(device)


KV_E4M3, KV_Q8_0 = "e4m3", "q8_0"


def quantize_kv8(x: torch.Tensor, fmt: str, head_scales: Optional[torch.Tensor] = None):
    """Encode a cache slab x [..., L, D] (bf16/fp32) as 8-bit codes.

    e4m3: codes = x / s rounded to the nearest E4M3 value (clamped to +-448),
          with s the given per-slab scale (a 0-d fp32 tensor);
    q8_0: per 32 consecutive values, s = max|x| / 127 rounded to fp16 (1 where the
          block is all zero), codes = round(x / s) clamped to [-127, 127].
    Returns (codes, scales): float8_e4m3fn codes and s as given, or int8 codes and
    fp16 scales [..., L, D/32].  This is input preparation, not attention arithmetic.
    """
    xf = x.float()
    if fmt == KV_E4M3:
        return (xf / head_scales).clamp(-448.0, 448.0).to(torch.float8_e4m3fn), head_scales
    blocks = xf.unflatten(-1, (xf.shape[-1] // 32, 32))
    s = (blocks.abs().amax(-1) / 127.0).to(torch.float16)
    s = torch.where(s == 0, torch.ones_like(s), s)
    codes = torch.round(blocks / s.float().unsqueeze(-1)).clamp(-127, 127).to(torch.int8)
    return codes.flatten(-2), s


def e4m3_head_scales(Hkv: int) -> torch.Tensor:
    """Per-KV-head E4M3 scales: about max|x| / 448 for N(0,1) data, distinct per head."""
    return torch.tensor([6.5 / 448.0 * (1.0 + 0.125 * g) for g in range(Hkv)], dtype=torch.float32)


def decode_inputs_kv8(B: int, Hq: int, Hkv: int, Lmax: int, D: int, seqlen_lo: int, seqlen_hi: int, fmt: str,
                      seed: int = 0, device="cpu", Lq: int = 1, fill_beyond: bool = False):
    """(q [B,Hq,Lq,D] bf16, k_codes, v_codes [B,Hkv,Lmax,D], k_scale, v_scale, seqlens int32 [B]).

    The cache is drawn as N(0,1) one (b, KV head) slab at a time and encoded by
    quantize_kv8; seqlens are drawn first on the CPU generator.  With fill_beyond,
    rows at or past seqlens[b] get NaN codes (E4M3 0x7F) or code -128 with NaN
    scales (Q8_0), to show they are never used.
    """
    gcpu = _gen(seed, "cpu")
    seqlens = torch.randint(seqlen_lo, seqlen_hi + 1, (B,), generator=gcpu, dtype=torch.int64).to(torch.int32)
    g = gcpu if torch.device(device).type == "cpu" else _gen(seed, device)
    q = _randn_bf16((B, Hq, Lq, D), g, device)
    cdt = torch.float8_e4m3fn if fmt == KV_E4M3 else torch.int8
    k = torch.empty((B, Hkv, Lmax, D), dtype=cdt, device=device)
    v = torch.empty((B, Hkv, Lmax, D), dtype=cdt, device=device)
    if fmt == KV_E4M3:
        ks = e4m3_head_scales(Hkv).to(device)
        vs = (e4m3_head_scales(Hkv) * 0.75).to(device)
    else:
        ks = torch.empty((B, Hkv, Lmax, D // 32), dtype=torch.float16, device=device)
        vs = torch.empty((B, Hkv, Lmax, D // 32), dtype=torch.float16, device=device)
    for cache, sc in ((k, ks), (v, vs)):
        for b in range(B):
            for h in range(Hkv):
                x = _randn_bf16((Lmax, D), g, device)
                if fmt == KV_E4M3:
                    cache[b, h].copy_(quantize_kv8(x, fmt, sc[h])[0])
                else:
                    c, s = quantize_kv8(x, fmt)
                    cache[b, h].copy_(c)
                    sc[b, h].copy_(s)
    if fill_beyond:
        for b in range(B):
            n = int(seqlens[b])
            if n < Lmax:
                if fmt == KV_E4M3:
                    k[b, :, n:].view(torch.uint8).fill_(0x7F)
                    v[b, :, n:].view(torch.uint8).fill_(0x7F)
                else:
                    k[b, :, n:] = -128
                    v[b, :, n:] = -128
                    ks[b, :, n:] = float("nan")
                    vs[b, :, n:] = float("nan")
    return q, k, v, ks, vs, seqlens.to(device)


def decode_inputs_for(shape: DecodeShape, seed: int = 0, device="cpu", fill_beyond=None):
    return decode_inputs(shape.B, shape.Hq, shape.Hkv, shape.Lmax, shape.D, shape.seqlen_lo,
                         shape.seqlen_hi, seed, device, fill_beyond)
