"""fp64 eager attention oracle (CPU).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library and
its Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it, marshals numpy arrays into it and shapes the
results.  What it computes is stated in the header of ``attn_oracle.c``:
softmax(scale * Q K^T + mask) V with grouped-query heads (query head h reads
KV head h // G), the bottom-right causal mask of the causal-alignment section
of the SDPA / FlashAttention selection guide, and the natural-log LSE.

For an 8-bit KV cache (``attention_decode_kv8``) the codes are first turned
into fp64 element values by ``dequantize_kv8`` (FP8 E4M3 with one scale per KV
head, or q8_0 int8 codes with an fp16 scale per 32 values; the decoders are in
``attn_oracle.c``), and the same eager attention runs on them.

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
the pages print (the numpy mask demonstration), against closed forms, and (the
8-bit decoders) against torch's and numpy's own decoders.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libattn_oracle.so")

F64, F32, BF16 = 0, 1, 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into libattn_oracle.so next to it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           "-Wall", "-Wextra", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            vp, i32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
            lib.oracle_attn_prefill.restype = i32
            lib.oracle_attn_prefill.argtypes = [
                vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f64, i32,
                vp, i32, vp, vp, vp, i32]
            lib.oracle_attn_decode.restype = i32
            lib.oracle_attn_decode.argtypes = [
                vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, f64, vp, vp, i32]
            lib.oracle_num_threads.restype = i32
            lib.oracle_num_threads.argtypes = [i32]
            lib.oracle_e4m3_value.restype = f64
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_f16_value.restype = f64
            lib.oracle_f16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_dequant_kv8.restype = i32
            lib.oracle_dequant_kv8.argtypes = [vp, i32, vp, i32, i32, i32, i32, vp]
            lib.oracle_widen.restype = i32
            lib.oracle_widen.argtypes = [vp, i32, ctypes.c_size_t, vp]
            _lib = lib
    return _lib


def num_threads(nthreads: int = 0) -> int:
    """Threads the oracle uses for a request of ``nthreads`` (0 = OpenMP default)."""
    return _load().oracle_num_threads(int(nthreads))


def _as_input(x):
    """numpy array or torch CPU tensor -> (contiguous numpy array, dtype code).

    bf16 tensors travel as their raw 16-bit patterns; the C side widens them.
    """
    try:
        import torch  # plumbing only: viewing a CPU tensor's bytes
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return np.ascontiguousarray(x.view(torch.int16).numpy().view(np.uint16)), BF16
            x = x.numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs must be float64, float32 or bf16 bits, got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def attention_prefill(q, k, v, scale: float, is_causal: bool, rows=None,
                      want_probs: bool = False, nthreads: int = 0):
    """Eager fp64 attention for Q [B,Hq,Lq,D] against K/V [B,Hkv,Lk,D].

    rows: optional sequence of query positions to evaluate (default: all).
    Returns (out [B,Hq,R,D], lse [B,Hq,R]) and, with want_probs, the softmax
    weights [B,Hq,R,Lk] as a third element.  All fp64.
    """
    qa, dt = _as_input(q)
    ka, dk = _as_input(k)
    va, dv = _as_input(v)
    if not (dt == dk == dv):
        raise TypeError("q, k, v must share one element type")
    if qa.ndim != 4 or ka.ndim != 4 or va.ndim != 4:
        raise ValueError("q, k, v must be 4-d [B,H,L,D]")
    B, Hq, Lq, D = qa.shape
    Bk, Hkv, Lk, Dk = ka.shape
    if (Bk, Dk) != (B, D) or va.shape != ka.shape:
        raise ValueError("shape mismatch between q, k, v")
    if rows is None:
        rows_arr = None
        R = Lq
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        R = rows_arr.size
    out = np.zeros((B, Hq, R, D), dtype=np.float64)
    lse = np.zeros((B, Hq, R), dtype=np.float64)
    probs = np.zeros((B, Hq, R, Lk), dtype=np.float64) if want_probs else None
    rc = _load().oracle_attn_prefill(
        _ptr(qa), _ptr(ka), _ptr(va), dt, B, Hq, Hkv, Lq, Lk, D, float(scale),
        int(bool(is_causal)), None if rows_arr is None else _ptr(rows_arr), R,
        _ptr(out), _ptr(lse), None if probs is None else _ptr(probs), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_prefill failed with code {rc}")
    return (out, lse, probs) if want_probs else (out, lse)


def attention_decode(q, k_cache, v_cache, seqlens, scale: float, nthreads: int = 0):
    """Eager fp64 decode: q [B,Hq,D] against a cache [B,Hkv,Lmax,D] of which
    rows 0..seqlens[b]-1 are valid.  Returns (out [B,Hq,D], lse [B,Hq])."""
    qa, dt = _as_input(q)
    ka, dk = _as_input(k_cache)
    va, dv = _as_input(v_cache)
    if not (dt == dk == dv):
        raise TypeError("q, k_cache, v_cache must share one element type")
    B, Hq, D = qa.shape
    Bk, Hkv, Lmax, Dk = ka.shape
    if (Bk, Dk) != (B, D) or va.shape != ka.shape:
        raise ValueError("shape mismatch between q and the cache")
    sl = np.ascontiguousarray(np.asarray(
        seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int32))
    if sl.shape != (B,):
        raise ValueError("seqlens must have shape [B]")
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    rc = _load().oracle_attn_decode(
        _ptr(qa), _ptr(ka), _ptr(va), dt, _ptr(sl), B, Hq, Hkv, Lmax, D, float(scale),
        _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_decode failed with code {rc}")
    return out, lse


KV_E4M3, KV_Q8_0 = 1, 2


def e4m3_value(code: int) -> float:
    """Value of one FP8 E4M3 code (OCP definition; NaN for S.1111.111)."""
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def f16_value(bits: int) -> float:
    """Value of one IEEE binary16 bit pattern."""
    return float(_load().oracle_f16_value(int(bits) & 0xFFFF))


def _raw_bytes(x) -> np.ndarray:
    """8-bit codes (torch float8 / int8 / uint8 tensor or numpy array) as a uint8 array."""
    try:
        import torch  # plumbing only: viewing a CPU tensor's bytes
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous().view(torch.uint8).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype.itemsize != 1:
        raise TypeError("8-bit codes expected")
    return x.view(np.uint8)


def dequantize_kv8(codes, fmt: int, scales) -> np.ndarray:
    """codes [B,Hkv,L,D] -> fp64 element values.

    fmt KV_E4M3: scales fp32 [Hkv], element = scales[g] * value(code).
    fmt KV_Q8_0: scales fp16 [B,Hkv,L,D/32], element = scales[b,g,r,d//32] * int8(code).
    """
    c = _raw_bytes(codes)
    if c.ndim != 4:
        raise ValueError("codes must be [B,Hkv,L,D]")
    B, Hkv, L, D = c.shape
    try:
        import torch
        if isinstance(scales, torch.Tensor):
            scales = scales.detach().cpu().contiguous()
            scales = scales.view(torch.int16).numpy().view(np.uint16) if scales.dtype == torch.float16 \
                else scales.numpy()
    except ImportError:  # pragma: no cover
        pass
    sc = np.ascontiguousarray(scales)
    if fmt == KV_E4M3:
        sc = np.ascontiguousarray(sc, dtype=np.float32)
        if sc.shape != (Hkv,):
            raise ValueError("E4M3 scales must be [Hkv]")
    elif fmt == KV_Q8_0:
        if sc.dtype == np.float16:
            sc = sc.view(np.uint16)
        if sc.dtype != np.uint16 or sc.shape != (B, Hkv, L, D // 32):
            raise ValueError("Q8_0 scales must be fp16 [B,Hkv,L,D/32]")
    else:
        raise ValueError("unknown 8-bit format")
    out = np.zeros((B, Hkv, L, D), dtype=np.float64)
    rc = _load().oracle_dequant_kv8(_ptr(c), int(fmt), _ptr(sc), B, Hkv, L, D, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_dequant_kv8 failed with code {rc}")
    return out


def widen(x) -> np.ndarray:
    """fp64, fp32 or bf16 input -> fp64 array of the same shape (exact)."""
    a, dt = _as_input(x)
    out = np.zeros(a.shape, dtype=np.float64)
    rc = _load().oracle_widen(_ptr(a), dt, a.size, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_widen failed")
    return out


def attention_decode_kv8(q, k_codes, v_codes, fmt: int, k_scale, v_scale, seqlens, scale: float,
                         nthreads: int = 0):
    """Lq new query rows per sequence against an 8-bit cache, exactly: the
    cache is dequantised to fp64 and the rows are the last Lq of sequence b's
    seqlens[b] rows (bottom-right causal, as attention_prefill with is_causal).

    q [B,Hq,Lq,D]; codes [B,Hkv,Lmax,D]; returns (out [B,Hq,Lq,D], lse [B,Hq,Lq]) fp64.
    """
    qd = widen(q)
    K = dequantize_kv8(k_codes, fmt, k_scale)
    V = dequantize_kv8(v_codes, fmt, v_scale)
    sl = np.asarray(seqlens.cpu().numpy() if hasattr(seqlens, "cpu") else seqlens, dtype=np.int64)
    B, Hq, Lq, D = qd.shape
    outs = np.zeros((B, Hq, Lq, D), dtype=np.float64)
    lses = np.zeros((B, Hq, Lq), dtype=np.float64)
    for b in range(B):
        n = int(sl[b])
        o, l = attention_prefill(qd[b:b + 1], np.ascontiguousarray(K[b:b + 1, :, :n]),
                                 np.ascontiguousarray(V[b:b + 1, :, :n]), scale, True, nthreads=nthreads)
        outs[b], lses[b] = o[0], l[0]
    return outs, lses
