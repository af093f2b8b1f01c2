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

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
the pages print (the numpy mask demonstration) and against closed forms.
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
