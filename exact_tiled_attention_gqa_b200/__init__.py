"""Exact tiled grouped-query attention for NVIDIA B200 (sm_100a).

Two calls, both thin wrappers over the C ABI in ``include/attn_gqa.h``:

* ``prefill(q, k, v, is_causal=True)`` -- softmax(scale Q K^T + mask) V with
  the bottom-right causal mask, for Q [B,Hq,Lq,D] and K/V [B,Hkv,Lk,D] bf16.
* ``decode(q, k_cache, v_cache, seqlens)`` -- one new token per sequence
  against a KV cache [B,Hkv,Lmax,D] whose rows 0..seqlens[b]-1 are valid.
* ``decode_mq(q, k_cache, v_cache, seqlens)`` -- Lq new tokens per sequence
  (q [B,Hq,Lq,D]), the last Lq rows of the cache, bottom-right causal: the
  verify step of speculative decoding.
* ``decode_paged(q, k_pages, v_pages, block_table, seqlens)`` -- decode_mq over
  a paged cache: pools [n_pages,Hkv,page_size,D] and a block table [B,max_pages].

Both return ``(out, lse)``: out bf16 shaped like q, lse fp32 (natural log).
PyTorch supplies device memory and the current stream; every step of the
computation runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _native
from ._native import AttnError

__all__ = ["prefill", "prefill_workspace_size", "prefill_host", "decode", "decode_host", "decode_host_workspace_size", "decode_partial", "decode_merge", "decode_merge_peers", "kvp_signal",
           "kvp_wait", "decode_mq", "decode_paged", "decode_noalloc", "decode_kv8", "decode_kv8_paged", "prefill_host_scratch_size", "decode_workspace_size", "decode_mq_workspace_size",
           "decode_kv8_workspace_size", "device_error", "AttnError", "library_path"]


def library_path() -> str:
    return _native.LIB_PATH


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(name: str, t: torch.Tensor, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-d, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _check_on(device: torch.device, _ref: str = "q", **tensors) -> None:
    """Every given tensor (None skipped) lives on `device`, the device of the tensor named `_ref`."""
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, but {_ref} is on {device}")


def _result(name: str, t: Optional[torch.Tensor], dtype: torch.dtype, shape, device: torch.device,
            want: bool = True) -> Optional[torch.Tensor]:
    """A caller's output tensor, checked against the shape the call writes, or a new one.

    The library writes exactly `shape` elements through the pointer, so a
    smaller or differently laid out buffer is refused here rather than
    overrun on the device."""
    shape = tuple(int(x) for x in shape)
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device) if want else None
    _check_tensor(name, t, dtype, len(shape))
    if tuple(t.shape) != shape:
        raise ValueError(f"{name} must have shape {shape}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, but q is on {device}")
    return t


def _workspace(ws: Optional[torch.Tensor], need: int, device: torch.device):
    """(pointer, size in bytes) of a caller's workspace, or of a new one of `need` bytes."""
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    if not isinstance(ws, torch.Tensor) or not ws.is_contiguous() or ws.device != device:
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    return ws, ws.numel() * ws.element_size()


def _squeezed_results(out, lse, q4: torch.Tensor, want_lse: bool, squeezed: bool):
    """out / lse for a call whose q was given as [B,Hq,D] and viewed as [B,Hq,1,D]:
    results the caller passed in that 3-d / 2-d form are viewed the same way."""
    B, Hq, Lq, D = q4.shape
    if squeezed:
        if out is not None:
            out = _result("out", out, torch.bfloat16, (B, Hq, D), q4.device).unsqueeze(2)
        if lse is not None:
            lse = _result("lse", lse, torch.float32, (B, Hq), q4.device).unsqueeze(2)
    out = _result("out", out, torch.bfloat16, q4.shape, q4.device)
    lse = _result("lse", lse, torch.float32, (B, Hq, Lq), q4.device, want_lse)
    return out, lse


def prefill_workspace_size(B: int, Hq: int, Hkv: int, Lq: int, Lk: int, D: int, is_causal: bool = True) -> int:
    return int(_native.lib().attn_prefill_workspace_size(B, Hq, Hkv, Lq, Lk, D, int(bool(is_causal))))


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: Optional[float] = None,
            is_causal: bool = True, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            want_lse: bool = True, workspace: Optional[torch.Tensor] = None, split: bool = True, stream=None):
    """Exact GQA attention.  q [B,Hq,Lq,D], k/v [B,Hkv,Lk,D] bf16 (CUDA, contiguous).

    With split (default) the call goes through attn_prefill_ws whenever
    prefill_workspace_size(...) is non-zero (a launch ending in a part-filled
    wave of near-equal units), using `workspace` or a new one; split=False is
    always attn_prefill."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t, torch.bfloat16, 4)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != D or v.shape != k.shape:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    _check_on(q.device, k=k, v=v)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = _result("out", out, torch.bfloat16, q.shape, q.device)
    lse = _result("lse", lse, torch.float32, (B, Hq, Lq), q.device, want_lse)
    with torch.cuda.device(q.device):
        need = prefill_workspace_size(B, Hq, Hkv, Lq, Lk, D, is_causal) if split and B * Lq * Lk > 0 else 0
        if need > 0:
            workspace, ws_bytes = _workspace(workspace, need, q.device)
            st = _native.lib().attn_prefill_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lk,
                                               D, float(scale), int(bool(is_causal)), _ptr(workspace), ws_bytes,
                                               _stream_handle(stream))
            _native.check(st, "attn_prefill_ws")
        else:
            st = _native.lib().attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lk, D,
                                            float(scale), int(bool(is_causal)), _stream_handle(stream))
            _native.check(st, "attn_prefill")
    return out, lse


def prefill_host_scratch_size(B: int, Hq: int, Hkv: int, Lq: int, Lk: int, D: int) -> int:
    return int(_native.lib().attn_prefill_host_scratch_size(B, Hq, Hkv, Lq, Lk, D))


def prefill_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: Optional[float] = None,
                 is_causal: bool = True, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 want_lse: bool = True, scratch: Optional[torch.Tensor] = None, device=None, stream=None):
    """attn_prefill on CPU tensors (pinned for overlap): copies in, kernels and copies out are
    pipelined by the library.  Results are in `out` / `lse` once `stream` (default: the current
    stream of `device`) has passed the call, e.g. after stream.synchronize()."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 4-d bf16 CPU tensor")
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("shape mismatch between q, k, v")
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, pin_memory=True)
    for name, t, dt, shp in (("out", out, torch.bfloat16, tuple(q.shape)), ("lse", lse, torch.float32, (B, Hq, Lq))):
        if t is not None and (t.is_cuda or not t.is_contiguous() or t.dtype != dt or tuple(t.shape) != shp):
            raise ValueError(f"{name} must be a contiguous {dt} CPU tensor of shape {shp}")
    need = prefill_host_scratch_size(B, Hq, Hkv, Lq, Lk, D)
    scratch, scratch_bytes = _workspace(scratch, need, device)
    with torch.cuda.device(device):
        st = _native.lib().attn_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lk,
                                             D, float(scale), int(bool(is_causal)), _ptr(scratch), scratch_bytes,
                                             _stream_handle(stream))
    _native.check(st, "attn_prefill_host")
    return out, lse


def decode_workspace_size(B: int, Hq: int, Hkv: int, Lmax: int, D: int) -> int:
    return int(_native.lib().attn_decode_workspace_size(B, Hq, Hkv, Lmax, D))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor, *,
           scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           want_lse: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """One query token per sequence.  q [B,Hq,D], caches [B,Hkv,Lmax,D] bf16, seqlens int32 [B] (CUDA)."""
    _check_tensor("q", q, torch.bfloat16, 3)
    _check_tensor("k_cache", k_cache, torch.bfloat16, 4)
    _check_tensor("v_cache", v_cache, torch.bfloat16, 4)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    _check_on(q.device, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = _result("out", out, torch.bfloat16, q.shape, q.device)
    lse = _result("lse", lse, torch.float32, (B, Hq), q.device, want_lse)
    workspace, ws_bytes = _workspace(workspace, decode_workspace_size(B, Hq, Hkv, Lmax, D), q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out), _ptr(lse),
                                       B, Hq, Hkv, Lmax, D, float(scale), _ptr(workspace), ws_bytes,
                                       _stream_handle(stream))
    _native.check(st, "attn_decode")
    return out, lse


def decode_host_workspace_size(B: int, Hq: int, Hkv: int, Lmax: int, D: int) -> int:
    return int(_native.lib().attn_decode_host_workspace_size(B, Hq, Hkv, Lmax, D))


def decode_host(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor, *,
                scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                want_lse: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """decode with q, seqlens, out and lse on the host (CPU tensors, pinned for asynchronous copies) and the
    caches on the device: one call copies q and seqlens in, decodes and copies the results out.  They are in
    `out` / `lse` once `stream` (default: the current stream of the caches' device) has passed the call."""
    for name, t, dt, nd in (("q", q, torch.bfloat16, 3), ("seqlens", seqlens, torch.int32, 1)):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != dt or t.dim() != nd or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {nd}-d {dt} CPU tensor")
    _check_tensor("k_cache", k_cache, torch.bfloat16, 4)
    _check_tensor("v_cache", v_cache, torch.bfloat16, 4)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    _check_on(k_cache.device, "k_cache", v_cache=v_cache)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, pin_memory=True)
    for name, t, dt, shp in (("out", out, torch.bfloat16, tuple(q.shape)), ("lse", lse, torch.float32, (B, Hq))):
        if t is not None and (t.is_cuda or not t.is_contiguous() or t.dtype != dt or tuple(t.shape) != shp):
            raise ValueError(f"{name} must be a contiguous {dt} CPU tensor of shape {shp}")
    need = decode_host_workspace_size(B, Hq, Hkv, Lmax, D)
    workspace, ws_bytes = _workspace(workspace, need, k_cache.device)
    with torch.cuda.device(k_cache.device):
        st = _native.lib().attn_decode_host(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out),
                                            _ptr(lse), B, Hq, Hkv, Lmax, D, float(scale), _ptr(workspace), ws_bytes,
                                            _stream_handle(stream))
    _native.check(st, "attn_decode_host")
    return out, lse


def decode_partial(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor, *,
                   scale: Optional[float] = None, o_part: Optional[torch.Tensor] = None,
                   lse_part: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """decode over the cache rows this device holds, results unrounded for decode_merge:
    (o_part fp32 [B,Hq,D], lse_part fp32 [B,Hq], natural log, -inf where a sequence has no rows here).
    o_part / lse_part may be given (e.g. slices of an exchange buffer) and are then written in place."""
    _check_tensor("q", q, torch.bfloat16, 3)
    _check_tensor("k_cache", k_cache, torch.bfloat16, 4)
    _check_tensor("v_cache", v_cache, torch.bfloat16, 4)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    _check_on(q.device, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    o_part = _result("o_part", o_part, torch.float32, (B, Hq, D), q.device)
    lse_part = _result("lse_part", lse_part, torch.float32, (B, Hq), q.device)
    workspace, ws_bytes = _workspace(workspace, decode_workspace_size(B, Hq, Hkv, Lmax, D), q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_partial(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(o_part),
                                               _ptr(lse_part), B, Hq, Hkv, Lmax, D, float(scale), _ptr(workspace),
                                               ws_bytes, _stream_handle(stream))
    _native.check(st, "attn_decode_partial")
    return o_part, lse_part


def decode_merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Merge partial decode results over disjoint cache rows: o_parts fp32 [n, ..., D], lse_parts fp32 [n, ...]
    (natural log) -> (out bf16 [..., D], lse fp32 [...])."""
    _check_tensor("o_parts", o_parts, torch.float32, o_parts.dim())
    _check_tensor("lse_parts", lse_parts, torch.float32, lse_parts.dim())
    n, D = o_parts.shape[0], o_parts.shape[-1]
    if tuple(lse_parts.shape) != tuple(o_parts.shape[:-1]) or o_parts.dim() < 3:
        raise ValueError("o_parts must be [n, ..., D] and lse_parts [n, ...]")
    rows = lse_parts[0].numel()
    _check_on(o_parts.device, lse_parts=lse_parts)
    out = _result("out", out, torch.bfloat16, o_parts.shape[1:], o_parts.device)
    lse = _result("lse", lse, torch.float32, lse_parts.shape[1:], o_parts.device, want_lse)
    with torch.cuda.device(o_parts.device):
        st = _native.lib().attn_decode_merge(_ptr(o_parts), _ptr(lse_parts), n, rows, D, _ptr(out), _ptr(lse),
                                             _stream_handle(stream))
    _native.check(st, "attn_decode_merge")
    return out, lse


def _ptr_array(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.int64 or t.dim() != 1 \
            or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 1-d int64 CUDA tensor of device pointers")
    return t


def kvp_signal(flag_ptrs: torch.Tensor, value: int, *, stream=None) -> None:
    """Store `value` to each flag whose address is in flag_ptrs (int64 device tensor of
    pointers), with release semantics, after this stream's earlier work is visible."""
    _ptr_array(flag_ptrs, "flag_ptrs")
    with torch.cuda.device(flag_ptrs.device):
        st = _native.lib().attn_kvp_signal(_ptr(flag_ptrs), flag_ptrs.numel(), int(value) & 0xFFFFFFFF,
                                           _stream_handle(stream))
    _native.check(st, "attn_kvp_signal")


def kvp_wait(flags: torch.Tensor, value: int, *, stream=None) -> None:
    """Make the stream wait until every flag (uint32 storage, given as an int32 tensor) has reached `value`."""
    _check_tensor("flags", flags, torch.int32, 1)
    with torch.cuda.device(flags.device):
        st = _native.lib().attn_kvp_wait(_ptr(flags), flags.numel(), int(value) & 0xFFFFFFFF,
                                         _stream_handle(stream))
    _native.check(st, "attn_kvp_wait")


def decode_merge_peers(o_ptrs: torch.Tensor, lse_ptrs: torch.Tensor, ready: torch.Tensor, value: int, rows: int,
                       D: int, *, out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    """decode_merge over parts that stay where they were computed: part p's O at o_ptrs[p]
    ([rows, D] fp32) and LSE at lse_ptrs[p] ([rows]), read once ready[p] has reached `value`."""
    _ptr_array(o_ptrs, "o_ptrs")
    _ptr_array(lse_ptrs, "lse_ptrs")
    _check_tensor("ready", ready, torch.int32, 1)
    if o_ptrs.numel() != lse_ptrs.numel() or ready.numel() != o_ptrs.numel():
        raise ValueError("o_ptrs, lse_ptrs and ready must have one entry per part")
    _check_tensor("out", out, torch.bfloat16, out.dim())
    if out.numel() != rows * D or (lse is not None and lse.numel() != rows):
        raise ValueError("out must hold rows * D values and lse rows values")
    with torch.cuda.device(out.device):
        st = _native.lib().attn_decode_merge_peers(_ptr(o_ptrs), _ptr(lse_ptrs), _ptr(ready), int(value) & 0xFFFFFFFF,
                                                   o_ptrs.numel(), rows, D, _ptr(out), _ptr(lse),
                                                   _stream_handle(stream))
    _native.check(st, "attn_decode_merge_peers")
    return out, lse


def decode_mq_workspace_size(B: int, Hq: int, Hkv: int, Lq: int, Lmax: int, D: int) -> int:
    return int(_native.lib().attn_decode_mq_workspace_size(B, Hq, Hkv, Lq, Lmax, D))


def decode_mq(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor, *,
              scale: Optional[float] = None, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
              want_lse: bool = True, workspace: Optional[torch.Tensor] = None, stream=None):
    """Lq new tokens per sequence.  q [B,Hq,Lq,D], caches [B,Hkv,Lmax,D] bf16, seqlens int32 [B] (CUDA);
    the new tokens are the last Lq of each sequence's seqlens[b] cached rows."""
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k_cache", k_cache, torch.bfloat16, 4)
    _check_tensor("v_cache", v_cache, torch.bfloat16, 4)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, Lq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    _check_on(q.device, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = _result("out", out, torch.bfloat16, q.shape, q.device)
    lse = _result("lse", lse, torch.float32, (B, Hq, Lq), q.device, want_lse)
    workspace, ws_bytes = _workspace(workspace, decode_mq_workspace_size(B, Hq, Hkv, Lq, Lmax, D), q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_mq(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out),
                                          _ptr(lse), B, Hq, Hkv, Lq, Lmax, D, float(scale), _ptr(workspace),
                                          ws_bytes, _stream_handle(stream))
    _native.check(st, "attn_decode_mq")
    return out, lse


def decode_kv8_workspace_size(B: int, Hq: int, Hkv: int, Lq: int, Lmax: int, D: int) -> int:
    return int(_native.lib().attn_decode_kv8_workspace_size(B, Hq, Hkv, Lq, Lmax, D))


def decode_kv8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: torch.Tensor,
               v_scale: torch.Tensor, seqlens: torch.Tensor, *, scale: Optional[float] = None,
               out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True,
               workspace: Optional[torch.Tensor] = None, stream=None):
    """Decode against an 8-bit cache.  q [B,Hq,Lq,D] (or [B,Hq,D]) bf16; caches [B,Hkv,Lmax,D] of
    torch.float8_e4m3fn (E4M3; k_scale / v_scale float32 [Hkv]) or torch.int8 (Q8_0; k_scale / v_scale
    float16 [B,Hkv,Lmax,D/32]); seqlens int32 [B]; all on one CUDA device."""
    squeeze = q.dim() == 3
    if squeeze:
        q = q.unsqueeze(2)
    _check_tensor("q", q, torch.bfloat16, 4)
    if k_cache.dtype == torch.float8_e4m3fn:
        fmt, sdt, sdim = _native.ATTN_KV_E4M3, torch.float32, 1
    elif k_cache.dtype == torch.int8:
        fmt, sdt, sdim = _native.ATTN_KV_Q8_0, torch.float16, 4
    else:
        raise TypeError(f"k_cache must be torch.float8_e4m3fn or torch.int8, got {k_cache.dtype}")
    _check_tensor("k_cache", k_cache, k_cache.dtype, 4)
    _check_tensor("v_cache", v_cache, k_cache.dtype, 4)
    _check_tensor("k_scale", k_scale, sdt, sdim)
    _check_tensor("v_scale", v_scale, sdt, sdim)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, Lq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    want_scale = (Hkv,) if fmt == _native.ATTN_KV_E4M3 else (B, Hkv, Lmax, D // 32)
    if tuple(k_scale.shape) != want_scale or tuple(v_scale.shape) != want_scale:
        raise ValueError(f"k_scale / v_scale must have shape {want_scale}")
    _check_on(q.device, k_cache=k_cache, v_cache=v_cache, k_scale=k_scale, v_scale=v_scale, seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out, lse = _squeezed_results(out, lse, q, want_lse, squeeze)
    workspace, ws_bytes = _workspace(workspace, decode_kv8_workspace_size(B, Hq, Hkv, Lq, Lmax, D), q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_kv8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), fmt,
                                           _ptr(seqlens), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lmax, D,
                                           float(scale), _ptr(workspace), ws_bytes, _stream_handle(stream))
    _native.check(st, "attn_decode_kv8")
    if squeeze:
        out = out.squeeze(2)
        lse = None if lse is None else lse.squeeze(2)
    return out, lse


def decode_kv8_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, k_scale: torch.Tensor,
                     v_scale: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor, *,
                     scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                     workspace: Optional[torch.Tensor] = None, stream=None):
    """Paged decode against an 8-bit cache.  q [B,Hq,Lq,D] (or [B,Hq,D]) bf16; code pools
    [n_pages,Hkv,page_size,D] of torch.float8_e4m3fn (k_scale / v_scale float32 [Hkv]) or torch.int8
    (k_scale / v_scale float16 [n_pages,Hkv,page_size,D/32]); block_table int32 [B,max_pages]; seqlens int32 [B]."""
    squeeze = q.dim() == 3
    if squeeze:
        q = q.unsqueeze(2)
    _check_tensor("q", q, torch.bfloat16, 4)
    if k_pages.dtype == torch.float8_e4m3fn:
        fmt, sdt, sdim = _native.ATTN_KV_E4M3, torch.float32, 1
    elif k_pages.dtype == torch.int8:
        fmt, sdt, sdim = _native.ATTN_KV_Q8_0, torch.float16, 4
    else:
        raise TypeError(f"k_pages must be torch.float8_e4m3fn or torch.int8, got {k_pages.dtype}")
    _check_tensor("k_pages", k_pages, k_pages.dtype, 4)
    _check_tensor("v_pages", v_pages, k_pages.dtype, 4)
    _check_tensor("k_scale", k_scale, sdt, sdim)
    _check_tensor("v_scale", v_scale, sdt, sdim)
    _check_tensor("block_table", block_table, torch.int32, 2)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, Lq, D = q.shape
    n_pages, Hkv, page_size = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = block_table.shape[1]
    if (k_pages.shape[3] != D or v_pages.shape != k_pages.shape or block_table.shape[0] != B
            or seqlens.shape[0] != B):
        raise ValueError("shape mismatch between q, the page pools, block_table and seqlens")
    want_scale = (Hkv,) if fmt == _native.ATTN_KV_E4M3 else (n_pages, Hkv, page_size, D // 32)
    if tuple(k_scale.shape) != want_scale or tuple(v_scale.shape) != want_scale:
        raise ValueError(f"k_scale / v_scale must have shape {want_scale}")
    _check_on(q.device, k_pages=k_pages, v_pages=v_pages, k_scale=k_scale, v_scale=v_scale, block_table=block_table,
              seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out, lse = _squeezed_results(out, lse, q, want_lse, squeeze)
    need = int(_native.lib().attn_decode_kv8_paged_workspace_size(B, Hq, Hkv, Lq, page_size, max_pages, D))
    workspace, ws_bytes = _workspace(workspace, need, q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_kv8_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(k_scale), _ptr(v_scale),
                                                 fmt, _ptr(block_table), _ptr(seqlens), _ptr(out), _ptr(lse), B, Hq,
                                                 Hkv, Lq, n_pages, page_size, max_pages, D, float(scale),
                                                 _ptr(workspace), ws_bytes, _stream_handle(stream))
    _native.check(st, "attn_decode_kv8_paged")
    if squeeze:
        out = out.squeeze(2)
        lse = None if lse is None else lse.squeeze(2)
    return out, lse


def decode_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_table: torch.Tensor,
                 seqlens: torch.Tensor, *, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, want_lse: bool = True, workspace: Optional[torch.Tensor] = None,
                 stream=None):
    """Paged-cache decode.  q [B,Hq,Lq,D] (or [B,Hq,D] for Lq = 1), pools [n_pages,Hkv,page_size,D],
    block_table int32 [B,max_pages], seqlens int32 [B], all on one CUDA device."""
    squeeze = q.dim() == 3
    if squeeze:
        q = q.unsqueeze(2)
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k_pages", k_pages, torch.bfloat16, 4)
    _check_tensor("v_pages", v_pages, torch.bfloat16, 4)
    _check_tensor("block_table", block_table, torch.int32, 2)
    _check_tensor("seqlens", seqlens, torch.int32, 1)
    B, Hq, Lq, D = q.shape
    n_pages, Hkv, page_size = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    max_pages = block_table.shape[1]
    if (k_pages.shape[3] != D or v_pages.shape != k_pages.shape or block_table.shape[0] != B
            or seqlens.shape[0] != B):
        raise ValueError("shape mismatch between q, the page pools, block_table and seqlens")
    _check_on(q.device, k_pages=k_pages, v_pages=v_pages, block_table=block_table, seqlens=seqlens)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out, lse = _squeezed_results(out, lse, q, want_lse, squeeze)
    need = int(_native.lib().attn_decode_paged_workspace_size(B, Hq, Hkv, Lq, page_size, max_pages, D))
    workspace, ws_bytes = _workspace(workspace, need, q.device)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                             _ptr(seqlens), _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, n_pages, page_size,
                                             max_pages, D, float(scale), _ptr(workspace), ws_bytes,
                                             _stream_handle(stream))
    _native.check(st, "attn_decode_paged")
    if squeeze:
        out = out.squeeze(2)
        lse = None if lse is None else lse.squeeze(2)
    return out, lse


def decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, seqlens: torch.Tensor, *,
                   scale: Optional[float] = None, out: torch.Tensor, lse: Optional[torch.Tensor] = None, stream=None):
    """decode() for callers that cannot allocate: the split partials use the
    library's own fixed scratch (16 MiB per GPU), and `out` (and `lse`, if
    wanted) must be passed in.  Calls on one GPU must not overlap in time."""
    for n, t, dt, nd in (("q", q, torch.bfloat16, 3), ("k_cache", k_cache, torch.bfloat16, 4),
                         ("v_cache", v_cache, torch.bfloat16, 4), ("seqlens", seqlens, torch.int32, 1)):
        _check_tensor(n, t, dt, nd)
    B, Hq, D = q.shape
    Hkv, Lmax = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape[0] != B or k_cache.shape[3] != D or v_cache.shape != k_cache.shape or seqlens.shape[0] != B:
        raise ValueError("shape mismatch between q, the caches and seqlens")
    _check_on(q.device, k_cache=k_cache, v_cache=v_cache, seqlens=seqlens)
    if out is None:
        raise ValueError("out must be given: decode_noalloc allocates nothing")
    _result("out", out, torch.bfloat16, q.shape, q.device)
    if lse is not None:
        _result("lse", lse, torch.float32, (B, Hq), q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    with torch.cuda.device(q.device):
        st = _native.lib().attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(out),
                                               _ptr(lse), B, Hq, Hkv, Lmax, D, float(scale), _stream_handle(stream))
    _native.check(st, "attn_decode_noalloc")
    return out, lse


def device_error(reset: bool = True) -> int:
    """Synchronise and return (and by default clear) the device-side error word."""
    flags = ctypes.c_uint(0)
    _native.check(_native.lib().attn_device_error(ctypes.byref(flags), int(bool(reset))), "attn_device_error")
    return int(flags.value)
