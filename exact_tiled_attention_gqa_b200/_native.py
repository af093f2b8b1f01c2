"""ctypes binding of include/attn_gqa.h -- argument marshalling only.

Every call converts tensors to device pointers and sizes, passes the caller's
CUDA stream, and raises ``AttnError`` on a non-zero status.  All computation
happens in the CUDA kernels of ``libattn_gqa_sm100.so``; there is no other
path: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

from .build import DEBUG_LIB_PATH, LIB_PATH

# ATTN_GQA_DEBUG_BOUNDS=1 in the environment loads the bounds-checking build of
# the same sources instead (build.py, debug_bounds=True); tests use it.
if os.environ.get("ATTN_GQA_DEBUG_BOUNDS") == "1":
    LIB_PATH = DEBUG_LIB_PATH

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_WORKSPACE = -3
ATTN_ERR_CUDA = -4
ATTN_DEVERR_TIMEOUT = 0x1
ATTN_DEVERR_SEQLEN = 0x2
ATTN_DEVERR_PAGE = 0x4
ATTN_DEVERR_SCHED = 0x8
ATTN_DEVERR_BOUNDS = 0x10
ATTN_DECODE_NOALLOC_SCRATCH_BYTES = 16 << 20
ATTN_KV_E4M3 = 1
ATTN_KV_Q8_0 = 2

# name -> (restype, argtypes): every symbol the header declares
_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "attn_prefill": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp]),
    "attn_prefill_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_prefill_split_plan": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "attn_prefill_ws": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp]),
    "attn_prefill_host_scratch_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_prefill_host": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz,
                                 _vp]),
    "attn_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "attn_decode": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _sz, _vp]),
    "attn_decode_host_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "attn_decode_host": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _sz, _vp]),
    "attn_decode_partial": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _sz, _vp]),
    "attn_decode_merge": (_i32, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "attn_kvp_signal": (_i32, [_vp, _i32, ctypes.c_uint, _vp]),
    "attn_kvp_wait": (_i32, [_vp, _i32, ctypes.c_uint, _vp]),
    "attn_decode_merge_peers": (_i32, [_vp, _vp, _vp, ctypes.c_uint, _i32, _i32, _i32, _vp, _vp, _vp]),
    "attn_decode_mq_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_decode_mq": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _sz,
                              _vp]),
    "attn_decode_paged_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_decode_paged": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                 _f32, _vp, _sz, _vp]),
    "attn_decode_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp]),
    "attn_decode_kv8_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_decode_kv8": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                               _f32, _vp, _sz, _vp]),
    "attn_decode_kv8_paged_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "attn_decode_kv8_paged": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                     _i32, _i32, _i32, _f32, _vp, _sz, _vp]),
    "attn_selftest_kv8_convert": (_i32, [_vp, _vp, _i32, _i32, _vp]),
    "attn_selftest_wait": (_i32, [ctypes.c_ulonglong, _vp, _vp]),
    "attn_prefill_sched_busy": (_i32, [ctypes.POINTER(_i32)]),
    "attn_status_string": (ctypes.c_char_p, [_i32]),
    "attn_last_error": (ctypes.c_char_p, []),
    "attn_device_error": (_i32, [ctypes.POINTER(ctypes.c_uint), _i32]),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library (built in-tree); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_gqa_b200.build` "
                    "(there is no fallback implementation)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def check(status: int, what: str) -> None:
    if status != ATTN_OK:
        L = lib()
        name = L.attn_status_string(status).decode()
        detail = L.attn_last_error().decode()
        raise AttnError(status, f"{what}: {name}: {detail}")
