"""The C ABI: every symbol the header declares is exported, and argument checks
fail cleanly before anything reaches a GPU (these calls never launch work)."""
import ctypes
import os
import re

import pytest

from exact_tiled_attention_gqa_b200 import _native
from exact_tiled_attention_gqa_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_gqa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _native.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_calls():
    assert declared_symbols() == sorted(_native.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.attn_status_string(0) == b"ATTN_OK"
    assert lib.attn_status_string(-1) == b"ATTN_ERR_INVALID_ARG"
    assert lib.attn_status_string(-2) == b"ATTN_ERR_UNSUPPORTED"
    assert lib.attn_status_string(-3) == b"ATTN_ERR_WORKSPACE"
    assert lib.attn_status_string(-4) == b"ATTN_ERR_CUDA"
    assert lib.attn_status_string(7) == b"ATTN_ERR_UNKNOWN"


# fake, aligned addresses: only ever passed together with an invalid argument,
# so the call returns before touching CUDA
A = ctypes.c_void_p(0x10000)
NULL = None


def _prefill(lib, **kw):
    args = dict(q=A, k=A, v=A, out=A, lse=NULL, B=1, Hq=8, Hkv=2, Lq=16, Lk=16, D=128, scale=0.1, causal=1)
    args.update(kw)
    return lib.attn_prefill(args["q"], args["k"], args["v"], args["out"], args["lse"], args["B"], args["Hq"],
                            args["Hkv"], args["Lq"], args["Lk"], args["D"], args["scale"], args["causal"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(q=NULL), -1), (dict(out=NULL), -1), (dict(B=-1), -1), (dict(Lq=-3), -1), (dict(Lk=-1), -1),
    (dict(Hq=0), -1), (dict(Hkv=0), -1), (dict(Hq=6, Hkv=4), -1), (dict(scale=0.0), -1),
    (dict(scale=-1.0), -1), (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1),
    (dict(q=ctypes.c_void_p(0x10008)), -1), (dict(lse=ctypes.c_void_p(0x10002)), -1),
    (dict(D=96), -2), (dict(D=512), -2), (dict(Hq=256, Hkv=1), -2),
])
def test_prefill_rejects(lib, bad, code):
    assert _prefill(lib, **bad) == code
    assert lib.attn_last_error() != b""


def test_prefill_empty_is_noop(lib):
    assert _prefill(lib, B=0) == 0
    assert _prefill(lib, Lq=0) == 0
    # empty tensors have no storage: null is accepted for them, and only for them
    assert _prefill(lib, B=0, q=NULL, k=NULL, v=NULL, out=NULL) == 0
    assert _prefill(lib, Lq=0, q=NULL, out=NULL) == 0
    assert _prefill(lib, Lq=0, q=NULL, out=NULL, k=NULL) == -1
    assert _prefill(lib, Lk=0, k=NULL, v=NULL, q=NULL) == -1


def _decode(lib, **kw):
    args = dict(q=A, k=A, v=A, sl=A, out=A, lse=NULL, B=2, Hq=8, Hkv=2, Lmax=64, D=128, scale=0.1, ws=A,
                wsb=1 << 30)
    args.update(kw)
    return lib.attn_decode(args["q"], args["k"], args["v"], args["sl"], args["out"], args["lse"], args["B"],
                           args["Hq"], args["Hkv"], args["Lmax"], args["D"], args["scale"], args["ws"],
                           args["wsb"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(sl=NULL), -1), (dict(sl=ctypes.c_void_p(0x10001)), -1), (dict(Lmax=0), -1), (dict(Hq=5, Hkv=2), -1),
    (dict(k=NULL), -1), (dict(D=32), -2), (dict(Hq=256, Hkv=1), -2), (dict(ws=NULL), -3), (dict(wsb=16), -3),
    (dict(ws=ctypes.c_void_p(0x10010)), -1),
])
def test_decode_rejects(lib, bad, code):
    assert _decode(lib, **bad) == code


def test_decode_empty_batch_is_noop(lib):
    assert _decode(lib, B=0) == 0
    assert _decode(lib, B=0, q=NULL, k=NULL, v=NULL, out=NULL, sl=NULL, ws=NULL) == 0


def test_workspace_size(lib):
    f = lib.attn_decode_workspace_size
    assert f(0, 8, 2, 64, 128) == 0
    assert f(2, 8, 3, 64, 128) == 0        # Hq % Hkv
    assert f(2, 8, 2, 64, 96) == 0         # D
    assert f(2, 8, 2, 64, 512) == 0
    assert f(2, 8, 2, 64, 256) > 0
    assert f(2, 8, 2, 0, 128) == 0         # Lmax
    assert f(1, 256, 1, 64, 128) == 0      # G > 128
    a = f(2, 8, 2, 1000, 128)
    assert a > 0 and a % 256 == 0
    assert f(2, 8, 2, 100000, 128) >= a
    # big enough for one fp32 partial row per split plus its lse
    assert f(64, 32, 8, 32768, 128) >= 64 * 32 * (128 + 1) * 4


def _decode_ws(splits, B, Hq, D=128):
    rows = B * Hq * splits
    return -(-rows * D * 4 // 256) * 256 + -(-rows * 4 // 256) * 256


def test_decode_split_lengths(lib):
    """The split lengths the decode picks for the measured workloads, seen through the
    workspace size (one fp32 partial row and LSE per query row and split)."""
    f = lib.attn_decode_workspace_size
    # group sweep, batch 8, 131072 cached rows: tcgen05 kernel, splits of 4096 rows at
    # G = 64 (32 splits, 256 CTAs) and 8192 rows at G = 32 (16 splits, 256 CTAs)
    assert f(8, 64, 1, 131072, 128) == _decode_ws(32, 8, 64)
    assert f(8, 64, 2, 131072, 128) == _decode_ws(16, 8, 64)
    # Qwen3-8B decode batch (G = 4): mma.sync kernel, splits of 4096 rows at Lmax 32768
    assert f(64, 32, 8, 32768, 128) == _decode_ws(8, 64, 32)


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        _native.lib()


def _decode_mq(lib, **kw):
    args = dict(q=A, k=A, v=A, sl=A, out=A, lse=NULL, B=2, Hq=8, Hkv=2, Lq=4, Lmax=64, D=128, scale=0.1, ws=A,
                wsb=1 << 30)
    args.update(kw)
    return lib.attn_decode_mq(args["q"], args["k"], args["v"], args["sl"], args["out"], args["lse"], args["B"],
                              args["Hq"], args["Hkv"], args["Lq"], args["Lmax"], args["D"], args["scale"], args["ws"],
                              args["wsb"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(Lq=0), -1), (dict(Lq=-2), -1), (dict(sl=NULL), -1), (dict(Hq=6, Hkv=4), -1), (dict(D=80), -2),
    (dict(Lq=33), -2), (dict(Hq=64, Hkv=1, Lq=3), -2), (dict(ws=NULL), -3), (dict(wsb=100), -3),
])
def test_decode_mq_rejects(lib, bad, code):
    assert _decode_mq(lib, **bad) == code


def test_decode_mq_workspace(lib):
    f = lib.attn_decode_mq_workspace_size
    assert f(2, 8, 2, 0, 64, 128) == 0
    assert f(2, 8, 2, 33, 64, 128) == 0          # G * Lq > 128
    assert f(2, 8, 2, 1, 1000, 128) == lib.attn_decode_workspace_size(2, 8, 2, 1000, 128)
    assert f(2, 8, 2, 4, 1000, 128) >= 4 * lib.attn_decode_workspace_size(2, 8, 2, 1000, 128) - 1024


def test_decode_paged_rejects(lib):
    f = lambda **kw: lib.attn_decode_paged(
        kw.get("q", A), A, A, kw.get("bt", A), A, A, None, 2, 8, 2, kw.get("Lq", 1), kw.get("n_pages", 16),
        kw.get("ps", 128), kw.get("mp", 8), 128, 0.1, A, 1 << 30, None)
    assert f(ps=96) == -1 and f(ps=0) == -1 and f(ps=-64) == -1
    assert f(n_pages=0) == -1 and f(mp=0) == -1
    assert f(bt=NULL) == -1
    assert f(Lq=0) == -1
    assert lib.attn_decode_paged_workspace_size(2, 8, 2, 1, 96, 8, 128) == 0
    assert lib.attn_decode_paged_workspace_size(2, 8, 2, 1, 128, 8, 128) == \
        lib.attn_decode_mq_workspace_size(2, 8, 2, 1, 1024, 128)


def _decode_kv8(lib, **kw):
    args = dict(q=A, k=A, v=A, ks=A, vs=A, fmt=1, sl=A, out=A, lse=NULL, B=2, Hq=8, Hkv=2, Lq=1, Lmax=64, D=128,
                scale=0.1, ws=A, wsb=1 << 30)
    args.update(kw)
    return lib.attn_decode_kv8(args["q"], args["k"], args["v"], args["ks"], args["vs"], args["fmt"], args["sl"],
                               args["out"], args["lse"], args["B"], args["Hq"], args["Hkv"], args["Lq"], args["Lmax"],
                               args["D"], args["scale"], args["ws"], args["wsb"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(fmt=0), -1), (dict(fmt=3), -1), (dict(ks=NULL), -1), (dict(vs=NULL), -1), (dict(Lq=0), -1),
    (dict(sl=NULL), -1), (dict(fmt=2, Lmax=66), -1), (dict(D=256), -2), (dict(D=96), -2),
    (dict(Hq=128, Hkv=1), -2), (dict(Lq=9, Hq=16), -2), (dict(ws=NULL), -3), (dict(wsb=64), -3),
])
def test_decode_kv8_rejects(lib, bad, code):
    assert _decode_kv8(lib, **bad) == code


def test_decode_kv8_empty_batch_and_workspace(lib):
    assert _decode_kv8(lib, B=0) == 0
    f = lib.attn_decode_kv8_workspace_size
    assert f(2, 8, 2, 1, 1000, 256) == 0 and f(2, 64, 1, 2, 1000, 128) == 0 and f(0, 8, 2, 1, 64, 128) == 0
    assert f(2, 8, 2, 1, 1000, 128) > 0 and f(2, 8, 2, 1, 1000, 128) % 256 == 0


def test_decode_kv8_paged_rejects(lib):
    f = lambda **kw: lib.attn_decode_kv8_paged(
        *[kw.get(n, d) for n, d in (("q", A), ("k", A), ("v", A), ("ks", A), ("vs", A), ("fmt", 1), ("bt", A),
                                    ("sl", A), ("out", A), ("lse", NULL), ("B", 2), ("Hq", 8), ("Hkv", 2), ("Lq", 1),
                                    ("n_pages", 10), ("page_size", 64), ("max_pages", 4), ("D", 128),
                                    ("scale", 0.1), ("ws", A), ("wsb", 1 << 30))], None)
    assert f(page_size=32) == -1 and f(page_size=100) == -1 and f(n_pages=0) == -1 and f(bt=NULL) == -1
    assert f(fmt=5) == -1 and f(D=256) == -2 and f(ws=NULL) == -3 and f(B=0) == 0
    w = lib.attn_decode_kv8_paged_workspace_size
    assert w(2, 8, 2, 1, 64, 4, 128) == lib.attn_decode_kv8_workspace_size(2, 8, 2, 1, 256, 128)
    assert w(2, 8, 2, 1, 100, 4, 128) == 0


def test_prefill_host_rejects(lib):
    f = lambda **kw: lib.attn_prefill_host(
        *[kw.get(n, d) for n, d in (("q", A), ("k", A), ("v", A), ("out", A), ("lse", NULL), ("B", 2), ("Hq", 8),
                                    ("Hkv", 2), ("Lq", 64), ("Lk", 64), ("D", 128), ("scale", 0.1), ("causal", 1),
                                    ("ws", A), ("wsb", 1 << 30))], None)
    assert f(ws=NULL) == -3 and f(wsb=1024) == -3 and f(ws=ctypes.c_void_p(0x10010)) == -1
    assert f(D=96) == -2 and f(Hq=7) == -1 and f(B=0) == 0
    s = lib.attn_prefill_host_scratch_size
    assert s(2, 8, 2, 64, 64, 128) > 0 and s(2, 8, 2, 64, 64, 96) == 0 and s(0, 8, 2, 64, 64, 128) == 0


def test_prefill_ws_rejects(lib):
    f = lambda **kw: lib.attn_prefill_ws(*[kw.get(n, d) for n, d in (
        ("q", A), ("k", A), ("v", A), ("out", A), ("lse", NULL), ("B", 1), ("Hq", 8), ("Hkv", 2), ("Lq", 16),
        ("Lk", 16), ("D", 128), ("scale", 0.1), ("causal", 1), ("ws", NULL), ("wsb", 0))], None)
    assert f(ws=ctypes.c_void_p(0x10010), wsb=1024) == -1 and f(q=NULL) == -1 and f(Hq=7) == -1
    assert f(D=96) == -2 and f(B=0) == 0 and f(Lq=0) == 0
    s = lib.attn_prefill_workspace_size
    assert s(1, 8, 2, 16, 16, 96, 1) == 0 and s(0, 8, 2, 16, 16, 128, 1) == 0 and s(1, 8, 3, 16, 16, 128, 1) == 0


def test_decode_host_rejects(lib):
    f = lambda **kw: lib.attn_decode_host(*[kw.get(n, d) for n, d in (
        ("q", A), ("k", A), ("v", A), ("sl", A), ("out", A), ("lse", NULL), ("B", 2), ("Hq", 8), ("Hkv", 2),
        ("Lmax", 64), ("D", 128), ("scale", 0.1), ("ws", A), ("wsb", 1 << 30))], None)
    assert f(ws=NULL) == -3 and f(wsb=1024) == -3 and f(ws=ctypes.c_void_p(0x10010)) == -1
    assert f(q=NULL) == -1 and f(sl=NULL) == -1 and f(sl=ctypes.c_void_p(0x10002)) == -1 and f(Lmax=0) == -1
    assert f(D=96) == -2 and f(Hq=7) == -1 and f(Hq=256, Hkv=1) == -2 and f(B=0) == 0
    s = lib.attn_decode_host_workspace_size
    # the partials, then q, out, lse and seqlens, each rounded up to 256 bytes
    part = lib.attn_decode_workspace_size(2, 8, 2, 64, 128)
    up = lambda x: (x + 255) // 256 * 256
    assert s(2, 8, 2, 64, 128) == up(part) + 2 * up(2 * 8 * 128 * 2) + up(2 * 8 * 4) + up(2 * 4)
    assert s(2, 8, 2, 64, 96) == 0 and s(0, 8, 2, 64, 128) == 0


def test_decode_partial_and_merge_reject(lib):
    m = lambda **kw: lib.attn_decode_merge(*[kw.get(n, d) for n, d in (("o", A), ("l", A), ("n", 2), ("rows", 8),
                                                                        ("D", 128), ("out", A), ("lse", NULL))], None)
    assert m(n=0) == -1 and m(rows=-1) == -1 and m(D=96) == -2 and m(rows=0) == 0 and m(o=NULL) == -1
    assert m(o=ctypes.c_void_p(0x10008)) == -1
    p = lambda **kw: lib.attn_decode_partial(*[kw.get(n, d) for n, d in (
        ("q", A), ("k", A), ("v", A), ("sl", A), ("o", A), ("l", A), ("B", 2), ("Hq", 8), ("Hkv", 2), ("Lmax", 64),
        ("D", 128), ("scale", 0.1), ("ws", A), ("wsb", 1 << 30))], None)
    assert p(l=NULL) == -1 and p(D=96) == -2 and p(ws=NULL) == -3 and p(B=0) == 0


def test_decode_noalloc_rejects_before_any_gpu_work(lib):
    """The no-alloc decode shares attn_decode's checks, and refuses sizes whose
    partials do not fit its static scratch before it looks the scratch up."""
    f = lambda **kw: lib.attn_decode_noalloc(*[kw.get(n, d) for n, d in (
        ("q", A), ("k", A), ("v", A), ("sl", A), ("out", A), ("lse", NULL), ("B", 2), ("Hq", 8), ("Hkv", 2),
        ("Lmax", 64), ("D", 128), ("scale", 0.1))], None)
    assert f(sl=NULL) == -1 and f(Lmax=0) == -1 and f(Hq=5) == -1 and f(k=NULL) == -1 and f(scale=0.0) == -1
    assert f(D=96) == -2 and f(Hq=256, Hkv=1) == -2
    assert f(B=0) == 0
    # Hq 64 at 131072 cached rows for 64 sequences: far more partials than the 16 MiB scratch
    assert lib.attn_decode_workspace_size(64, 64, 8, 131072, 128) > _native.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    assert f(B=64, Hq=64, Hkv=8, Lmax=131072) == -3
    assert b"static scratch" in lib.attn_last_error()


def test_diagnostics_reject(lib):
    assert lib.attn_selftest_wait(0, A, None) == -1
    assert lib.attn_selftest_wait(1000, NULL, None) == -1
    assert lib.attn_selftest_wait(3_000_000_000, A, None) == -1
    assert lib.attn_prefill_sched_busy(None) == -1


def test_fused_merge_calls_reject(lib):
    assert lib.attn_kvp_signal(NULL, 2, 1, None) == -1
    assert lib.attn_kvp_signal(NULL, 0, 1, None) == 0
    assert lib.attn_kvp_wait(NULL, 2, 1, None) == -1
    assert lib.attn_kvp_wait(ctypes.c_void_p(0x10002), 2, 1, None) == -1
    f = lambda **kw: lib.attn_decode_merge_peers(*[kw.get(n, d) for n, d in (
        ("o", A), ("l", A), ("r", A), ("v", 1), ("n", 2), ("rows", 8), ("D", 128), ("out", A), ("lse", NULL))], None)
    assert f(n=0) == -1 and f(rows=-1) == -1 and f(D=96) == -2 and f(rows=0) == 0
    assert f(o=NULL) == -1 and f(r=NULL) == -1 and f(out=ctypes.c_void_p(0x10008)) == -1
