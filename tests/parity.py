"""Shared comparison for the GPU parity tests (CUDA result vs the fp64 oracle).

Tolerances (fixed before any kernel ran): bf16 inputs, fp32 accumulation and
a bf16 output must agree with the exact result to
    O   : max |err| <= 2e-2 and ||err||_2 / ||ref||_2 <= 5e-3
    LSE : max |err| <= 1e-3 (fp32 natural log)
Rows that see no key must give O == 0 exactly and LSE == -inf.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    o = to_f64(out_gpu)
    assert o.shape == out_ref.shape, (o.shape, out_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - out_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(out_ref))
    rel = float(np.linalg.norm(o - out_ref)) / denom if denom > 0 else float(np.linalg.norm(o))
    assert max_abs <= O_MAX_ABS, f"{what}: O max abs err {max_abs:.3e}"
    assert rel <= O_REL_L2, f"{what}: O rel L2 err {rel:.3e}"
    if lse_gpu is not None:
        l = to_f64(lse_gpu)
        assert l.shape == lse_ref.shape
        ninf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(l), ninf_ref), f"{what}: -inf LSE rows differ"
        if (~ninf_ref).any():
            lerr = float(np.abs(l[~ninf_ref] - lse_ref[~ninf_ref]).max())
            assert lerr <= LSE_MAX_ABS, f"{what}: LSE max abs err {lerr:.3e}"
        if ninf_ref.any():
            assert np.all(o[ninf_ref] == 0.0), f"{what}: rows without keys must be 0"
    return max_abs, rel
