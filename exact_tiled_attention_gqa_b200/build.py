"""Build the sm_100a library in-tree: ``python -m exact_tiled_attention_gqa_b200.build``.

One translation unit (csrc/attn_gqa.cu) compiled by nvcc for sm_100a only into
``libattn_gqa_sm100.so`` next to this file.  The runtime is linked statically,
and cuTensorMapEncodeTiled is fetched through the runtime's driver entry point,
so the library needs nothing beyond the CUDA driver at load time.
"""
from __future__ import annotations

import glob
import os
import re
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
LIB_NAME = "libattn_gqa_sm100.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
# The same sources built with -DATTN_DEBUG_BOUNDS=1: the kernels check their
# unit mapping, ring positions, TMA coordinates and output indices and report a
# violation as ATTN_DEVERR_BOUNDS (a checking build for tests, not for speed).
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libattn_gqa_sm100_debug_bounds.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(ROOT, "include", "attn_gqa.h")])


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(s) <= t for s in sources())


# The prefill kernel launches with this many registers per thread and then
# moves registers between its warpgroups with setmaxnreg; the exchange only
# balances if the compiled count is exactly this (see prefill_sm100.cuh).
PREFILL_LAUNCH_REGS = 168


def check_ptxas_report(report: str) -> dict:
    """Parse `-Xptxas -v` output: {kernel: (registers, spill_bytes)}; enforce the prefill register count."""
    kernels, current = {}, None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and current:
            kernels.setdefault(current, [0, 0])[1] = int(m.group(1))
        m = re.search(r"Used (\d+) registers", line)
        if m and current:
            kernels.setdefault(current, [0, 0])[0] = int(m.group(1))
    # the kernels with two Q tiles per CTA exchange registers with setmaxnreg
    prefill = {k: v for k, v in kernels.items() if re.search(r"attn_prefill_sm100_kernelILi\d+ELi2E", k)}
    if not prefill:
        raise RuntimeError("ptxas report has no prefill kernel entry")
    for name, (regs, _) in prefill.items():
        if regs != PREFILL_LAUNCH_REGS:
            raise RuntimeError(f"{name} compiled to {regs} registers, expected exactly {PREFILL_LAUNCH_REGS}: "
                               "the setmaxnreg exchange would not balance")
    return {k: tuple(v) for k, v in kernels.items()}


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    path = DEBUG_LIB_PATH if debug_bounds else LIB_PATH
    if not force and up_to_date(path):
        return path
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-std=c++17", "-O3", "-lineinfo", *ARCH_FLAGS, "-Xcompiler", "-fPIC", "-shared",
           "-Xptxas", "-v", *(["-DATTN_DEBUG_BOUNDS=1"] if debug_bounds else []),
           os.path.join(CSRC, "attn_gqa.cu"), "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
    try:
        kernels = check_ptxas_report(res.stdout + res.stderr)
    except RuntimeError:
        os.remove(tmp)
        raise
    if verbose:
        for name, (regs, spill) in sorted(kernels.items()):
            print(f"{regs:4d} regs {spill:6d} B spill  {name}")
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
