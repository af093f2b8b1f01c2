"""The bounds-checking build: the same sources compiled with -DATTN_DEBUG_BOUNDS=1,
whose kernels check their work-unit mapping, ring positions, TMA coordinates and
output indices and report a violation in the device error word (they never trap).
Small parity cases for every kernel family, persistent prefills whose units run
in bands of KV groups, and prefills with a key-split tail go through it in a child
process; each must match the
oracle with the error word clear."""
import os
import subprocess
import sys

import pytest
import torch

from exact_tiled_attention_gqa_b200 import build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_bounds_build_passes_parity_with_clean_error_word():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    path = build.build(debug_bounds=True)
    assert os.path.exists(path)
    env = dict(os.environ, ATTN_GQA_DEBUG_BOUNDS="1")
    res = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_cases.py")], env=env,
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    assert "debug-bounds cases passed" in res.stdout
