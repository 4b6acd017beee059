"""The FMA-pipe exp2, softplus and silu of csrc/common.cuh against fp64 and
CUDA's exp2f (compiled into a small checker, run on the GPU)."""

import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_causal_b200", "csrc")

pytestmark = pytest.mark.gpu


def test_fastmath_accuracy(tmp_path):
    exe = os.path.join(tmp_path, "fastmath_check")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", CSRC, "-o", exe, os.path.join(ROOT, "tests", "cuda", "fastmath_check.cu")],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    vals = {m.group(1): float(m.group(2)) for m in re.finditer(r"^(\w+) max_rel ([0-9.e+-]+)", out, re.M)}
    cuda_exp2 = float(re.search(r"CUDA exp2f max_rel ([0-9.e+-]+)", out).group(1))
    # within a few ulp: no worse than 4e-7 relative, and within 4x CUDA's exp2f
    assert vals["exp2_fma2"] <= 4e-7, out
    assert vals["exp2_fma2"] <= 4 * max(cuda_exp2, 1.2e-7), out
    # Both go through 2^(x * log2 e); rounding that product to fp32 alone costs
    # up to |x| * log2(e) * 2^-24 * ln 2 relative (1.2e-6 at |x| = 20, 5e-6 at
    # |x| = 85). |x| <= 20 covers every delta and gate input of the workloads.
    assert vals["softplus2_core"] <= 2e-6, out
    assert vals["silu2_core"] <= 2e-6, out
    assert vals["softplus2"] <= 1e-5, out
    assert vals["silu2"] <= 1e-5, out
    assert "status no error" in out
