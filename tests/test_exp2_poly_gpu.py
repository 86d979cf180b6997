"""The attention softmax evaluates part of its exponentials with the
library's own polynomial 2^x on the FMA pipe (dd_device.cuh: exp2_poly2).
Checked against CUDA's exp2f: relative error <= 1e-4 on [-125, 8] (the
products are rounded to bf16, whose spacing is 2^-8), and tiny, finite,
non-negative values where inputs are clamped."""
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_exp2_poly_against_exp2f(tmp_path):
    exe = str(tmp_path / "exp2_poly_check")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I" + os.path.join(ROOT, "block_discrete_diffusion_dd_b200", "csrc"),
                    "-o", exe, os.path.join(HERE, "helpers", "exp2_poly_check.cu")], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    maxrel = float(out[1])
    clamp = [float(v) for v in out[3:7]]
    assert maxrel <= 1e-4, maxrel
    assert all(0.0 <= v < 1e-37 for v in clamp[:3]), clamp
    assert abs(clamp[3] - 1.0) <= 1e-4
