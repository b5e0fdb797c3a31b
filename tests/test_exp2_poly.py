"""The FMA-pipe exp2 the softmax uses for part of its exponentials.

CPU: the coefficients in sm100_ptx.cuh are the linear-programming minimax fit that
fit_exp2_poly.py produces, and their float32 Horner evaluation meets the
stated 1.02e-4 relative-error bound against 2^f computed in float64.
GPU: the kernel-side evaluation (range reduction + polynomial + exponent add)
matches float64 2^x within the same bound over the range the softmax uses.
"""
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "tiled_attention_15_b200", "csrc", "sm100_ptx.cuh")
FIT = os.path.join(ROOT, "tiled_attention_15_b200", "csrc", "fit_exp2_poly.py")
BOUND = 1.02e-4


def _coefs():
    txt = open(HDR).read()
    return [1.0] + [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", txt).group(1)) for i in (1, 2, 3)]


def test_coefficients_come_from_the_fit():
    out = subprocess.run([sys.executable, FIT], capture_output=True, text=True, check=True).stdout
    fitted = [float(v) for v in re.search(r"coefs \[(.*)\]", out).group(1).split(",")]
    assert np.allclose(fitted, _coefs(), rtol=0, atol=1e-7)


def test_polynomial_bound_float32():
    c = np.array(_coefs(), dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    p = c[3]
    for k in (2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() <= BOUND


@pytest.mark.gpu
def test_gpu_exp2_fma(cuda_dev):
    import torch
    import tiled_attention_15_b200 as fa
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 1.0, 7.25])])
    y = fa.exp2_fma(x.to(cuda_dev)).cpu().double().numpy()
    want = np.exp2(x.double().numpy())
    rel = np.abs(y / want - 1.0)
    assert rel.max() <= BOUND, rel.max()
    # exact at integers (p(0) = 1): 2^0 = 1, 2^1 = 2, 2^-3 = 1/8
    e = fa.exp2_fma(torch.tensor([0.0, 1.0, -3.0, 7.0], device=cuda_dev)).cpu().numpy()
    assert e.tolist() == [1.0, 2.0, 0.125, 128.0]
    # below the clamp the result is ~2^-125, never negative, NaN or huge
    z = fa.exp2_fma(torch.tensor([-126.0, -500.0, float("-inf")], device=cuda_dev)).cpu().numpy()
    assert np.all(z >= 0) and np.all(z < 1e-37)
