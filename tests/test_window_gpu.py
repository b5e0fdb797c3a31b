"""GPU parity of key-window attention (fa_fwd_window) against the oracle.

Query i sees keys i - left .. i + right (-1: unbounded on that side); causal
fixes right = 0.  Rows that see no key must come back as O = 0, LSE = -inf.
Tolerances as for the other parity tests.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import tiled_attention_15_b200 as fa
from fa_inputs import Workload, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

TOL = {"fp16": (4e-3, 1e-3), "bf16": (1.6e-2, 1e-3)}


def _run(w, window, dev, use_ws=True):
    q, k, v = make_qkv(w)
    o, lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), scale=w.softmax_scale, causal=w.causal,
                       window=window, use_workspace=use_ws)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    return (q, k, v), o, lse


def _check(w, window, got_o, got_l, ref_o, ref_l, tag=""):
    got_o = got_o.astype(np.float64)
    empty = np.isneginf(ref_l)
    np.testing.assert_array_equal(np.isneginf(got_l), empty)
    assert np.all(got_o[empty] == 0.0)
    assert np.isfinite(got_o).all()
    do = np.abs(got_o - ref_o).max()
    dl = np.abs(got_l[~empty] - ref_l[~empty]).max() if (~empty).any() else 0.0
    report = os.environ.get("FA_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"case": f"{w.name} window {window}{tag}", "dtype": w.dtype,
                                "max_abs_dO": float(do), "max_abs_dLSE": float(dl)}) + "\n")
    to, tl = TOL[w.dtype]
    assert do <= to, f"{w.name}: max|dO| = {do:.3e}"
    assert dl <= tl, f"{w.name}: max|dLSE| = {dl:.3e}"


WINDOWS = [
    (Workload("causal sliding D128 fp16", 1, 4, 2, 2000, 2000, 128, "fp16", True, seed=71), (255, -1)),
    (Workload("local D64 bf16", 2, 3, 3, 777, 777, 64, "bf16", False, seed=72), (100, 50)),
    (Workload("narrow D128 fp16", 1, 2, 2, 600, 600, 128, "fp16", False, seed=73), (5, 3)),
    (Workload("left only D256 bf16 Nq<Nk", 1, 2, 1, 300, 1000, 256, "bf16", False, seed=74), (200, -1)),
    (Workload("right only D128 fp16", 1, 2, 2, 500, 500, 128, "fp16", False, seed=75), (-1, 64)),
    (Workload("empty rows D64 fp16", 1, 2, 2, 700, 300, 64, "fp16", False, seed=76), (100, 10)),
    (Workload("causal = (-1,0) D128 bf16", 1, 2, 2, 513, 513, 128, "bf16", True, seed=77), (-1, 0)),
    (Workload("wide = none D64 fp16 GQA", 2, 8, 2, 300, 400, 64, "fp16", False, seed=78), (1000, 1000)),
    (Workload("causal window 128 D256 fp16", 1, 2, 2, 640, 640, 256, "fp16", True, seed=79), (128, 0)),
]


@pytest.mark.parametrize("use_ws", [True, False])
@pytest.mark.parametrize("w,window", WINDOWS, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_window_parity(cuda_dev, w, window, use_ws):
    (q, k, v), o, lse = _run(w, window, cuda_dev, use_ws)
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, w.causal, window=window)
    _check(w, window, o.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l,
           "" if use_ws else " nows")


def test_zero_window_returns_values(cuda_dev):
    # each query sees only its own key: P = 1, O = V exactly
    w = Workload("own value", 1, 2, 2, 300, 300, 128, "bf16", False, seed=80)
    (q, k, v), o, lse = _run(w, (0, 0), cuda_dev)
    assert torch.equal(o.cpu(), v)
    s = w.softmax_scale * (q.double() * k.double()).sum(-1)
    np.testing.assert_allclose(lse.cpu().double().numpy(), s.numpy(), rtol=0, atol=1e-4)


def test_window_long_sampled(cuda_dev):
    # a sliding-window shape at full length: causal, 1024-key window, 8192 positions
    w = Workload("sliding 1024 N8192 D128 fp16", 1, 8, 2, 8192, 8192, 128, "fp16", True, seed=81)
    (q, k, v), o, lse = _run(w, (1023, -1), cuda_dev)
    rows = sample_rows(w.Nq, 96, seed=5)
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, True, rows=rows, window=(1023, -1))
    _check(w, (1023, -1), o.float().cpu().numpy()[:, :, rows], lse.cpu().numpy()[:, :, rows],
           ref_o, ref_l)


def test_window_deterministic(cuda_dev):
    w = Workload("det window", 1, 4, 2, 1000, 1200, 128, "bf16", False, seed=82)
    (_, _, _), o1, l1 = _run(w, (300, 20), cuda_dev)
    (_, _, _), o2, l2 = _run(w, (300, 20), cuda_dev)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
