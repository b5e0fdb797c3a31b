"""GPU parity of attention with an additive score bias (fa_fwd_bias) against the oracle.

The bias is added to the scaled scores (-inf removes a key); rows left with
no key must come back as O = 0, LSE = -inf.  Tolerances as for the other
forward parity tests.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import tiled_attention_15_b200 as fa
from fa_inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu

TOL = {"fp16": (4e-3, 1e-3), "bf16": (1.6e-2, 1e-3)}
TD = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _bias(w, shape, seed, scale=2.0, neg_inf_frac=0.0):
    rng = np.random.default_rng(seed)
    b = (scale * rng.standard_normal(shape)).astype(np.float32)
    if neg_inf_frac > 0:
        b[rng.random(shape) < neg_inf_frac] = -np.inf
    return torch.from_numpy(b).to(TD[w.dtype])


def _check(w, bias, dev, tag="", window=(-1, -1)):
    q, k, v = make_qkv(w)
    o, lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), scale=w.softmax_scale, causal=w.causal,
                       bias=bias.to(dev), window=window)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, w.causal, bias=bias.float(),
                                    window=window)
    got_o, got_l = o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy()
    empty = np.isneginf(ref_l)
    np.testing.assert_array_equal(np.isneginf(got_l), empty)
    assert np.all(got_o[empty] == 0.0) and np.isfinite(got_o).all()
    do = np.abs(got_o - ref_o).max()
    dl = np.abs(got_l[~empty] - ref_l[~empty]).max() if (~empty).any() else 0.0
    report = os.environ.get("FA_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"case": f"bias {w.name}{tag}", "dtype": w.dtype,
                                "max_abs_dO": float(do), "max_abs_dLSE": float(dl)}) + "\n")
    to, tl = TOL[w.dtype]
    assert do <= to, f"{w.name}: max|dO| = {do:.3e}"
    assert dl <= tl, f"{w.name}: max|dLSE| = {dl:.3e}"
    return o, lse


def test_full_bias_fp16(cuda_dev):
    w = Workload("full [B,H,Nq,Nk] D128 fp16", 2, 4, 2, 300, 333, 128, "fp16", False, seed=111)
    _check(w, _bias(w, (2, 4, 300, 333), 1), cuda_dev)


def test_broadcast_bias_causal_bf16(cuda_dev):
    w = Workload("shared [Nq,Nk] D64 bf16 causal", 2, 3, 3, 700, 700, 64, "bf16", True, seed=112)
    _check(w, _bias(w, (1, 1, 700, 700), 2), cuda_dev)


def test_key_padding_mask(cuda_dev):
    # [B, 1, 1, Nk]: one bias row for every query (broadcast over queries and heads)
    w = Workload("key padding [B,1,1,Nk] D128 fp16", 2, 4, 4, 200, 333, 128, "fp16", False, seed=113)
    b = torch.zeros(2, 1, 1, 333)
    b[0, :, :, 250:] = -float("inf")
    b[1, :, :, 100:] = -float("inf")
    _check(w, b.half(), cuda_dev)


def test_per_head_bias_d256(cuda_dev):
    w = Workload("per head [1,H,Nq,Nk] D256 bf16", 2, 4, 1, 256, 512, 256, "bf16", False, seed=114)
    _check(w, _bias(w, (1, 4, 256, 512), 3), cuda_dev)


def test_bias_removes_whole_rows(cuda_dev):
    w = Workload("empty rows D64 fp16", 1, 2, 2, 150, 260, 64, "fp16", False, seed=115)
    b = _bias(w, (1, 2, 150, 260), 4, neg_inf_frac=0.3)
    b[0, 0, 7, :] = -float("inf")
    b[0, 1, 140:, :] = -float("inf")
    _check(w, b, cuda_dev)


def test_large_bias_values(cuda_dev):
    # +-30 bias: the running max moves by large steps between blocks (rescales)
    w = Workload("large bias D128 bf16", 1, 2, 2, 400, 1000, 128, "bf16", False, seed=116)
    _check(w, _bias(w, (1, 2, 400, 1000), 5, scale=30.0), cuda_dev)


def test_zero_bias_equals_no_bias(cuda_dev):
    w = Workload("zero bias D128 fp16", 1, 2, 2, 300, 300, 128, "fp16", True, seed=117)
    o, lse = _check(w, torch.zeros(1, 1, 1, 300, dtype=torch.float16), cuda_dev)
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    o2, lse2 = fa.fa_fwd(q, k, v, scale=w.softmax_scale, causal=True, use_workspace=False)
    torch.cuda.synchronize()
    assert (o.float() - o2.float()).abs().max().item() <= 2e-3
    assert (lse - lse2).abs().max().item() <= 1e-5


def test_unaligned_key_count_is_padded(cuda_dev):
    # Nk = 77: the binding copies the bias into rows padded to 80 keys
    w = Workload("Nk 77 D64 fp16", 1, 2, 2, 90, 77, 64, "fp16", False, seed=118)
    _check(w, _bias(w, (1, 2, 90, 77), 6), cuda_dev)


def test_bias_many_tiles_per_cta(cuda_dev):
    # two-query-tile bias kernel over several work tiles per CTA (CTA cap 8):
    # the bias producer and the softmax warps stay in step across units
    w = Workload("shared [N,N] D128 fp16 many tiles", 2, 8, 8, 1024, 1024, 128, "fp16", False,
                 seed=119)
    prev = fa.set_max_ctas(8)
    try:
        _check(w, _bias(w, (1, 1, 1024, 1024), 7), cuda_dev)
        wc = w.with_(name="per head [1,H,N,N] D64 bf16 causal many tiles", D=64, dtype="bf16",
                     causal=True, seed=120)
        _check(wc, _bias(wc, (1, 8, 1024, 1024), 8), cuda_dev)
    finally:
        fa.set_max_ctas(prev)


# ---- key window and score bias in one call (fa_fwd_bias_window)

def test_window_and_bias_causal_sliding(cuda_dev):
    # causal sliding window of 200 keys over three 128-row tiles and a ragged tail,
    # with a full [B, H, Nq, Nk] bias
    w = Workload("window 200 causal + full bias D128 fp16", 1, 4, 2, 600, 600, 128, "fp16", True,
                 seed=121)
    _check(w, _bias(w, (1, 4, 600, 600), 9), cuda_dev, " window", window=(200, -1))


def test_window_and_bias_two_sided_padding_mask(cuda_dev):
    # two-sided window (37 left, 19 right) with a key-padding mask of -inf and
    # per-key values, broadcast over heads and queries
    w = Workload("window 37/19 + padding mask D64 bf16", 2, 4, 4, 300, 320, 64, "bf16", False,
                 seed=122)
    b = _bias(w, (2, 1, 1, 320), 10, neg_inf_frac=0.2)
    _check(w, b, cuda_dev, " window", window=(37, 19))


def test_window_and_bias_rows_without_keys(cuda_dev):
    # window (0, 0): query i sees key i only; rows i >= Nk see nothing, and a
    # bias of -inf on some keys empties their rows too: O = 0, LSE = -inf there
    w = Workload("window 0/0 + -inf bias D128 fp16", 1, 2, 2, 260, 200, 128, "fp16", False,
                 seed=123)
    b = _bias(w, (1, 2, 260, 200), 11, neg_inf_frac=0.3)
    o, lse = _check(w, b, cuda_dev, " window", window=(0, 0))
    assert torch.isneginf(lse[:, :, 200:]).all()


def test_window_and_bias_d256_per_head(cuda_dev):
    w = Workload("window 96 causal + per-head bias D256 bf16", 1, 4, 1, 400, 400, 256, "bf16",
                 True, seed=124)
    _check(w, _bias(w, (1, 4, 400, 400), 12), cuda_dev, " window", window=(96, -1))


# ---- split tail and dynamic schedule with a bias (fa_fwd_bias_ws)

def test_bias_split_tail_and_removed_rows(cuda_dev):
    # 20 tiles of 256 rows on 16 CTAs: the last 4 tiles are split over two CTAs
    # each (8 key blocks -> two halves) and merged.  Rows 300..339 of head 0 lose
    # every key; rows 600..639 lose exactly the first half of the keys (one part
    # of their split tile sees no key) and rows 700..739 the second half.
    w = Workload("split tail + removed rows D128 fp16", 1, 5, 5, 1024, 1024, 128, "fp16", False,
                 seed=125)
    b = 2.0 * np.random.default_rng(13).standard_normal((1, 5, 1024, 1024)).astype(np.float32)
    b[0, 0, 300:340, :] = -np.inf
    b[0, 4, 600:640, :512] = -np.inf
    b[0, 4, 700:740, 512:] = -np.inf
    bias = torch.from_numpy(b).half()
    prev = fa.set_max_ctas(16)
    try:
        o, lse = _check(w, bias, cuda_dev, " split")
        assert torch.isneginf(lse[0, 0, 300:340]).all() and (o[0, 0, 300:340] == 0).all()
        wb = w.with_(name="split tail shared [N,N] bias D64 bf16", D=64, dtype="bf16", seed=126)
        _check(wb, _bias(wb, (1, 1, 1024, 1024), 14), cuda_dev, " split")
    finally:
        fa.set_max_ctas(prev)


def test_bias_workspace_matches_no_workspace(cuda_dev):
    # the dynamic schedule does not change a unit's arithmetic: bit-identical
    # to the static order (no split: 8 tiles on 8 CTAs per round)
    w = Workload("bias ws vs none D128 bf16", 2, 4, 4, 512, 700, 128, "bf16", False, seed=127)
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    bias = _bias(w, (2, 4, 512, 700), 15).to(cuda_dev)
    prev = fa.set_max_ctas(5)
    try:
        a = fa.fa_fwd(q, k, v, scale=w.softmax_scale, bias=bias)
        b_ = fa.fa_fwd(q, k, v, scale=w.softmax_scale, bias=bias, use_workspace=False)
    finally:
        fa.set_max_ctas(prev)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b_[0]) and torch.equal(a[1], b_[1])


def test_window_and_bias_dynamic_schedule(cuda_dev):
    # windowed bias launches (one-query-tile bias kernel) on 4 CTAs: 20 units go
    # through the dynamic schedule's ring, with the bias tiles loaded beside K/V;
    # the result equals the static order bit for bit
    w = Workload("window 150 + bias D128 fp16, 4 CTAs", 1, 4, 2, 600, 600, 128, "fp16", True,
                 seed=128)
    b = _bias(w, (1, 4, 600, 600), 16)
    prev = fa.set_max_ctas(4)
    try:
        o, lse = _check(w, b, cuda_dev, " window dynamic", window=(150, -1))
        q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
        o2, lse2 = fa.fa_fwd(q, k, v, scale=w.softmax_scale, causal=True, window=(150, -1),
                             bias=b.to(cuda_dev), use_workspace=False)
    finally:
        fa.set_max_ctas(prev)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
