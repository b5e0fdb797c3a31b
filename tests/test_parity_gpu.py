"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small and ragged shapes, the LLaMA-7B layer (all four variants) and the
sequence sweep up to N=4096 (all four seeds) are compared on every output
element.  The largest workloads -- the sweep at N=8192, the GQA/MQA and
head-dim sweep at N=8192 and the 128K context -- are compared on seeded
samples of query rows (every head, rows 0 and N-1 always included), plus
properties that hold at any size.

Tolerances (max abs difference against the fp64 oracle): fp16 inputs O 4e-3
and LSE 1e-3; bf16 inputs O 1.6e-2 and LSE 1e-3.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import tiled_attention_15_b200 as fa
from fa_inputs import (SWEEP_SEEDS, TINY, LONG, Workload, gqa, llama7b, make_qkv, sample_rows,
                       seq_sweep)

pytestmark = pytest.mark.gpu

TOL = {"fp16": (4e-3, 1e-3), "bf16": (1.6e-2, 1e-3)}


def run_cuda(w: Workload, dev, q=None, k=None, v=None):
    if q is None:
        q, k, v = make_qkv(w)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    o, lse = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    return (q, k, v), o, lse


def compare(w: Workload, dev, rows=None):
    (q, k, v), o, lse = run_cuda(w, dev)
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, w.causal, rows=rows)
    got_o = o.float().cpu().numpy().astype(np.float64)
    got_l = lse.cpu().numpy().astype(np.float64)
    if rows is not None:
        got_o, got_l = got_o[:, :, rows], got_l[:, :, rows]
    assert np.isfinite(got_o).all() and np.isfinite(got_l).all()
    to, tl = TOL[w.dtype]
    do = np.abs(got_o - ref_o).max()
    dl = np.abs(got_l - ref_l).max()
    report = os.environ.get("FA_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"case": w.name, "dtype": w.dtype, "rows": "all" if rows is None
                                else len(rows), "max_abs_dO": do, "max_abs_dLSE": dl}) + "\n")
    assert do <= to, f"{w.name}: max|dO| = {do:.3e} > {to}"
    assert dl <= tl, f"{w.name}: max|dLSE| = {dl:.3e} > {tl}"
    return o, lse, (q, k, v), do, dl


# ------------------------------------------------------------ every element
def test_tiny_config(cuda_dev):
    compare(TINY, cuda_dev)


EDGE = []
for D in (64, 128, 256):
    for nq, nk in ((1, 1), (17, 17), (127, 127), (129, 129), (255, 300), (300, 255), (513, 513),
                   (1, 700), (700, 1)):
        for causal in (False, True):
            EDGE.append(Workload(f"edge D{D} {nq}x{nk} {'c' if causal else 'nc'}", 1, 2, 1, nq, nk,
                                 D, "fp16", causal, seed=nq + nk + D))


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_ragged_shapes(cuda_dev, w):
    compare(w, cuda_dev)


MIXED = [
    Workload("bf16 D128 GQA4 B2", 2, 8, 2, 384, 384, 128, "bf16", True, seed=11),
    Workload("bf16 D64 MQA", 1, 4, 1, 640, 640, 64, "bf16", False, seed=12),
    Workload("bf16 D256 GQA", 1, 4, 2, 520, 520, 256, "bf16", True, seed=13),
    Workload("fp16 D128 peaky", 1, 2, 2, 1024, 1024, 128, "fp16", False, seed=14, q_mult=4.0),
    Workload("fp16 D256 peaky causal", 1, 2, 1, 700, 700, 256, "fp16", True, seed=15, q_mult=4.0),
    Workload("bf16 D128 outliers", 1, 2, 1, 1000, 1000, 128, "bf16", True, seed=16,
             outlier_frac=0.01),
    Workload("fp16 D64 many tiles", 3, 5, 5, 1100, 900, 64, "fp16", True, seed=17),
]


# Several tiles per CTA with D = 256 and long causal rows: a softmax warp can
# run a key block ahead of the others there (regression: per-buffer P barriers).
def test_d256_multi_tile_causal(cuda_dev):
    _full(Workload("fp16 D256 B2 H16 N2048 causal", 2, 16, 16, 2048, 2048, 256, "fp16", True,
                   seed=4), 64, cuda_dev)


@pytest.mark.parametrize("w", MIXED, ids=lambda w: w.name)
def test_mixed(cuda_dev, w):
    compare(w, cuda_dev)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("D", [64, 128, 256])
def test_single_visible_key_is_exact(cuda_dev, dtype, D):
    """A row that sees one key has softmax weight exactly 1: O must equal that V row bit
    for bit.  Holds for every row when Nk = 1 and for row 0 under causal masking, for
    positive and negative scores alike (a wrong row max shows up here first)."""
    w = Workload("nk1", 2, 4, 2, 700, 1, D, dtype, False, seed=21)
    (q, k, v), o, _ = run_cuda(w, cuda_dev)
    want = v[:, :, 0].repeat_interleave(2, dim=1)[:, :, None, :].expand(-1, -1, 700, -1)
    assert torch.equal(o.cpu(), want.contiguous())
    wc = Workload("c-row0", 2, 4, 2, 300, 300, D, dtype, True, seed=22, q_mult=3.0)
    (q, k, v), o, _ = run_cuda(wc, cuda_dev)
    assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0].repeat_interleave(2, dim=1))


# Split tails: with the CTA cap at 8, these shapes leave a last round of at most 4 work
# tiles, which the workspace path gives to two CTAs each (one per half of the key
# blocks) and merges.  Ragged query/key lengths and an odd number of key blocks included.
# (Splitting needs at least 24 key blocks of 128, so Nk >= 2945 here.)
SPLIT = [
    Workload("split D128 fp16", 1, 5, 5, 512, 3072, 128, "fp16", False, seed=31),
    Workload("split D128 bf16 GQA ragged", 1, 10, 5, 300, 3500, 128, "bf16", False, seed=32),
    Workload("split D64 fp16 odd blocks", 2, 5, 5, 256, 3201, 64, "fp16", False, seed=33),
    Workload("split D256 bf16", 1, 5, 5, 512, 3072, 256, "bf16", False, seed=34),
    Workload("split D256 fp16 ragged", 1, 3, 1, 333, 4000, 256, "fp16", False, seed=35),
]


@pytest.mark.parametrize("w", SPLIT, ids=lambda w: w.name)
def test_split_tail(cuda_dev, w):
    tiles = fa.num_tiles(w.B, w.Hq, w.Nq, w.D)
    assert tiles > 8 and 0 < tiles % 8 <= 4  # the shape really exercises the split
    prev = fa.set_max_ctas(8)
    try:
        o1, l1, (q, k, v), _, _ = compare(w, cuda_dev)
        # a second call on the same workspace: counters were left at zero
        o2, l2 = fa.fa_fwd(q.to(cuda_dev), k.to(cuda_dev), v.to(cuda_dev), scale=w.softmax_scale)
        torch.cuda.synchronize()
        assert fa.device_status(reset=True) == 0
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        # and agrees with the no-workspace path within rounding
        o3, l3 = fa.fa_fwd(q.to(cuda_dev), k.to(cuda_dev), v.to(cuda_dev), scale=w.softmax_scale,
                           use_workspace=False)
        torch.cuda.synchronize()
        tol = TOL[w.dtype][0]
        assert (o1.float() - o3.float()).abs().max().item() <= tol
        assert (l1 - l3).abs().max().item() <= 1e-4
    finally:
        fa.set_max_ctas(prev)


# KV-cache decode shapes: a few query rows per head against a long key range.
# With Hq > Hkv and Hq/Hkv * Nq <= 128 one tile packs all query heads of a key/value
# head; with a workspace every tile's key range is also split across CTAs (split-K)
# when there are fewer tiles than SMs.
DECODE = [
    Workload("decode GQA4 Nq1 D128 fp16", 4, 32, 8, 1, 8192, 128, "fp16", False, seed=51),
    Workload("decode GQA4 Nq1 D128 bf16 ragged Nk", 2, 16, 4, 1, 5000, 128, "bf16", False, seed=52),
    Workload("decode GQA8 Nq4 D64 fp16", 2, 32, 4, 4, 4096, 64, "fp16", False, seed=53),
    Workload("decode MQA Nq2 D256 bf16", 2, 16, 1, 2, 3000, 256, "bf16", False, seed=54),
    Workload("decode GQA8 Nq16 D128 fp16 (128 rows)", 1, 16, 2, 16, 4096, 128, "fp16", False, seed=55),
    Workload("decode GQA8 Nq17 D128 fp16 (not packed)", 1, 8, 1, 17, 2048, 128, "fp16", False, seed=56),
    Workload("decode MHA Nq1 D128 fp16", 2, 16, 16, 1, 8192, 128, "fp16", False, seed=57),
    Workload("decode GQA4 Nq3 D128 fp16 short Nk", 1, 8, 2, 3, 300, 128, "fp16", False, seed=58),
]


# Stream-K: non-causal launches with fewer work tiles than SMs share the key
# blocks of all tiles out evenly over the CTAs; a tile is merged from the parts
# of every CTA whose range touched it.
STREAMK = [
    # one 128-row tile, 512 key blocks -> 128 CTAs of 4 blocks, 128 parts
    Workload("stream-K one tile 128 parts", 1, 1, 1, 128, 65536, 128, "fp16", False, seed=61),
    Workload("stream-K D256 bf16 ragged", 2, 4, 2, 200, 9000, 256, "bf16", False, seed=62),
    # 256-row tiles (two query tiles per work tile), D 64
    Workload("stream-K D64 256-row tiles", 1, 8, 8, 256, 12000, 64, "fp16", False, seed=63),
    Workload("stream-K ragged 130 rows bf16", 1, 3, 3, 130, 5000, 128, "bf16", False, seed=64),
]


@pytest.mark.parametrize("w", STREAMK, ids=lambda w: w.name)
def test_stream_k(cuda_dev, w):
    o1, l1, (q, k, v), _, _ = compare(w, cuda_dev)
    qd, kd, vd = (x.to(cuda_dev) for x in (q, k, v))
    # a second call on the same workspace: counters were left at zero, and the
    # fixed merge order gives the same bits
    o2, l2 = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("use_ws", [True, False])
@pytest.mark.parametrize("w", DECODE, ids=lambda w: w.name)
def test_decode_shapes(cuda_dev, w, use_ws):
    q, k, v = make_qkv(w)
    o, lse = fa.fa_fwd(q.to(cuda_dev), k.to(cuda_dev), v.to(cuda_dev), scale=w.softmax_scale,
                       use_workspace=use_ws)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, False)
    do = np.abs(o.float().cpu().numpy() - ref_o).max()
    dl = np.abs(lse.cpu().numpy() - ref_l).max()
    report = os.environ.get("FA_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"case": w.name + (" ws" if use_ws else " nows"), "dtype": w.dtype,
                                "rows": "all", "max_abs_dO": float(do), "max_abs_dLSE": float(dl)}) + "\n")
    assert do <= TOL[w.dtype][0], f"{w.name}: max|dO| = {do:.3e}"
    assert dl <= TOL[w.dtype][1], f"{w.name}: max|dLSE| = {dl:.3e}"


@pytest.mark.parametrize("scale", [0.0, -0.0883883, 0.5])
def test_scale_values(cuda_dev, scale):
    w = Workload("scale", 1, 2, 2, 300, 300, 128, "fp16", True, seed=3, scale=scale)
    o, lse, (q, k, v), _, _ = compare(w, cuda_dev)
    if scale == 0.0:  # uniform average over the visible prefix
        n = torch.arange(1, 301, dtype=torch.float64)
        np.testing.assert_allclose(lse.cpu().double().numpy(), np.log(n.numpy())[None, None].repeat(2, 1),
                                   atol=1e-5)


@pytest.mark.parametrize("scale", [0.0, -0.0883883])
def test_scale_values_two_tile_kernel(cuda_dev, scale):
    # enough 256-row tiles for the two-query-tile kernel, whose causal diagonal
    # blocks keep fp16 scores unscaled with -inf * sign(scale) at masked keys
    # (scale 0 takes the scaled form)
    w = Workload("scale two-tile", 2, 40, 40, 600, 600, 128, "fp16", True, seed=6, scale=scale)
    assert 2 * fa.num_tiles(w.B, w.Hq, w.Nq, w.D) >= 148
    compare(w, cuda_dev)


# fp16 without a mask over at most 4096 keys runs the staged epilogue (output
# rows through shared memory, written as whole lines); one key more runs the
# plain one.  600 query rows: the last 256-row tile holds 88 live rows.
@pytest.mark.parametrize("nk,hkv", [(1500, 40), (4096, 40), (4097, 40), (2000, 10)])
def test_staged_epilogue(cuda_dev, nk, hkv):
    w = Workload(f"staged nk{nk} hkv{hkv}", 2, 40, hkv, 600, nk, 128, "fp16", False, seed=7)
    assert 2 * fa.num_tiles(w.B, w.Hq, w.Nq, w.D) >= 148
    rows = np.unique(np.concatenate([sample_rows(w.Nq, 24, w.seed), np.arange(505, 600, 6), [511, 512]]))
    compare(w, cuda_dev, rows=rows)


def test_deterministic_and_lse_optional(cuda_dev):
    w = Workload("det", 1, 4, 2, 777, 777, 128, "bf16", True, seed=5)
    (q, k, v), o1, l1 = run_cuda(w, cuda_dev)
    qd, kd, vd = (x.to(cuda_dev) for x in (q, k, v))
    o2, l2 = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale, causal=True)
    o3, none = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale, causal=True, return_lse=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3)


def test_side_stream(cuda_dev):
    w = Workload("stream", 1, 2, 2, 512, 512, 64, "fp16", False, seed=6)
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    ref, _ = fa.fa_fwd(q, k, v, causal=False)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, _ = fa.fa_fwd(q, k, v, causal=False)
    s.synchronize()
    assert torch.equal(o, ref)


# ------------------------------------------------------------ full-size workloads
def _full(w, n_rows, cuda_dev):
    """Every element when n_rows is None, else a seeded sample of n_rows query rows per head."""
    rows = None if n_rows is None else sample_rows(w.Nq, n_rows, w.seed)
    o, lse, (q, k, v), do, dl = compare(w, cuda_dev, rows=rows)
    # properties at every row: O is a convex combination of V rows, LSE is finite
    vmax = v.float().abs().amax(dim=(2, 3)).to(cuda_dev)
    g = w.Hq // w.Hkv
    bound = vmax.repeat_interleave(g, dim=1)[..., None, None]
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert bool((o.float().abs() <= bound * (1 + 1e-2) + 1e-2).all())
    return do, dl


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("peaky", [False, True])
def test_llama7b_layer(cuda_dev, causal, peaky):
    _full(llama7b(causal, peaky), None, cuda_dev)


@pytest.mark.parametrize("seed", SWEEP_SEEDS)
@pytest.mark.parametrize("n", [512, 2048, 4096, 8192])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_sweep(cuda_dev, n, causal, seed):
    _full(seq_sweep(n, causal, seed), None if n <= 4096 else 48, cuda_dev)


@pytest.mark.parametrize("hkv,d", [(8, 128), (1, 128), (8, 64), (8, 256)])
def test_gqa_headdim(cuda_dev, hkv, d):
    _full(gqa(hkv, d), 16, cuda_dev)


def test_long_context_128k(cuda_dev):
    _full(LONG, 256, cuda_dev)
