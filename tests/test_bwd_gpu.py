"""GPU parity of the backward pass (fa_bwd) against the float64 gradient oracle.

The forward pass runs on the GPU first (its O and LSE feed fa_bwd, as in
training); the oracle computes the exact gradients from Q, K, V and dO alone.
Tolerance (no stated bound for gradients): P and dS are rounded to the input
dtype before their MMAs and each output is rounded once, each a relative error
of about one unit roundoff u of the dtype (fp16 2^-11, bf16 2^-8) against the
tensor's own scale, so max |got - ref| <= 4 u max|ref| + A per tensor.  A is
zero for dV.  For dQ and dK it bounds what survives a cancellation the exact
gradient has: dS = P (dP - Delta), and dP and Delta are two fp32 dot products
of length D (dO . V_j and dO . O_i) that agree exactly when a row sees one
key, so their difference is only their rounding, at most 2 D 2^-24 max|dO|
max|V|; times the scale and max|K| (dQ) or max|Q| (dK).  Where nothing cancels
A is a few percent of the first term.
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

U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


def _dout(w):
    g = np.random.default_rng(w.seed + 1000).standard_normal((w.B, w.Hq, w.Nq, w.D)).astype(np.float32)
    return torch.from_numpy(g).to(torch.float16 if w.dtype == "fp16" else torch.bfloat16)


def _run(w, dev, window=(-1, -1), bias=None):
    q, k, v = make_qkv(w)
    g = _dout(w)
    qd, kd, vd, gd = (x.to(dev) for x in (q, k, v, g))
    bd = bias.to(dev) if bias is not None else None
    o, lse = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal, window=window, bias=bd)
    dq, dk, dv = fa.fa_bwd(qd, kd, vd, o, lse, gd, scale=w.softmax_scale, causal=w.causal,
                           window=window, bias=bd)
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    return (q, k, v, g), (dq, dk, dv)


def grad_tolerance(w, q, k, v, g, ref):
    """Per-tensor bound 4 u max|ref| + A (see the module docstring)."""
    u = U[w.dtype]
    mx = lambda x: float(x.float().abs().max())  # noqa: E731
    resid = 2 * w.D * 2.0 ** -24 * mx(g) * mx(v) * abs(w.softmax_scale)
    extra = {"dQ": resid * mx(k), "dK": resid * mx(q), "dV": 0.0}
    return {n: 4 * u * float(np.abs(r).max()) + extra[n] for n, r in zip(("dQ", "dK", "dV"), ref)}


def _check(w, got, ref, inputs, tag=""):
    report = os.environ.get("FA_PARITY_REPORT")
    tol = grad_tolerance(w, *inputs, ref)
    rows = {}
    for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
        a = a.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), name
        scale = np.abs(b).max()
        err = np.abs(a - b).max()
        rows[name] = (err, scale)
    if report:
        with open(report, "a") as f:
            f.write(json.dumps({"case": "bwd " + w.name + tag, "dtype": w.dtype,
                                **{f"max_abs_d{n}": float(e) for n, (e, _) in rows.items()},
                                **{f"max_ref_{n}": float(s) for n, (_, s) in rows.items()}}) + "\n")
    for name, (err, scale) in rows.items():
        assert err <= tol[name], f"{w.name} {name}: {err:.3e} > {tol[name]:.3e} (max|ref| {scale:.3e})"


CASES = [
    Workload("bwd tiny D64 fp16", 1, 2, 2, 256, 256, 64, "fp16", False, seed=91),
    Workload("bwd D128 fp16 causal ragged GQA", 1, 4, 2, 700, 700, 128, "fp16", True, seed=92),
    Workload("bwd D128 bf16 Nq<Nk GQA 4", 1, 8, 2, 300, 1000, 128, "bf16", False, seed=93),
    Workload("bwd D64 bf16 causal Nk<Nq", 2, 2, 1, 1000, 600, 64, "bf16", True, seed=94),
    Workload("bwd D128 fp16 causal Nk>Nq", 1, 2, 2, 300, 1000, 128, "fp16", True, seed=95),
    Workload("bwd single row and key", 1, 3, 1, 1, 1, 128, "fp16", False, seed=96),
    Workload("bwd D64 fp16 odd sizes", 2, 3, 3, 129, 255, 64, "fp16", False, seed=97),
    Workload("bwd D128 fp16 N2048 causal", 1, 4, 4, 2048, 2048, 128, "fp16", True, seed=98),
    Workload("bwd D128 bf16 N2048", 1, 4, 4, 2048, 2048, 128, "bf16", False, seed=99),
    # head_dim 256: 64-row streamed blocks, dV and dK from separate launches
    Workload("bwd D256 fp16 ragged", 1, 2, 2, 300, 333, 256, "fp16", False, seed=141),
    Workload("bwd D256 bf16 causal GQA 4", 1, 8, 2, 520, 520, 256, "bf16", True, seed=142),
    Workload("bwd D256 fp16 causal Nk>Nq", 2, 2, 1, 200, 700, 256, "fp16", True, seed=143),
    Workload("bwd D256 bf16 N1024", 1, 4, 4, 1024, 1024, 256, "bf16", False, seed=144),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_bwd_parity(cuda_dev, w):
    (q, k, v, g), got = _run(w, cuda_dev)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal)
    _check(w, got, (dq, dk, dv), (q, k, v, g))


def test_bwd_deterministic(cuda_dev):
    w = Workload("bwd det", 1, 4, 2, 500, 640, 128, "bf16", True, seed=100)
    _, a = _run(w, cuda_dev)
    _, b = _run(w, cuda_dev)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bwd_back_to_back_calls(cuda_dev):
    # two calls on one stream and one workspace, enqueued without a host wait: the
    # second (other data, other shape) must see only its own Delta and LSE, and
    # gives what the same call gives alone (the kernels of a call overlap their
    # predecessor's tail through programmatic launch)
    wa = Workload("bwd b2b a", 2, 40, 40, 512, 512, 128, "fp16", True, seed=101)
    wb = Workload("bwd b2b b", 1, 40, 10, 640, 700, 128, "fp16", False, seed=102)
    ws = torch.empty(max(fa.load_library().fa_bwd_workspace_size(w.B, w.Hq, w.Nq) for w in (wa, wb)),
                     dtype=torch.uint8, device=cuda_dev)

    def prepare(w):
        q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
        g = _dout(w).to(cuda_dev)
        o, lse = fa.fa_fwd(q, k, v, scale=w.softmax_scale, causal=w.causal)
        return q, k, v, o, lse, g

    def bwd(w, t):
        q, k, v, o, lse, g = t
        return fa.fa_bwd(q, k, v, o, lse, g, scale=w.softmax_scale, causal=w.causal, workspace=ws)

    ta, tb = prepare(wa), prepare(wb)
    torch.cuda.synchronize()
    alone = bwd(wb, tb)
    torch.cuda.synchronize()
    bwd(wa, ta)
    after = bwd(wb, tb)  # enqueued right behind the first call
    torch.cuda.synchronize()
    assert fa.device_status(reset=True) == 0
    for x, y in zip(alone, after):
        assert torch.equal(x, y)


def test_bwd_sum_invariants_on_device(cuda_dev):
    # the key-sum of dK vanishes and the key-sum of dV is the query-sum of dO
    w = Workload("bwd sums", 1, 2, 2, 512, 512, 64, "fp16", False, seed=101)
    (q, k, v, g), (dq, dk, dv) = _run(w, cuda_dev)
    s_dv = dv.double().sum(dim=2).cpu().numpy()
    want = g.double().sum(dim=2).numpy()
    np.testing.assert_allclose(s_dv, want, rtol=0, atol=0.05 * np.abs(want).max())
    assert np.abs(dk.double().sum(dim=2).cpu().numpy()).max() <= 0.02 * np.abs(dk.double().cpu().numpy()).sum(2).max()


# key windows (the gradient of fa_fwd_window's operation)
WINDOW_CASES = [
    (Workload("bwd sliding causal 255 D128 fp16", 1, 4, 2, 1000, 1000, 128, "fp16", True, seed=131), (255, -1)),
    (Workload("bwd local 100/50 D64 bf16", 2, 2, 2, 777, 777, 64, "bf16", False, seed=132), (100, 50)),
    (Workload("bwd narrow 5/3 D128 fp16", 1, 2, 2, 600, 600, 128, "fp16", False, seed=133), (5, 3)),
    # queries 410.. see no key (Nq > Nk + left): their dQ rows are 0
    (Workload("bwd empty rows D64 fp16", 1, 2, 2, 700, 300, 64, "fp16", False, seed=134), (110, 10)),
    (Workload("bwd right only 64 D128 bf16 GQA", 1, 4, 2, 500, 600, 128, "bf16", False, seed=135), (-1, 64)),
    (Workload("bwd causal window 128 D128 fp16 Nk>Nq", 1, 2, 2, 300, 900, 128, "fp16", True, seed=136), (128, 0)),
    (Workload("bwd local 70/30 D256 bf16", 1, 2, 2, 400, 400, 256, "bf16", False, seed=137), (70, 30)),
    (Workload("bwd empty rows D256 fp16", 1, 2, 1, 500, 200, 256, "fp16", False, seed=138), (40, 5)),
]


@pytest.mark.parametrize("w,window", WINDOW_CASES, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_bwd_window_parity(cuda_dev, w, window):
    (q, k, v, g), got = _run(w, cuda_dev, window)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal, window=window)
    _check(w, got, (dq, dk, dv), (q, k, v, g), f" window {window}")


# ---- additive score bias (fa_bwd_bias): P includes the bias

def _bias(w, shape, seed, scale=2.0, neg_inf_frac=0.0):
    rng = np.random.default_rng(seed)
    b = (scale * rng.standard_normal(shape)).astype(np.float32)
    if neg_inf_frac > 0:
        b[rng.random(shape) < neg_inf_frac] = -np.inf
    return torch.from_numpy(b).to(torch.float16 if w.dtype == "fp16" else torch.bfloat16)


BIAS_CASES = [
    (Workload("bwd bias full D128 fp16 ragged GQA", 1, 4, 2, 300, 333, 128, "fp16", False, seed=151),
     (1, 4, 300, 333), 0.0),
    (Workload("bwd bias shared [N,N] D128 bf16 causal", 2, 2, 2, 640, 640, 128, "bf16", True, seed=152),
     (1, 1, 640, 640), 0.0),
    (Workload("bwd bias key padding D64 fp16", 2, 4, 4, 500, 520, 64, "fp16", False, seed=153),
     (2, 1, 1, 520), 0.2),
    (Workload("bwd bias per head D64 bf16 causal GQA 4", 1, 8, 2, 384, 384, 64, "bf16", True, seed=154),
     (1, 8, 384, 384), 0.05),
]


@pytest.mark.parametrize("w,shape,ninf", BIAS_CASES, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_bwd_bias_parity(cuda_dev, w, shape, ninf):
    bias = _bias(w, shape, w.seed + 7, neg_inf_frac=ninf)
    inputs, got = _run(w, cuda_dev, bias=bias)
    q, k, v, g = inputs
    ref = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal, bias=bias.float())[:3]
    _check(w, got, ref, inputs, tag=" bias")


def test_bwd_bias_rows_without_keys(cuda_dev):
    # rows whose keys the bias removes entirely: lse = -inf, their dQ rows are 0
    w = Workload("bwd bias empty rows D128 fp16", 1, 2, 2, 260, 200, 128, "fp16", False, seed=155)
    b = np.zeros((1, 2, 260, 200), dtype=np.float32)
    b[:, :, 100:140] = -np.inf
    bias = torch.from_numpy(b).half()
    inputs, got = _run(w, cuda_dev, bias=bias)
    q, k, v, g = inputs
    ref = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal, bias=bias.float())[:3]
    _check(w, got, ref, inputs, tag=" bias")
    assert (got[0][:, :, 100:140] == 0).all()


def test_bwd_zero_bias_equals_no_bias(cuda_dev):
    # the same forward outputs: a zero bias leaves every backward operation unchanged
    w = Workload("bwd zero bias D64 fp16", 1, 2, 2, 256, 256, 64, "fp16", True, seed=156)
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    g = _dout(w).to(cuda_dev)
    o, lse = fa.fa_fwd(q, k, v, scale=w.softmax_scale, causal=True)
    plain = fa.fa_bwd(q, k, v, o, lse, g, scale=w.softmax_scale, causal=True)
    for shape in ((1, 1, 256, 256), (1, 1, 1, 256)):
        zero = fa.fa_bwd(q, k, v, o, lse, g, scale=w.softmax_scale, causal=True,
                         bias=torch.zeros(shape, dtype=torch.float16, device=cuda_dev))
        torch.cuda.synchronize()
        assert fa.device_status(reset=True) == 0
        for a, b in zip(plain, zero):
            assert torch.equal(a, b)


# ---- a key window and a score bias together (fa_bwd_bias_window)

@pytest.mark.parametrize("w,window,shape", [
    (Workload("bwd window 200 causal + full bias D128 fp16", 1, 4, 2, 600, 600, 128, "fp16", True,
              seed=161), (200, -1), (1, 4, 600, 600)),
    (Workload("bwd window 40/20 + padding mask D64 bf16", 2, 2, 2, 333, 350, 64, "bf16", False,
              seed=162), (40, 20), (2, 1, 1, 350)),
], ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_bwd_window_and_bias_parity(cuda_dev, w, window, shape):
    bias = _bias(w, shape, w.seed + 7, neg_inf_frac=0.1)
    inputs, got = _run(w, cuda_dev, window=window, bias=bias)
    q, k, v, g = inputs
    ref = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal, window=window,
                               bias=bias.float())[:3]
    _check(w, got, ref, inputs, tag=" window bias")


# ---- the persistent kernels: more tiles than SMs, so a CTA takes several

MANY = [
    # causal over 256 keys: tiles of one and two query blocks (a short tile's
    # staging gate is still pending when the next tile's items are issued)
    (Workload("bwd many tiles D128 fp16 causal", 4, 40, 40, 256, 256, 128, "fp16", True, seed=171),
     (-1, -1), None),
    # causal with Nk > Nq: key tiles no query sees (zeros) between the others
    (Workload("bwd many tiles D128 bf16 causal Nk>Nq GQA", 4, 40, 20, 256, 512, 128, "bf16", True,
              seed=172), (-1, -1), None),
    (Workload("bwd many tiles D64 fp16", 3, 40, 40, 384, 384, 64, "fp16", False, seed=173), (-1, -1), None),
    (Workload("bwd many tiles D128 fp16 window", 2, 40, 20, 640, 640, 128, "fp16", False, seed=174),
     (100, 50), None),
    (Workload("bwd many tiles D128 fp16 bias", 2, 40, 40, 256, 300, 128, "fp16", False, seed=175),
     (-1, -1), (1, 1, 256, 300)),
]


@pytest.mark.parametrize("w,window,shape", MANY, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_bwd_many_tiles_per_cta(cuda_dev, w, window, shape):
    kv_tiles = w.B * w.Hkv * -(-w.Nk // 128)
    q_tiles = w.B * w.Hq * -(-w.Nq // 128)
    assert min(kv_tiles, q_tiles) > 148
    bias = _bias(w, shape, w.seed + 7, neg_inf_frac=0.05) if shape is not None else None
    inputs, got = _run(w, cuda_dev, window=window, bias=bias)
    q, k, v, g = inputs
    ref = oracle.attention_bwd(q, k, v, g, w.softmax_scale, w.causal, window=window,
                               bias=None if bias is None else bias.float())[:3]
    _check(w, got, ref, inputs, tag=" many tiles")
