"""Pins for the oracle (CPU only).

The oracle (``oracle/attn_oracle.c``) is the three-step definition of
attention.  It is pinned here against things that do not come from the oracle
itself, chosen so that a plausible mistake in it -- a dropped scale, a missing
1/Z, a log base, a transposed or mis-indexed operand, a causal off-by-one, a
wrong GQA head map -- fails at least one test:

* closed-form cases worked by hand (``tests/golden/closed_forms.json``);
* brute force: pure-Python loops without the max-subtraction, on tiny inputs;
* the tiled online-softmax recurrence of the mooersco.com page (section
  "昇腾NPU上的分块策略", steps 1-5, normalising at every block as written
  there), in float64 numpy, which the pages say gives exactly the standard
  result (hwcomputing.csdn.net page, "在线softmax" paragraph);
* invariants: rows of the softmax sum to one, permuting keys and values
  together, identical keys, causal row 0, scale 0, a single key, GQA equal to
  repeated K/V heads;
* a library routine that shares no code: torch's scaled_dot_product_attention
  on the CPU in float64.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from fa_inputs import Workload, make_qkv, sample_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _ev(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"ln": math.log, "exp": math.exp, "sqrt": math.sqrt}))


def _rand(shape, seed, dtype=np.float32):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# ---------------------------------------------------------------- closed forms
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_closed_forms(case):
    q = np.array(case["q"], dtype=np.float32)[None, None]
    k = np.array(case["k"], dtype=np.float32)[None, None]
    v = np.array(case["v"], dtype=np.float32)[None, None]
    o, lse = oracle.attention(q, k, v, _ev(case["scale"]), case["causal"])
    want_o = np.array([[_ev(e) for e in row] for row in case["o"]])
    want_lse = np.array([_ev(e) for e in case["lse"]])
    np.testing.assert_allclose(o[0, 0], want_o, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], want_lse, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- brute force
def _brute(q, k, v, scale, causal):
    """Element-wise loops, no stabiliser: O[i,d] = sum_j e^{s_ij} v_jd / sum_j e^{s_ij}."""
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    O = np.zeros((B, Hq, Nq, D))
    L = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i in range(Nq):
                num = [0.0] * D
                den = 0.0
                for j in range(Nk):
                    if causal and j > i:
                        continue
                    s = 0.0
                    for d in range(D):
                        s += float(q[b, h, i, d]) * float(k[b, kh, j, d])
                    e = math.exp(scale * s)
                    den += e
                    for d in range(D):
                        num[d] += e * float(v[b, kh, j, d])
                for d in range(D):
                    O[b, h, i, d] = num[d] / den
                L[b, h, i] = math.log(den)
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 5, 7, 3), (2, 4, 2, 9, 6, 4), (1, 3, 1, 12, 12, 1),
                                   (1, 2, 2, 7, 3, 5)])
def test_brute_force(shape, causal):
    B, Hq, Hkv, Nq, Nk, D = shape
    q = _rand((B, Hq, Nq, D), 1)
    k = _rand((B, Hkv, Nk, D), 2)
    v = _rand((B, Hkv, Nk, D), 3)
    scale = 0.37
    o, lse = oracle.attention(q, k, v, scale, causal)
    bo, bl = _brute(q, k, v, scale, causal)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=1e-12, atol=1e-12)


# ------------------------------------------------- the pages' tiled recurrence
def _tiled_online_softmax(q, k, v, scale, causal, bm, bn):
    """Steps 1-5 of the mooersco.com page's tiling section, in float64.

    For each Q row block i and K column block j: S_block = scale * Q[i] K[j]^T,
    m_new = max(m_old, rowmax S_block), l_new = l_old*e^{m_old-m_new} + rowsum e^{S_block-m_new},
    P_block = e^{S_block-m_new} / l_new, O[i] = O[i] * (l_old*e^{m_old-m_new}/l_new) + P_block V[j].
    (The page's recurrence lost its '+' and '=' signs in extraction; this is the
    reading in which the final O is the softmax average.)
    """
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    O = np.zeros((B, Hq, Nq, D))
    LSE = np.zeros((B, Hq, Nq))
    q = q.astype(np.float64)
    k = k.astype(np.float64)
    v = v.astype(np.float64)
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i0 in range(0, Nq, bm):
                Qi = q[b, h, i0:i0 + bm]
                rows = np.arange(i0, min(i0 + bm, Nq))
                m = np.full(len(rows), -np.inf)
                l = np.zeros(len(rows))
                Oi = np.zeros((len(rows), D))
                for j0 in range(0, Nk, bn):
                    cols = np.arange(j0, min(j0 + bn, Nk))
                    S = scale * (Qi @ k[b, kh, j0:j0 + bn].T)
                    if causal:
                        S = np.where(cols[None, :] <= rows[:, None], S, -np.inf)
                    m_new = np.maximum(m, S.max(axis=1))
                    # a row that has seen no visible key yet keeps m = -inf; guard e^{-inf - -inf}
                    safe = np.where(np.isfinite(m_new), m_new, 0.0)
                    decay = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
                    E = np.exp(S - safe[:, None])
                    l_new = l * decay + E.sum(axis=1)
                    seen = l_new > 0
                    inv = np.where(seen, 1.0 / np.where(seen, l_new, 1.0), 0.0)
                    P = E * inv[:, None]
                    Oi = Oi * (l * decay * inv)[:, None] + P @ v[b, kh, j0:j0 + bn]
                    m, l = m_new, l_new
                O[b, h, rows] = Oi
                LSE[b, h, rows] = m + np.log(l)
    return O, LSE


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bm,bn", [(1, 1), (4, 7), (64, 64), (16, 128)])
def test_tiled_recurrence_equals_definition(causal, bm, bn):
    w = Workload("t", 1, 4, 2, 130, 130, 16, "fp16", causal, seed=5, q_mult=3.0)
    q, k, v = make_qkv(w)
    o, lse = oracle.attention(q, k, v, 0.25, causal)
    to, tl = _tiled_online_softmax(q.float().numpy(), k.float().numpy(), v.float().numpy(), 0.25,
                                   causal, bm, bn)
    np.testing.assert_allclose(o, to, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, tl, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- invariants
def _scores(q, k, scale):
    """Scores with numpy's float64 matmul (independent of the oracle's loops)."""
    B, Hq, Nq, D = q.shape
    Hkv = k.shape[1]
    krep = np.repeat(k.astype(np.float64), Hq // Hkv, axis=1)
    return scale * np.einsum("bhid,bhjd->bhij", q.astype(np.float64), krep)


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    q = _rand((2, 4, 33, 8), 11) * 3
    k = _rand((2, 2, 40, 8), 12)
    v = _rand((2, 2, 40, 8), 13)
    _, lse = oracle.attention(q, k, v, 0.5, causal)
    s = _scores(q, k, 0.5)
    if causal:
        mask = np.arange(40)[None, :] <= np.arange(33)[:, None]
        s = np.where(mask, s, -np.inf)
    tot = np.exp(s - lse[..., None]).sum(axis=-1)
    np.testing.assert_allclose(tot, 1.0, rtol=0, atol=1e-12)


def test_permuting_keys_and_values_together():
    q = _rand((1, 2, 17, 8), 21)
    k = _rand((1, 2, 29, 8), 22)
    v = _rand((1, 2, 29, 8), 23)
    perm = np.random.default_rng(24).permutation(29)
    o1, l1 = oracle.attention(q, k, v, 0.3, False)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], 0.3, False)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-13)
    # permuting keys alone changes the result (the pin would catch a K/V mix-up)
    o3, _ = oracle.attention(q, k[:, :, perm], v, 0.3, False)
    assert np.abs(o3 - o1).max() > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_values(causal):
    n, d = 23, 6
    q = _rand((1, 1, n, d), 31)
    krow = _rand((d,), 32)
    k = np.broadcast_to(krow, (1, 1, n, d)).copy()
    v = _rand((1, 1, n, d), 33)
    o, lse = oracle.attention(q, k, v, 0.7, causal)
    s = 0.7 * (q[0, 0].astype(np.float64) @ krow.astype(np.float64))
    cnt = np.arange(1, n + 1) if causal else np.full(n, n)
    if causal:
        want = np.cumsum(v[0, 0].astype(np.float64), axis=0) / cnt[:, None]
    else:
        want = np.broadcast_to(v[0, 0].astype(np.float64).mean(axis=0), (n, d))
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], s + np.log(cnt), rtol=1e-13, atol=1e-12)


def test_causal_row_zero_is_first_value():
    q = _rand((2, 2, 9, 5), 41)
    k = _rand((2, 2, 9, 5), 42)
    v = _rand((2, 2, 9, 5), 43)
    o, lse = oracle.attention(q, k, v, 0.9, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0].astype(np.float64))
    want = 0.9 * np.einsum("bhd,bhd->bh", q[:, :, 0].astype(np.float64), k[:, :, 0].astype(np.float64))
    np.testing.assert_allclose(lse[:, :, 0], want, rtol=1e-13, atol=1e-13)


def test_scale_zero_is_uniform_average():
    q = _rand((1, 2, 10, 4), 51)
    k = _rand((1, 2, 13, 4), 52)
    v = _rand((1, 2, 13, 4), 53)
    o, lse = oracle.attention(q, k, v, 0.0, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.astype(np.float64).mean(axis=2, keepdims=True),
                                                  o.shape), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, math.log(13), rtol=1e-14)


def test_single_key():
    q = _rand((1, 3, 6, 4), 61)
    k = _rand((1, 3, 1, 4), 62)
    v = _rand((1, 3, 1, 4), 63)
    o, _ = oracle.attention(q, k, v, 1.3, False)
    np.testing.assert_array_equal(o, np.broadcast_to(v.astype(np.float64), o.shape))


@pytest.mark.parametrize("hq,hkv", [(4, 2), (8, 1), (6, 3)])
def test_gqa_equals_repeated_kv(hq, hkv):
    q = _rand((2, hq, 11, 8), 71)
    k = _rand((2, hkv, 14, 8), 72)
    v = _rand((2, hkv, 14, 8), 73)
    o1, l1 = oracle.attention(q, k, v, 0.35, True)
    g = hq // hkv
    o2, l2 = oracle.attention(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), 0.35, True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(64, 64), (50, 80), (80, 50)])
def test_against_torch_sdpa_float64(causal, nq, nk):
    q = _rand((2, 4, nq, 16), 81)
    k = _rand((2, 4, nk, 16), 82)
    v = _rand((2, 4, nk, 16), 83)
    o, lse = oracle.attention(q, k, v, 0.2, causal)
    tq, tk, tv = (torch.from_numpy(x.astype(np.float64)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.2)
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-11, atol=1e-12)
    s = torch.einsum("bhid,bhjd->bhij", tq, tk) * 0.2
    if causal:
        s = s.masked_fill(torch.ones(nq, nk, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12, atol=1e-12)


def test_sampled_rows_match_full():
    w = Workload("t", 1, 4, 2, 300, 300, 32, "bf16", True, seed=3)
    q, k, v = make_qkv(w)
    rows = sample_rows(300, 20, 9)
    assert rows[0] == 0 and rows[-1] == 299 and len(rows) == 20
    o, l = oracle.attention(q, k, v, 0.17, True)
    os_, ls = oracle.attention(q, k, v, 0.17, True, rows=rows)
    np.testing.assert_array_equal(os_, o[:, :, rows])
    np.testing.assert_array_equal(ls, l[:, :, rows])


def test_rejects_bad_arguments():
    q = _rand((1, 3, 4, 4), 1)
    k = _rand((1, 2, 4, 4), 2)
    with pytest.raises(ValueError):
        oracle.attention(q, k, k, 1.0, False)  # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.attention(q[:, :2], k, k, 1.0, False, rows=np.array([0, 4]))  # row out of range


def test_inputs_are_seeded_and_rounded():
    w = Workload("t", 1, 2, 1, 40, 50, 8, "bf16", False, seed=7, outlier_frac=0.1, outlier_mult=8.0)
    a = make_qkv(w)
    b = make_qkv(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and x.dtype == torch.bfloat16 and x.is_contiguous()
    assert a[0].shape == (1, 2, 40, 8) and a[1].shape == (1, 1, 50, 8)
    # 10% of the key rows carry the x8 outlier factor: their norms stand out
    norms = a[1].float().norm(dim=-1)[0, 0]
    assert int((norms > 4 * norms.median()).sum()) == 5
