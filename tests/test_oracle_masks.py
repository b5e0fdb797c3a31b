"""Pins for the oracle's masks beyond causal (CPU only).

The pages put a mask step on the vector unit and call PyTorch's
scaled_dot_product_attention, whose attn_mask adds to the scores (mooersco.com
page, PyTorch section).  The oracle reads that as two masks: a key window
(query i sees keys i - left .. i + right) and an additive score bias (-inf
removes a key); a row left with no key has O = 0 and LSE = -inf.  They are
pinned here against:

* brute force: pure-Python loops over an explicit visibility test, on tiny
  inputs, with no max subtraction;
* torch's scaled_dot_product_attention on the CPU in float64, given the same
  masks as a boolean or float attn_mask (rows that keep a key);
* closed forms and special cases: a (0, 0) window is the value at the query's
  own position; (-1, 0) is causal; a window wider than the keys is no mask;
  a bias constant along a row shifts only LSE; -inf bias outside a window is
  that window; a one-hot large bias selects one value.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def _visible(i, j, causal, wl, wr):
    if causal and j > i:
        return False
    if wl >= 0 and j < i - wl:
        return False
    if wr >= 0 and j > i + wr:
        return False
    return True


def _brute(q, k, v, scale, causal, wl, wr, bias=None):
    """O and LSE by plain loops: Z = sum of exp(score) over visible keys."""
    B, H, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = H // Hkv
    o = np.zeros((B, H, Nq, D))
    lse = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        for h in range(H):
            kv = h // g
            for i in range(Nq):
                w = {}
                for j in range(Nk):
                    if not _visible(i, j, causal, wl, wr):
                        continue
                    s = scale * sum(float(q[b, h, i, d]) * float(k[b, kv, j, d]) for d in range(D))
                    if bias is not None:
                        s += float(bias[b, h, i, j])
                    if s == -math.inf:
                        continue
                    w[j] = math.exp(s)
                if not w:
                    continue
                z = math.fsum(w.values())
                lse[b, h, i] = math.log(z)
                for d in range(D):
                    o[b, h, i, d] = math.fsum(w[j] / z * float(v[b, kv, j, d]) for j in w)
    return o, lse


WINDOWS = [(-1, -1), (0, 0), (2, 1), (3, -1), (-1, 2), (1, 0), (5, 5)]


@pytest.mark.parametrize("wl,wr", WINDOWS)
@pytest.mark.parametrize("causal", [False, True])
def test_window_brute_force(wl, wr, causal):
    q, k, v = _rand((1, 2, 9, 4), 1), _rand((1, 1, 7, 4), 2), _rand((1, 1, 7, 4), 3)
    o, lse = oracle.attention(q, k, v, 0.7, causal, window=(wl, wr))
    bo, bl = _brute(q, k, v, 0.7, causal, wl, wr)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=1e-12, atol=1e-12)


def test_bias_brute_force():
    q, k, v = _rand((2, 2, 6, 3), 4), _rand((2, 1, 5, 3), 5), _rand((2, 1, 5, 3), 6)
    bias = _rand((2, 2, 6, 5), 7)
    bias[0, 1, 2, :] = -np.inf  # a row with every key removed
    bias[1, 0, :, 3] = -np.inf  # one key removed for every row of a head
    o, lse = oracle.attention(q, k, v, 0.5, False, bias=bias)
    bo, bl = _brute(q, k, v, 0.5, False, -1, -1, bias)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    assert np.isneginf(lse[0, 1, 2]) and np.all(o[0, 1, 2] == 0.0)
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=1e-12, atol=1e-12)


def _sdpa(q, k, v, scale, mask):
    """torch SDPA in float64 with a boolean (True = keep) or float attn_mask."""
    g = q.shape[1] // k.shape[1]
    kt = torch.from_numpy(k).double().repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).double().repeat_interleave(g, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double(), kt, vt, attn_mask=mask, scale=scale).numpy()


@pytest.mark.parametrize("wl,wr,causal,nq,nk", [(16, 16, False, 64, 80), (31, -1, True, 96, 96),
                                                (7, 0, False, 40, 40), (0, 40, False, 50, 30)])
def test_window_against_torch_sdpa(wl, wr, causal, nq, nk):
    q, k, v = _rand((2, 4, nq, 16), 8), _rand((2, 2, nk, 16), 9), _rand((2, 2, nk, 16), 10)
    keep = np.array([[_visible(i, j, causal, wl, wr) for j in range(nk)] for i in range(nq)])
    o, _ = oracle.attention(q, k, v, 0.25, causal, window=(wl, wr))
    ref = _sdpa(q, k, v, 0.25, torch.from_numpy(keep))
    rows = keep.any(axis=1)
    np.testing.assert_allclose(o[:, :, rows], ref[:, :, rows], rtol=1e-10, atol=1e-12)
    assert np.all(o[:, :, ~rows] == 0.0)


def test_bias_against_torch_sdpa():
    q, k, v = _rand((1, 4, 33, 8), 11), _rand((1, 4, 47, 8), 12), _rand((1, 4, 47, 8), 13)
    bias = 3.0 * _rand((1, 1, 33, 47), 14)  # broadcast over heads
    o, _ = oracle.attention(q, k, v, 0.3, False, bias=bias)
    ref = _sdpa(q, k, v, 0.3, torch.from_numpy(bias).double())
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)


def test_zero_window_is_own_value():
    q, k, v = _rand((1, 2, 6, 8), 15), _rand((1, 2, 6, 8), 16), _rand((1, 2, 6, 8), 17)
    o, lse = oracle.attention(q, k, v, 0.9, False, window=(0, 0))
    np.testing.assert_array_equal(o, v.astype(np.float64))
    s = 0.9 * np.einsum("bhid,bhid->bhi", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, s, rtol=1e-13, atol=1e-13)


def test_left_unbounded_right_zero_is_causal():
    q, k, v = _rand((1, 2, 30, 8), 18), _rand((1, 2, 30, 8), 19), _rand((1, 2, 30, 8), 20)
    a = oracle.attention(q, k, v, 0.4, False, window=(-1, 0))
    b = oracle.attention(q, k, v, 0.4, True)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_wide_window_is_no_mask():
    q, k, v = _rand((1, 2, 20, 8), 21), _rand((1, 2, 25, 8), 22), _rand((1, 2, 25, 8), 23)
    a = oracle.attention(q, k, v, 0.4, False, window=(30, 30))
    b = oracle.attention(q, k, v, 0.4, False)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_rows_beyond_window_are_empty():
    # Nq > Nk + left: queries 12.. see no key
    q, k, v = _rand((1, 1, 16, 4), 24), _rand((1, 1, 10, 4), 25), _rand((1, 1, 10, 4), 26)
    o, lse = oracle.attention(q, k, v, 0.5, False, window=(2, 3))
    assert np.all(np.isneginf(lse[0, 0, 12:])) and np.all(o[0, 0, 12:] == 0.0)
    assert np.all(np.isfinite(lse[0, 0, :12]))


def test_row_constant_bias_shifts_lse_only():
    q, k, v = _rand((1, 2, 12, 8), 27), _rand((1, 2, 14, 8), 28), _rand((1, 2, 14, 8), 29)
    c = _rand((1, 2, 12, 1), 30)
    bias = np.repeat(c, 14, axis=3)
    o0, l0 = oracle.attention(q, k, v, 0.6, False)
    o1, l1 = oracle.attention(q, k, v, 0.6, False, bias=bias)
    np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l0 + c[..., 0].astype(np.float64), rtol=1e-12, atol=1e-12)


def test_neg_inf_bias_outside_window_is_window():
    q, k, v = _rand((1, 2, 24, 8), 31), _rand((1, 2, 24, 8), 32), _rand((1, 2, 24, 8), 33)
    i, j = np.meshgrid(np.arange(24), np.arange(24), indexing="ij")
    bias = np.where((j >= i - 5) & (j <= i + 2), 0.0, -np.inf).astype(np.float32)
    a = oracle.attention(q, k, v, 0.5, False, bias=bias)
    b = oracle.attention(q, k, v, 0.5, False, window=(5, 2))
    np.testing.assert_allclose(a[0], b[0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-13, atol=1e-14)


def test_one_hot_large_bias_selects_a_value():
    q, k, v = _rand((1, 1, 5, 8), 34), _rand((1, 1, 9, 8), 35), _rand((1, 1, 9, 8), 36)
    bias = np.zeros((1, 1, 5, 9), dtype=np.float32)
    pick = [3, 0, 8, 4, 4]
    for i, j in enumerate(pick):
        bias[0, 0, i, j] = 1000.0  # every other weight is below e^-900
    o, _ = oracle.attention(q, k, v, 0.1, False, bias=bias)
    np.testing.assert_allclose(o[0, 0], v[0, 0, pick].astype(np.float64), rtol=0, atol=1e-300)


def test_bias_rejects_bad_shape():
    q, k, v = _rand((1, 2, 4, 4), 37), _rand((1, 2, 5, 4), 38), _rand((1, 2, 5, 4), 39)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0, False, bias=np.zeros((1, 2, 4, 6), np.float32))
