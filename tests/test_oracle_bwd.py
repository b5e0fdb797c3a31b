"""Pins for the oracle's gradients (CPU only).

The backward oracle (``oracle_attention_bwd``) writes out the chain rule for
O = softmax(scale * Q K^T) V.  It is pinned against things that do not come
from its own formulas, so that a dropped scale, a missing Delta, a transposed
operand, a wrong GQA sum or a causal off-by-one fails at least one test:

* central finite differences of L = sum(dO * O) in float64 (the forward used
  there is checked against the forward oracle first);
* torch autograd through scaled_dot_product_attention in float64 on the CPU;
* invariants: the key-sum of dK is zero, the key-sum of dV is the query-sum of
  dO, Delta = dO . O; scale 0 and a single key give dQ = dK = 0;
* GQA equals repeated K/V heads with dK, dV summed over each group.
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed, scale=1.0):
    return (scale * np.random.default_rng(seed).standard_normal(shape)).astype(np.float32)


def _forward64(q, k, v, scale, causal):
    """softmax(scale q k^T) v in float64 (numpy), GQA by repeating K/V heads."""
    g = q.shape[1] // k.shape[1]
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    s = scale * np.einsum("bhid,bhjd->bhij", q, kr)
    if causal:
        i, j = np.meshgrid(np.arange(q.shape[2]), np.arange(k.shape[2]), indexing="ij")
        s = np.where(j <= i, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return np.einsum("bhij,bhjd->bhid", p, vr)


@pytest.mark.parametrize("causal", [False, True])
def test_forward64_matches_oracle(causal):
    q, k, v = _rand((1, 4, 7, 5), 1), _rand((1, 2, 9, 5), 2), _rand((1, 2, 9, 5), 3)
    o, _ = oracle.attention(q, k, v, 0.6, causal)
    np.testing.assert_allclose(_forward64(q.astype(np.float64), k.astype(np.float64),
                                          v.astype(np.float64), 0.6, causal), o, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    q, k, v = _rand((1, 2, 5, 3), 4), _rand((1, 1, 6, 3), 5), _rand((1, 1, 6, 3), 6)
    g = _rand((1, 2, 5, 3), 7)
    scale = 0.8
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, scale, causal)
    x = [q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)]
    h = 1e-5

    def loss(xs):
        return float(np.sum(g.astype(np.float64) * _forward64(*xs, scale, causal)))

    for which, grad in enumerate((dq, dk, dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += h
            xm[which][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal,nq,nk,hq,hkv", [(False, 33, 47, 4, 2), (True, 40, 40, 2, 2),
                                                 (True, 25, 31, 6, 1), (False, 1, 17, 2, 1)])
def test_against_torch_autograd(causal, nq, nk, hq, hkv):
    q, k, v = _rand((2, hq, nq, 16), 8), _rand((2, hkv, nk, 16), 9), _rand((2, hkv, nk, 16), 10)
    g = _rand((2, hq, nq, 16), 11)
    dq, dk, dv, delta = oracle.attention_bwd(q, k, v, g, 0.3, causal)
    qt, kt, vt = (torch.from_numpy(a).double().requires_grad_() for a in (q, k, v))
    grp = hq // hkv
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(grp, dim=1), vt.repeat_interleave(grp, dim=1), is_causal=causal,
        scale=0.3)
    o.backward(torch.from_numpy(g).double())
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(delta, (g.astype(np.float64) * o.detach().numpy()).sum(-1),
                               rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_sum_invariants(causal):
    q, k, v = _rand((2, 4, 20, 8), 12), _rand((2, 2, 24, 8), 13), _rand((2, 2, 24, 8), 14)
    g = _rand((2, 4, 20, 8), 15)
    _, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.5, causal)
    # every row of dS sums to zero -> the key-sum of dK vanishes
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # every row of P sums to one -> the key-sum of dV is the query-sum of dO over the group
    want = g.astype(np.float64).reshape(2, 2, 2, 20, 8).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), want, rtol=1e-12, atol=1e-12)


def test_scale_zero_and_single_key():
    q, k, v = _rand((1, 2, 6, 4), 16), _rand((1, 2, 9, 4), 17), _rand((1, 2, 9, 4), 18)
    g = _rand((1, 2, 6, 4), 19)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.0, False)
    assert np.all(dq == 0.0) and np.all(dk == 0.0)
    np.testing.assert_allclose(dv, np.repeat(g.astype(np.float64).sum(axis=2, keepdims=True) / 9,
                                             9, axis=2), rtol=1e-13, atol=1e-14)
    dq, dk, dv, _ = oracle.attention_bwd(q, k[:, :, :1], v[:, :, :1], g, 0.7, False)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dk, 0.0, atol=1e-13)
    np.testing.assert_allclose(dv[:, :, 0], g.astype(np.float64).sum(axis=2), rtol=1e-13)


def test_gqa_equals_repeated_kv():
    q, k, v = _rand((1, 6, 11, 4), 20), _rand((1, 2, 13, 4), 21), _rand((1, 2, 13, 4), 22)
    g = _rand((1, 6, 11, 4), 23)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.4, True)
    dq2, dk2, dv2, _ = oracle.attention_bwd(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), g,
                                            0.4, True)
    np.testing.assert_allclose(dq, dq2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(dk, dk2.reshape(1, 2, 3, 13, 4).sum(axis=2), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(1, 2, 3, 13, 4).sum(axis=2), rtol=1e-12, atol=1e-13)


def test_delta_is_dout_dot_output():
    q, k, v = _rand((1, 2, 15, 8), 24), _rand((1, 2, 15, 8), 25), _rand((1, 2, 15, 8), 26)
    g = _rand((1, 2, 15, 8), 27)
    _, _, _, delta = oracle.attention_bwd(q, k, v, g, 0.5, True)
    o, _ = oracle.attention(q, k, v, 0.5, True)
    np.testing.assert_allclose(delta, (g.astype(np.float64) * o).sum(-1), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- key windows
def _forward64_window(q, k, v, scale, causal, wl, wr):
    """Windowed softmax(scale q k^T) v in float64; rows with no visible key give 0."""
    g = q.shape[1] // k.shape[1]
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    s = scale * np.einsum("bhid,bhjd->bhij", q, kr)
    i, j = np.meshgrid(np.arange(q.shape[2]), np.arange(k.shape[2]), indexing="ij")
    keep = np.ones_like(i, dtype=bool)
    if causal:
        keep &= j <= i
    if wl >= 0:
        keep &= j >= i - wl
    if wr >= 0:
        keep &= j <= i + wr
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m)
    z = p.sum(axis=-1, keepdims=True)
    p = np.divide(p, z, out=np.zeros_like(p), where=z > 0)
    return np.einsum("bhij,bhjd->bhid", p, vr)


@pytest.mark.parametrize("causal,wl,wr,nq,nk", [(False, 2, 1, 6, 7), (True, 3, -1, 7, 7),
                                                 (False, 1, 2, 9, 5)])  # the last: rows 7, 8 see no key
def test_window_finite_differences(causal, wl, wr, nq, nk):
    q, k, v = _rand((1, 2, nq, 3), 40), _rand((1, 1, nk, 3), 41), _rand((1, 1, nk, 3), 42)
    g = _rand((1, 2, nq, 3), 43)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.8, causal, window=(wl, wr))
    x = [q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)]
    o_or, _ = oracle.attention(q, k, v, 0.8, causal, window=(wl, wr))
    np.testing.assert_allclose(_forward64_window(*x, 0.8, causal, wl, wr), o_or, rtol=1e-12, atol=1e-13)
    h = 1e-5

    def loss(xs):
        return float(np.sum(g.astype(np.float64) * _forward64_window(*xs, 0.8, causal, wl, wr)))

    for which, grad in enumerate((dq, dk, dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += h
            xm[which][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal,wl,wr", [(False, 8, 4), (True, 16, -1), (False, -1, 10)])
def test_window_against_torch_autograd(causal, wl, wr):
    q, k, v = _rand((2, 4, 40, 8), 44), _rand((2, 2, 40, 8), 45), _rand((2, 2, 40, 8), 46)
    g = _rand((2, 4, 40, 8), 47)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.4, causal, window=(wl, wr))
    i, j = np.meshgrid(np.arange(40), np.arange(40), indexing="ij")
    keep = np.ones((40, 40), dtype=bool)
    if causal:
        keep &= j <= i
    if wl >= 0:
        keep &= j >= i - wl
    if wr >= 0:
        keep &= j <= i + wr
    qt, kt, vt = (torch.from_numpy(a).double().requires_grad_() for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(2, dim=1), vt.repeat_interleave(2, dim=1),
        attn_mask=torch.from_numpy(keep), scale=0.4)
    o.backward(torch.from_numpy(g).double())
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_window_special_cases():
    q, k, v = _rand((1, 2, 12, 4), 48), _rand((1, 2, 12, 4), 49), _rand((1, 2, 12, 4), 50)
    g = _rand((1, 2, 12, 4), 51)
    a = oracle.attention_bwd(q, k, v, g, 0.5, False, window=(-1, 0))
    b = oracle.attention_bwd(q, k, v, g, 0.5, True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    a = oracle.attention_bwd(q, k, v, g, 0.5, False, window=(50, 50))
    b = oracle.attention_bwd(q, k, v, g, 0.5, False)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    # (0, 0): O_i = v_i, so dV = dO and dQ = dK = 0
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.5, False, window=(0, 0))
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(dk, 0.0)
    np.testing.assert_array_equal(dv, g.astype(np.float64))


# ---- additive score bias (float attn_mask): P includes the bias

def _forward64_bias(q, k, v, scale, causal, bias):
    """softmax(scale q k^T + bias) v in float64; rows with no finite score -> 0."""
    g = q.shape[1] // k.shape[1]
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    s = scale * np.einsum("bhid,bhjd->bhij", q, kr) + bias
    if causal:
        i, j = np.meshgrid(np.arange(q.shape[2]), np.arange(k.shape[2]), indexing="ij")
        s = np.where(j <= i, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(s - m)
    z = p.sum(axis=-1, keepdims=True)
    p = np.divide(p, z, out=np.zeros_like(p), where=z > 0)
    return np.einsum("bhij,bhjd->bhid", p, vr)


@pytest.mark.parametrize("causal", [False, True])
def test_bias_finite_differences(causal):
    q, k, v = _rand((1, 2, 5, 3), 60), _rand((1, 1, 6, 3), 61), _rand((1, 1, 6, 3), 62)
    g = _rand((1, 2, 5, 3), 63)
    bias = _rand((1, 2, 5, 6), 64, 1.5).astype(np.float64)
    bias[0, 1, 2, 0] = -np.inf  # one removed key
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.7, causal, bias=bias.astype(np.float32))
    x = [q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)]
    bias32 = bias.astype(np.float32).astype(np.float64)
    o_or, _ = oracle.attention(q, k, v, 0.7, causal, bias=bias.astype(np.float32))
    np.testing.assert_allclose(_forward64_bias(*x, 0.7, causal, bias32), o_or, rtol=1e-12, atol=1e-13)
    h = 1e-5

    def loss(xs):
        return float(np.sum(g.astype(np.float64) * _forward64_bias(*xs, 0.7, causal, bias32)))

    for which, grad in enumerate((dq, dk, dv)):
        fd = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += h
            xm[which][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal,shape", [(False, (2, 4, 30, 36)), (True, (1, 1, 30, 36)),
                                          (False, (2, 1, 1, 36))])
def test_bias_against_torch_autograd(causal, shape):
    # full, shared [N, N] and key-padding shaped biases, with some -inf entries
    q, k, v = _rand((2, 4, 30, 8), 65), _rand((2, 2, 36, 8), 66), _rand((2, 2, 36, 8), 67)
    g = _rand((2, 4, 30, 8), 68)
    bias = _rand(shape, 69, 2.0)
    bias[np.random.default_rng(70).random(shape) < 0.15] = -np.inf
    bias[..., 0] = 0.0  # key 0 stays, so every row keeps a key
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.45, causal, bias=bias)
    qt, kt, vt = (torch.from_numpy(a).double().requires_grad_() for a in (q, k, v))
    mask = torch.from_numpy(bias).double().expand(2, 4, 30, 36)
    if causal:
        mask = mask.masked_fill(~torch.ones(30, 36, dtype=torch.bool).tril(), float("-inf"))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(2, dim=1), vt.repeat_interleave(2, dim=1), attn_mask=mask,
        scale=0.45)
    o.backward(torch.from_numpy(g).double())
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_bias_special_cases():
    q, k, v = _rand((1, 2, 10, 4), 71), _rand((1, 2, 12, 4), 72), _rand((1, 2, 12, 4), 73)
    g = _rand((1, 2, 10, 4), 74)
    # a bias that is constant along each row changes no probability: same gradients
    shift = _rand((1, 2, 10, 1), 75, 3.0) * np.ones((1, 1, 1, 12), dtype=np.float32)
    a = oracle.attention_bwd(q, k, v, g, 0.5, False, bias=shift)
    b = oracle.attention_bwd(q, k, v, g, 0.5, False)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-11, atol=1e-12)
    # -inf everywhere but key j = i: O_i = v_i, so dV = dO and dQ = dK = 0
    eye = np.full((1, 1, 10, 12), -np.inf, dtype=np.float32)
    eye[0, 0, np.arange(10), np.arange(10)] = 0.0
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, g, 0.5, False, bias=eye)
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(dk, 0.0)
    want = np.zeros_like(dv)
    want[:, :, :10] = g.astype(np.float64)
    np.testing.assert_array_equal(dv, want)
    # a row whose keys are all removed contributes nothing
    cut = np.zeros((1, 1, 10, 12), dtype=np.float32)
    cut[0, 0, 3] = -np.inf
    dq, dk, dv, delta = oracle.attention_bwd(q, k, v, g, 0.5, False, bias=cut)
    np.testing.assert_array_equal(dq[:, :, 3], 0.0)
    np.testing.assert_array_equal(delta[:, :, 3], 0.0)
    g2 = g.copy()
    g2[:, :, 3] = 0.0
    _, dk2, dv2, _ = oracle.attention_bwd(q, k, v, g2, 0.5, False, bias=cut)
    np.testing.assert_allclose(dk, dk2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv, dv2, rtol=1e-12, atol=1e-14)
