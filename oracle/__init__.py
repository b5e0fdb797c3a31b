"""Oracle for the attention forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (``tiled_attention_15_b200``)
never imports it, and it never imports the product path.

``attention(q, k, v, scale, causal, rows=None)`` is the plain three-pass
definition of attention in double precision (S = scale*Q K^T, row softmax,
times V), written in C (``attn_oracle.c``) and run on the host cores with
OpenMP.  Source of the definition: the "standard attention" steps on the
mooersco.com page (section "标准 Attention 的瓶颈在哪") and section 二 of the
gitcode.csdn.net page; the scale 1/sqrt(head_dim) from the Scale step of the
hwcomputing.csdn.net page's fused-kernel listing.  Every function of this
package is pinned by ``tests/test_oracle.py`` against values fixed by the pages
and by mathematics (see that file's header); nothing here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` with gcc (-O2 -fopenmp, no fast-math) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
            ctypes.c_int]
        lib.oracle_attention_ex.restype = ctypes.c_int
        lib.oracle_attention_ex.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int]
        lib.oracle_attention_bwd_ex.restype = ctypes.c_int
        lib.oracle_attention_bwd_ex.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
        lib.oracle_attention_bwd.restype = ctypes.c_int
        lib.oracle_attention_bwd.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int64] * 6 + [
            ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _as_f32(x) -> np.ndarray:
    """Widen a (rounded fp16/bf16) tensor or array to a contiguous float32 numpy array (exact)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu").float().numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def attention(q, k, v, scale: float, causal: bool, rows: Optional[np.ndarray] = None,
              nthreads: int = 0, window: Tuple[int, int] = (-1, -1),
              bias=None) -> Tuple[np.ndarray, np.ndarray]:
    """Reference attention in float64.

    q: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D] (torch tensors or numpy arrays).
    rows: optional sorted int64 array of query positions; only those rows are
    computed (then the result has R = len(rows) rows per head).
    window: (left, right): key j is visible to query i iff i - left <= j <= i + right;
    a negative bound is no bound (causal is right = 0).
    bias: optional additive score bias broadcastable to [B, Hq, Nq, Nk] (float32
    values; -inf removes a key).  A row with no key left gets O = 0, LSE = -inf.
    Returns (O [B, Hq, R, D] float64, LSE [B, Hq, R] float64).
    """
    lib = _load()
    qf, kf, vf = _as_f32(q), _as_f32(k), _as_f32(v)
    B, Hq, Nq, D = qf.shape
    Bk, Hkv, Nk, Dk = kf.shape
    if (Bk, Dk) != (B, D) or vf.shape != kf.shape:
        raise ValueError("shape mismatch between q, k, v")
    if rows is not None:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        if rows.ndim != 1 or rows.size == 0 or rows.min() < 0 or rows.max() >= Nq:
            raise ValueError("rows must be a non-empty 1-D array of positions in [0, Nq)")
        qf = np.ascontiguousarray(qf[:, :, rows, :])
        R = int(rows.shape[0])
        pos_ptr = rows.ctypes.data
    else:
        R = Nq
        pos_ptr = None
    o = np.empty((B, Hq, R, D), dtype=np.float64)
    lse = np.empty((B, Hq, R), dtype=np.float64)
    bf, bias_ptr, sb, sh, sq = _bias_args(bias, B, Hq, Nq, Nk)
    wl, wr = (int(x) for x in window)
    rc = lib.oracle_attention_ex(qf.ctypes.data, pos_ptr, R, kf.ctypes.data, vf.ctypes.data,
                                 o.ctypes.data, lse.ctypes.data, B, Hq, Hkv, Nq, Nk, D,
                                 float(scale), int(bool(causal)), wl, wr, bias_ptr, sb, sh, sq,
                                 int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attention rejected its arguments (code {rc})")
    return o, lse


def _bias_args(bias, B, Hq, Nq, Nk):
    """(array kept alive, pointer, stride_b, stride_h, stride_q) of a bias that
    broadcasts to [B, Hq, Nq, Nk]; all None / 0 without a bias."""
    if bias is None:
        return None, None, 0, 0, 0
    bf = _as_f32(bias)
    while bf.ndim < 4:
        bf = bf[None]
    if bf.ndim != 4 or bf.shape[3] != Nk or any(
            n not in (1, full) for n, full in zip(bf.shape[:3], (B, Hq, Nq))):
        raise ValueError("bias must broadcast to [B, Hq, Nq, Nk] with its last dim Nk")
    bf = np.ascontiguousarray(bf)
    # element strides; a broadcast dim gets stride 0
    st = [0 if bf.shape[d] == 1 else int(np.prod(bf.shape[d + 1:])) for d in range(3)]
    return bf, bf.ctypes.data, st[0], st[1], st[2]


def attention_bwd(q, k, v, dout, scale: float, causal: bool, nthreads: int = 0,
                  window: Tuple[int, int] = (-1, -1), bias=None):
    """Gradients of attention in float64 for the upstream gradient dout.

    q, dout: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D] (torch tensors or numpy arrays).
    window: (left, right) key window as in attention(); rows with no visible
    key contribute nothing.
    bias: optional additive score bias as in attention() (a given input: the
    gradients are those of Q, K and V).
    Returns (dQ [B, Hq, Nq, D], dK [B, Hkv, Nk, D], dV [B, Hkv, Nk, D],
    Delta [B, Hq, Nq]) as float64 numpy arrays; Delta_i = dO_i . O_i.
    """
    lib = _load()
    qf, kf, vf, gf = _as_f32(q), _as_f32(k), _as_f32(v), _as_f32(dout)
    B, Hq, Nq, D = qf.shape
    Bk, Hkv, Nk, Dk = kf.shape
    if (Bk, Dk) != (B, D) or vf.shape != kf.shape or gf.shape != qf.shape:
        raise ValueError("shape mismatch between q, k, v, dout")
    dq = np.empty((B, Hq, Nq, D), dtype=np.float64)
    dk = np.empty((B, Hkv, Nk, D), dtype=np.float64)
    dv = np.empty((B, Hkv, Nk, D), dtype=np.float64)
    delta = np.empty((B, Hq, Nq), dtype=np.float64)
    wl, wr = (int(x) for x in window)
    bf, bias_ptr, sb, sh, sq = _bias_args(bias, B, Hq, Nq, Nk)
    rc = lib.oracle_attention_bwd_ex(qf.ctypes.data, kf.ctypes.data, vf.ctypes.data,
                                     gf.ctypes.data, dq.ctypes.data, dk.ctypes.data,
                                     dv.ctypes.data, delta.ctypes.data, B, Hq, Hkv, Nq, Nk, D,
                                     float(scale), int(bool(causal)), wl, wr, bias_ptr, sb, sh,
                                     sq, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attention_bwd rejected its arguments (code {rc})")
    return dq, dk, dv, delta
