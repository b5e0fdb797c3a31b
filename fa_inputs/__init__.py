"""Seeded synthetic inputs for the attention forward pass.

This module is shared by the oracle side and the CUDA side of every test and
benchmark.  It draws random numbers and rounds them to the storage dtype; it
holds none of the attention arithmetic itself.

Recipe (one reading of the workloads on the pages, stated once here):

* Q, K, V are drawn i.i.d. N(0, 1) in float32 from ``numpy.random.default_rng(seed)``
  in the order Q, K, V, with shapes ``[B, Hq, Nq, D]``, ``[B, Hkv, Nk, D]``,
  ``[B, Hkv, Nk, D]`` (contiguous BHND, the layout of the PyTorch call snippet
  in "通过 PyTorch 调用 FlashAttention" on the mooersco.com page).
* ``q_mult`` multiplies Q before rounding ("peaky" variant: scores 4x larger,
  so the running row maximum moves a lot between key blocks).
* ``outlier_frac`` > 0 then draws, per (b, kv-head), floor(outlier_frac * Nk)
  distinct key rows without replacement and multiplies those K rows by
  ``outlier_mult`` before rounding (outlier keys).
* The float32 values are rounded to the storage dtype (fp16 or bf16) with
  round-to-nearest-even by ``torch.Tensor.to``.  Both sides then see exactly
  the same rounded values: the CUDA side gets the 16-bit tensors, the oracle
  gets them widened (exactly) to float32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, dtype, flags and the input recipe."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    D: int
    dtype: str = "fp16"
    causal: bool = False
    seed: int = 0
    q_mult: float = 1.0
    outlier_frac: float = 0.0
    outlier_mult: float = 8.0
    scale: Optional[float] = None  # None -> 1/sqrt(D)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.D) if self.scale is None else float(self.scale)

    def flops(self) -> float:
        """Algorithmic FLOPs: 4*B*Hq*Nq*Nk*D, halved for causal (square case)."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.D
        return f / 2.0 if self.causal else f

    def io_bytes(self) -> int:
        """Algorithmic HBM bytes: read Q, K, V once, write O and the fp32 LSE once."""
        elt = 2
        return (elt * self.D * (2 * self.B * self.Hq * self.Nq + 2 * self.B * self.Hkv * self.Nk)
                + 4 * self.B * self.Hq * self.Nq)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def make_qkv(w: Workload):
    """Return (q, k, v) as contiguous CPU tensors of dtype ``w.dtype``."""
    rng = np.random.default_rng(w.seed)
    q = rng.standard_normal((w.B, w.Hq, w.Nq, w.D), dtype=np.float32)
    k = rng.standard_normal((w.B, w.Hkv, w.Nk, w.D), dtype=np.float32)
    v = rng.standard_normal((w.B, w.Hkv, w.Nk, w.D), dtype=np.float32)
    if w.q_mult != 1.0:
        q *= np.float32(w.q_mult)
    if w.outlier_frac > 0.0:
        n_out = int(math.floor(w.outlier_frac * w.Nk))
        for b in range(w.B):
            for h in range(w.Hkv):
                rows = rng.choice(w.Nk, size=n_out, replace=False)
                k[b, h, rows, :] *= np.float32(w.outlier_mult)
    dt = DTYPES[w.dtype]
    return (torch.from_numpy(q).to(dt), torch.from_numpy(k).to(dt), torch.from_numpy(v).to(dt))


def sample_rows(n: int, count: int, seed: int) -> np.ndarray:
    """Seeded sorted sample of query rows; always contains rows 0 and n-1."""
    if count >= n:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed + 7919)
    inner = rng.choice(np.arange(1, n - 1), size=max(count - 2, 0), replace=False)
    return np.unique(np.concatenate([[0, n - 1], inner]).astype(np.int64))


# The workloads the pages measure on, restated with their sizes.
TINY = Workload("tiny B1 H1 N256 D64 fp16", 1, 1, 1, 256, 256, 64, "fp16", False, 0)
LLAMA7B = Workload("llama7b-attn B2 H32 N2048 D128 fp16", 2, 32, 32, 2048, 2048, 128, "fp16", False, 0)


def llama7b(causal: bool, peaky: bool = False) -> Workload:
    w = LLAMA7B.with_(causal=causal, q_mult=4.0 if peaky else 1.0)
    return w.with_(name=f"llama7b-attn B2 H32 N2048 D128 fp16 {'causal' if causal else 'noncausal'}"
                        + (" peaky" if peaky else ""))


SWEEP_SEEDS = (1, 2, 3, 4)


def seq_sweep(n: int, causal: bool, seed: Optional[int] = None) -> Workload:
    """Sequence sweep workload; the default seed is the k-th of 1-4 for the k-th length."""
    if seed is None:
        seed = {512: 1, 2048: 2, 4096: 3, 8192: 4}[n]
    return Workload(f"sweep B1 H32 N{n} D128 fp16 {'causal' if causal else 'noncausal'} seed{seed}",
                    1, 32, 32, n, n, 128, "fp16", causal, seed)


def gqa(hkv: int, d: int) -> Workload:
    return Workload(f"gqa B4 Hq32 Hkv{hkv} N8192 D{d} bf16 causal", 4, 32, hkv, 8192, 8192, d,
                    "bf16", True, 0)


LONG = Workload("long B1 Hq32 Hkv8 N131072 D128 bf16 causal outliers", 1, 32, 8, 131072, 131072, 128,
                "bf16", True, 0, outlier_frac=0.01, outlier_mult=8.0)


def all_configs() -> Sequence[Workload]:
    out = [TINY]
    for c in (False, True):
        out.append(llama7b(c))
        out.append(llama7b(c, peaky=True))
    for n in (512, 2048, 4096, 8192):
        for c in (False, True):
            out.append(seq_sweep(n, c))
    for hkv, d in ((8, 128), (1, 128), (8, 64), (8, 256)):
        out.append(gqa(hkv, d))
    out.append(LONG)
    return out
