"""GPU parity of the unfused comparison path (fa_fwd_unfused: S and P through
device memory) against the fp64 oracle, and its agreement with the fused
kernel, on the same seeded inputs and tolerances as the fused path's tests
(fp16 O 4e-3, bf16 O 1.6e-2, LSE 1e-3)."""
import numpy as np
import pytest
import torch

import oracle
import tiled_attention_15_b200 as fa
from fa_inputs import Workload, llama7b, make_qkv

pytestmark = pytest.mark.gpu

TOL = {"fp16": (4e-3, 1e-3), "bf16": (1.6e-2, 1e-3)}

CASES = [
    Workload("unfused tiny D64", 1, 1, 1, 256, 256, 64, "fp16", False, seed=0),
    Workload("unfused ragged causal GQA D128", 2, 4, 2, 300, 300, 128, "fp16", True, seed=71),
    Workload("unfused Nq<Nk bf16 MQA D256", 1, 4, 1, 77, 513, 256, "bf16", False, seed=72),
    Workload("unfused causal Nq>Nk bf16 D64", 1, 2, 2, 600, 129, 64, "bf16", True, seed=73),
    Workload("unfused one key", 1, 2, 1, 5, 1, 128, "fp16", False, seed=74),
]


def _check(w, dev, q, k, v, o, lse):
    ref_o, ref_l = oracle.attention(q, k, v, w.softmax_scale, w.causal)
    do = np.abs(o.float().cpu().numpy() - ref_o).max()
    dl = np.abs(lse.cpu().numpy() - ref_l).max()
    to, tl = TOL[w.dtype]
    assert do <= to and dl <= tl, f"{w.name}: max|dO| {do:.3e}, max|dLSE| {dl:.3e}"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_unfused_matches_oracle(cuda_dev, w):
    q, k, v = make_qkv(w)
    o, lse = fa.fa_fwd_unfused(q.to(cuda_dev), k.to(cuda_dev), v.to(cuda_dev),
                               scale=w.softmax_scale, causal=w.causal)
    torch.cuda.synchronize()
    _check(w, cuda_dev, q, k, v, o, lse)


@pytest.mark.parametrize("causal", [False, True])
def test_unfused_llama7b_layer_and_fused_agree(cuda_dev, causal):
    w = llama7b(causal)
    q, k, v = make_qkv(w)
    qd, kd, vd = (x.to(cuda_dev) for x in (q, k, v))
    o, lse = fa.fa_fwd_unfused(qd, kd, vd, scale=w.softmax_scale, causal=causal)
    of, lf = fa.fa_fwd(qd, kd, vd, scale=w.softmax_scale, causal=causal)
    torch.cuda.synchronize()
    _check(w, cuda_dev, q, k, v, o, lse)
    # both within the oracle's tolerance, so within twice of each other
    assert (o.float() - of.float()).abs().max().item() <= 2 * TOL["fp16"][0]
    assert (lse - lf).abs().max().item() <= 2 * TOL["fp16"][1]
