"""fa_fwd_noalloc: the split-tail forward whose scratch is a static device array.

Some callers cannot allocate device memory: a serving engine whose memory pool
already owns all free device memory, or a plug-in interface that hands the
library only its inputs and outputs.  fa_fwd_noalloc serves them: it allocates
nothing and keeps the split tail's scratch in a file-scope device array.

Each case calls it through the C ABI twice in a row and checks both results
against the existing workspace entry point (fa_fwd_ws with a caller-allocated
workspace of fa_fwd_workspace_size bytes): within the parity tolerances of the
other GPU tests, and in fact bit for bit, since both take the same split and
merge in the same fixed order.  The cases
include shapes whose last round of tiles is split and a decode shape split
stream-K (so the static scratch is really used), and a causal one (no split).  The file name makes pytest collect
it last, so a failure here leaves every other test already run.
"""
import ctypes

import pytest
import torch

import tiled_attention_15_b200 as fa
from fa_inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu

TOL = {"fp16": 4e-3, "bf16": 1.6e-2}

CASES = [
    # (workload, CTA cap): 512 tiles on 148 SMs leave a 68-tile last round -> split
    (Workload("N4096 D128 fp16 non-causal", 1, 32, 32, 4096, 4096, 128, "fp16", False, seed=3), 0),
    # capped at 8 CTAs: 20 tiles -> a 4-tile last round -> split; ragged Nq, GQA, bf16
    (Workload("capped D128 bf16 GQA ragged", 1, 10, 5, 300, 3500, 128, "bf16", False, seed=41), 8),
    (Workload("capped D256 fp16", 1, 5, 5, 512, 3072, 256, "fp16", False, seed=42), 8),
    (Workload("causal D64 bf16 (no split)", 2, 8, 2, 1000, 1000, 64, "bf16", True, seed=43), 0),
    # 32 packed decode tiles on 148 SMs: stream-K partials in the static scratch
    (Workload("decode GQA4 Nq1 D128 bf16 stream-K", 4, 32, 8, 1, 8192, 128, "bf16", False, seed=44), 0),
]


def _c_call(fn, q, k, v, o, lse, w, *extra):
    stream = torch.cuda.current_stream().cuda_stream or None
    dtype = fa.FA_BF16 if w.dtype == "bf16" else fa.FA_FP16
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.Hq,
              w.Hkv, w.Nq, w.Nk, w.D, ctypes.c_float(w.softmax_scale), int(w.causal), stream,
              dtype, *extra)


@pytest.mark.parametrize("w,cap", CASES, ids=lambda c: c.name if hasattr(c, "name") else str(c))
def test_noalloc_matches_workspace_entry_point(cuda_dev, w, cap):
    lib = fa.load_library()
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    prev = fa.set_max_ctas(cap)
    try:
        # the existing entry point, with a caller-allocated, zero-filled workspace
        size = int(lib.fa_fwd_workspace_size(w.D))
        assert size > 0
        ws = torch.zeros(size, dtype=torch.uint8, device=cuda_dev)
        o_ref = torch.empty_like(q)
        l_ref = torch.empty(q.shape[:3], dtype=torch.float32, device=cuda_dev)
        assert _c_call(lib.fa_fwd_ws, q, k, v, o_ref, l_ref, w, ws.data_ptr(), size) == fa.FA_OK
        torch.cuda.synchronize()
        assert size <= int(lib.fa_fwd_noalloc_scratch_bytes())
        for call in range(2):  # two calls in a row share the static scratch
            o = torch.full_like(q, float("nan"))
            lse = torch.full_like(l_ref, float("nan"))
            assert _c_call(lib.fa_fwd_noalloc, q, k, v, o, lse, w) == fa.FA_OK, call
            torch.cuda.synchronize()
            assert fa.device_status(reset=True) == fa.FA_OK
            assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
            assert (o.float() - o_ref.float()).abs().max().item() <= TOL[w.dtype], call
            assert (lse - l_ref).abs().max().item() <= 1e-3, call
            assert torch.equal(o, o_ref) and torch.equal(lse, l_ref), call
    finally:
        fa.set_max_ctas(prev)
