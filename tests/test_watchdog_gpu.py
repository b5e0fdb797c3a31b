"""Failure detection of the kernels' waits, without hanging or faulting the GPU.

The diagnostic entry point runs the kernels' own bounded mbarrier wait on a
barrier that nothing arrives on.  The wait must give up after its limit, record
FA_ERR_DEVICE_TIMEOUT and the site (CTA 0, warp 0), and return; the context stays
usable, which the attention call afterwards checks."""
import time

import pytest
import torch

import tiled_attention_15_b200 as fa
from fa_inputs import Workload, make_qkv

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(cuda_dev):
    lib = fa.load_library()
    assert fa.device_status(reset=True) == fa.FA_OK
    t0 = time.time()
    assert lib.fa_debug_wait_timeout(torch.cuda.current_stream().cuda_stream or None) == fa.FA_OK
    assert fa.device_status() == fa.FA_ERR_DEVICE_TIMEOUT
    elapsed = time.time() - t0
    assert 0.5 < elapsed < 30.0
    cta, warp, bar_addr, parity = fa.timeout_site()
    assert (cta, warp, parity) == (0, 0, 0)
    assert fa.device_status(reset=True) == fa.FA_ERR_DEVICE_TIMEOUT
    assert fa.device_status() == fa.FA_OK and fa.timeout_site() is None
    # the context is still usable
    w = Workload("after", 1, 2, 2, 256, 256, 64, "fp16", True, seed=9)
    q, k, v = (x.to(cuda_dev) for x in make_qkv(w))
    o, lse = fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and fa.device_status() == fa.FA_OK
