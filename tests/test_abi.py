"""C-ABI tests that need no GPU: the library loads, exports every function
include/fa.h declares, and rejects bad arguments on the host before any CUDA
work (fake, never-dereferenced pointer values are enough for that)."""
import ctypes
import os
import re
import subprocess

import pytest

import tiled_attention_15_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    from tiled_attention_15_b200.csrc import build
    build.build()
    return fa.load_library()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_binding_names():
    assert sorted(fa.EXPORTED) == _declared()


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z0-9_]+)$", out, flags=re.M))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code in range(0, 17):
        s = fa.status_string(code)
        assert s and s != "unknown status", code
    assert fa.status_string(99) == "unknown status"


def test_num_tiles(lib):
    # 256 query rows per work tile for D <= 128, 128 for D = 256
    assert fa.num_tiles(2, 32, 2048, 128) == 2 * 32 * 8
    assert fa.num_tiles(1, 1, 257, 64) == 2
    assert fa.num_tiles(1, 2, 129, 256) == 4
    assert fa.num_tiles(1, 1, 1, 96) == 0


A = 1 << 20  # fake 16-byte-aligned addresses, far apart; never dereferenced
GOOD = dict(q=1 * A, k=2 * A, v=3 * A, o=4 * A, lse=5 * A, B=1, Hq=4, Hkv=2, Nq=64, Nk=64, D=128,
            scale=0.125, causal=0, stream=0, dtype=fa.FA_FP16)


def _call(**kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_raw(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                         a["Nq"], a["Nk"], a["D"], a["scale"], a["causal"], a["stream"], a["dtype"])


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), 7),
    (dict(D=96), 5), (dict(D=32), 5), (dict(D=0), 5),
    (dict(B=0), 3), (dict(Hq=0), 3), (dict(Hkv=0), 3), (dict(Nq=0), 3), (dict(Nk=-1), 3),
    (dict(Hq=6, Hkv=4), 4),
    (dict(scale=float("nan")), 6), (dict(scale=float("inf")), 6),
    (dict(q=0), 1), (dict(o=0), 1),
    (dict(k=2 * A + 8), 2), (dict(lse=5 * A + 2), 2),
    (dict(o=1 * A + 64), 12), (dict(lse=3 * A + 32), 12),
])
def test_host_argument_checks(lib, kw, code):
    assert _call(**kw) == code


def test_valid_arguments_reach_the_device_check(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check")
    assert _call() == 8  # FA_ERR_NO_DEVICE without a GPU
    assert _call(lse=0) == 8  # lse may be NULL


def test_workspace_entry_point_host_checks(lib):
    a = dict(GOOD)
    args = (a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
            a["D"], ctypes.c_float(a["scale"]), a["causal"], None, a["dtype"])
    assert lib.fa_fwd_ws(*args, 7 * A + 128, 1 << 20) == 2  # workspace not 256-byte aligned
    assert lib.fa_fwd_ws(*args[:10], 96, *args[11:], 7 * A, 1 << 20) == 5  # head_dim checked first
    assert fa.set_max_ctas(-1) == 3
    assert fa.set_max_ctas(0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(dtype=2), 7), (dict(D=96), 5), (dict(B=0), 3), (dict(Hq=6, Hkv=4), 4),
    (dict(scale=float("nan")), 6), (dict(q=0), 1), (dict(k=2 * A + 8), 2), (dict(o=1 * A + 64), 12),
])
def test_noalloc_entry_point_host_checks(lib, kw, code):
    """fa_fwd_noalloc rejects bad arguments on the host, before its scratch lookup."""
    a = dict(GOOD)
    a.update(kw)
    assert lib.fa_fwd_noalloc(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                              a["Nq"], a["Nk"], a["D"], ctypes.c_float(a["scale"]), a["causal"],
                              None, a["dtype"]) == code


def test_unfused_entry_point_host_checks(lib):
    a = dict(GOOD)
    need = int(lib.fa_fwd_unfused_workspace_size(a["B"], a["Hq"], a["Nq"], a["Nk"]))
    assert need == 256 * ((a["B"] * a["Hq"] * a["Nq"] * a["Nk"] * 4 + 255) // 256) + \
        256 * ((a["B"] * a["Hq"] * a["Nq"] * a["Nk"] * 2 + 255) // 256)
    assert lib.fa_fwd_unfused_workspace_size(0, 1, 1, 1) == 0

    def call(ws=7 * A, nbytes=need, **kw):
        b = dict(a)
        b.update(kw)
        return lib.fa_fwd_unfused(b["q"], b["k"], b["v"], b["o"], b["lse"], b["B"], b["Hq"],
                                  b["Hkv"], b["Nq"], b["Nk"], b["D"], ctypes.c_float(b["scale"]),
                                  b["causal"], None, b["dtype"], ws, nbytes)
    bad_ws = fa.FA_ERR_BAD_WORKSPACE
    assert call(ws=None) == bad_ws
    assert call(nbytes=need - 1) == bad_ws
    assert call(ws=7 * A + 16) == bad_ws
    assert call(D=96) == 5 and call(dtype=2) == 7 and call(Hq=6, Hkv=4) == 4
    assert call(q=0) == 1 and call(k=2 * A + 8) == 2 and call(o=1 * A + 64) == 12
    import torch
    if not torch.cuda.is_available():
        assert call() == 8  # valid arguments reach the device check


def test_window_entry_point_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(wl, wr, causal=0, ws=None, dtype=a["dtype"], D=a["D"]):
        return lib.fa_fwd_window(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                                 a["Hkv"], a["Nq"], a["Nk"], D, ctypes.c_float(a["scale"]),
                                 causal, wl, wr, None, dtype, ws, 0)
    bad = fa.FA_ERR_BAD_WINDOW
    assert call(-2, 3) == bad and call(4, -2) == bad
    assert call(8, 1, causal=1) == bad  # causal fixes the right bound at 0
    assert call(8, 0, ws=7 * A + 128) == 2  # workspace not 256-byte aligned
    assert call(8, 0, dtype=5) == 7 and call(8, 0, D=80) == 5
    if not torch.cuda.is_available():
        for wl, wr, causal in ((-1, -1, 0), (0, 0, 0), (16, -1, 1), (16, 0, 1), (3, 7, 0)):
            assert call(wl, wr, causal) == 8  # valid: reaches the device check


def test_bias_entry_point_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(bias=9 * A, sb=0, sh=0, sq=64, D=a["D"]):
        return lib.fa_fwd_bias(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                               a["Nq"], a["Nk"], D, ctypes.c_float(a["scale"]), 0, bias, sb, sh, sq,
                               None, a["dtype"])
    assert call(bias=None) == 1
    assert call(sq=-8) == 3
    assert call(bias=9 * A + 8) == 2 and call(sq=63) == 2 and call(sh=4) == 2
    assert call(bias=4 * A + 256) == 12  # overlaps o
    if not torch.cuda.is_available():
        assert call() == 8 and call(sb=4096, sh=64 * 64, sq=64) == 8



def test_bias_window_entry_point_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(wl=-1, wr=-1, causal=0, bias=9 * A):
        return lib.fa_fwd_bias_window(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                                      a["Hkv"], a["Nq"], a["Nk"], a["D"], ctypes.c_float(a["scale"]),
                                      causal, bias, 0, 0, 64, wl, wr, None, a["dtype"])
    assert call(bias=None) == 1
    assert call(wl=-2) == 14 and call(wr=-3) == 14 and call(wl=4, wr=2, causal=1) == 14
    if not torch.cuda.is_available():
        for wl, wr, causal in ((-1, -1, 0), (16, -1, 1), (3, 7, 0), (0, 0, 0)):
            assert call(wl, wr, causal) == 8  # valid: reaches the device check


def test_bwd_bias_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(D=128, bias=13 * A, sq=64, ws=12 * A, dq=9 * A):
        return lib.fa_bwd_bias(a["q"], a["k"], a["v"], 6 * A, 7 * A, 8 * A, dq, 10 * A, 11 * A,
                               a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], D,
                               ctypes.c_float(a["scale"]), 0, bias, 0, 0, sq, None, a["dtype"], ws,
                               1 << 20)
    assert call(bias=None) == 1
    assert call(sq=-8) == 3
    assert call(bias=13 * A + 8) == 2 and call(sq=60) == 2
    assert call(D=256) == 5                # no bias tile room at head_dim 256
    assert call(bias=9 * A) == 12          # dq overlaps the bias
    assert call(bias=12 * A + 1024) == 12  # the workspace overlaps the bias
    if not torch.cuda.is_available():
        assert call() == 8 and call(D=64) == 8


def test_bias_ws_entry_point_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(ws=14 * A, bias=9 * A, causal=0, wl=-1):
        return lib.fa_fwd_bias_ws(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                                  a["Hkv"], a["Nq"], a["Nk"], a["D"], ctypes.c_float(a["scale"]),
                                  causal, bias, 0, 0, 64, wl, -1, None, a["dtype"], ws, 1 << 20)
    assert call(bias=None) == 1
    assert call(ws=14 * A + 128) == 2          # workspace not 256-byte aligned
    assert call(ws=9 * A - 4096) == 12         # the workspace overlaps the bias
    assert call(wl=-2) == 14
    if not torch.cuda.is_available():
        assert call() == 8 and call(ws=None) == 8 and call(wl=16, causal=1) == 8


def test_bwd_bias_window_host_checks(lib):
    import torch
    a = dict(GOOD)

    def call(wl=-1, wr=-1, causal=0, D=128):
        return lib.fa_bwd_bias_window(a["q"], a["k"], a["v"], 6 * A, 7 * A, 8 * A, 9 * A, 10 * A,
                                      11 * A, a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], D,
                                      ctypes.c_float(a["scale"]), causal, 13 * A, 0, 0, 64, wl, wr,
                                      None, a["dtype"], 12 * A, 1 << 20)
    assert call(wl=-2) == 14 and call(wr=3, causal=1) == 14
    assert call(D=256) == 5
    if not torch.cuda.is_available():
        assert call() == 8 and call(wl=32, causal=1) == 8 and call(wl=5, wr=7) == 8


def test_bwd_window_host_checks(lib):
    a = dict(GOOD)

    def call(wl, wr, causal=0):
        return lib.fa_bwd_window(a["q"], a["k"], a["v"], 6 * A, 7 * A, 8 * A, 9 * A, 10 * A, 11 * A,
                                 a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["D"],
                                 ctypes.c_float(a["scale"]), causal, wl, wr, None, a["dtype"],
                                 12 * A, 1 << 20)
    assert call(-2, 0) == fa.FA_ERR_BAD_WINDOW and call(3, -5) == fa.FA_ERR_BAD_WINDOW
    assert call(8, 2, causal=1) == fa.FA_ERR_BAD_WINDOW


def test_python_binding_argument_checks(lib):
    """The binding's own checks run before any CUDA call (argument marshalling only)."""
    import torch
    q = torch.zeros(1, 2, 16, 64, dtype=torch.float16)
    k = torch.zeros(1, 2, 16, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        fa.fa_fwd(q.float(), k.float(), k.float())
    with pytest.raises(TypeError):
        fa.fa_fwd(q, k.bfloat16(), k)
    with pytest.raises(ValueError):
        fa.fa_fwd(q[0], k[0], k[0])  # not 4-D
    with pytest.raises(ValueError):
        fa.fa_fwd(q, k, k)  # CPU tensors
    lse = torch.zeros(1, 2, 16)
    with pytest.raises(ValueError):
        fa.fa_bwd(q, k, k, q, lse, q)  # CPU tensors
    with pytest.raises(TypeError):
        fa.fa_bwd(q, k, k, q, lse.double(), q)  # lse must be float32
    if not torch.cuda.is_available():
        with pytest.raises(TypeError):
            fa._bias_view(torch.zeros(1, 1, 16, 16, dtype=torch.float16), torch.float16, 1, 2, 16, 16)


def test_size_limits_are_rejected_on_the_host(lib):
    # work-tile counts, row indices and TMA coordinates are 32-bit: sizes whose
    # B * H * N reaches 2^31 are refused before anything is enqueued
    assert _call(B=1 << 16, Hq=1 << 8, Hkv=1 << 8, Nq=1 << 8, Nk=64) == 3
    assert _call(B=1 << 16, Hq=4, Hkv=2, Nq=64, Nk=1 << 15) == 3


def test_bwd_host_checks(lib):
    a = dict(GOOD)

    def call(D=128, ws=12 * A, ws_bytes=1 << 20, dq=9 * A, dtype=a["dtype"], lse=8 * A):
        return lib.fa_bwd(a["q"], a["k"], a["v"], 6 * A, 7 * A, lse, dq, 10 * A, 11 * A, a["B"],
                          a["Hq"], a["Hkv"], a["Nq"], a["Nk"], D, ctypes.c_float(a["scale"]), 0,
                          None, dtype, ws, ws_bytes)
    assert call(D=96) == 5               # backward: head_dim 64, 128 or 256
    assert call(dtype=3) == 7
    assert call(ws=None) == fa.FA_ERR_BAD_WORKSPACE
    assert call(ws_bytes=16) == fa.FA_ERR_BAD_WORKSPACE
    assert call(ws=12 * A + 128) == 2   # workspace not 256-byte aligned
    assert call(lse=8 * A + 2) == 2
    assert call(dq=1 * A) == 12          # dq overlaps q
    assert call(lse=None) == 1
    assert lib.fa_bwd_workspace_size(1, 4, 64) == 2 * 4 * 128 * 4
    assert lib.fa_bwd_workspace_size(0, 4, 64) == 0
