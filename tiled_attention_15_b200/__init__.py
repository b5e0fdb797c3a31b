"""Python binding of the B200 fused attention forward library (``libfa.so``).

Argument marshalling only: every step of the attention forward pass runs in the
CUDA kernels behind the C ABI declared in ``include/fa.h``.  PyTorch supplies
device memory and the current stream.  There is no fallback: if the library is
missing, importing the functions raises.

    from tiled_attention_15_b200 import fa_fwd
    o, lse = fa_fwd(q, k, v, causal=True)          # q,k,v: cuda fp16/bf16 [B,H,N,D]
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_FP16, FA_BF16 = 0, 1
FA_OK = 0
FA_ERR_DEVICE_TIMEOUT = 11
FA_ERR_BAD_WINDOW = 14
FA_ERR_BAD_WORKSPACE = 15

# Every symbol include/fa.h declares (checked by the tests).
EXPORTED = ("fa_fwd", "fa_fwd_fp16", "fa_fwd_bf16", "fa_fwd_ws", "fa_fwd_workspace_size",
            "fa_fwd_window", "fa_fwd_bias", "fa_fwd_bias_window", "fa_fwd_bias_ws", "fa_bwd", "fa_bwd_window", "fa_bwd_bias", "fa_bwd_bias_window",
            "fa_bwd_workspace_size",
            "fa_fwd_noalloc", "fa_fwd_noalloc_scratch_bytes", "fa_set_max_ctas",
            "fa_fwd_unfused", "fa_fwd_unfused_workspace_size",
            "fa_status_string", "fa_device_status", "fa_device_timeout_site",
            "fa_debug_exp2_fma", "fa_debug_wait_timeout", "fa_fwd_num_tiles")


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: status {code} ({status_string(code)})")


_lib = None


def load_library() -> ctypes.CDLL:
    """Load libfa.so (built by ``python -m tiled_attention_15_b200.csrc.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run python -m tiled_attention_15_b200.csrc.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fwd_args = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
    lib.fa_fwd.argtypes = fwd_args + [i]
    lib.fa_fwd.restype = i
    for name in ("fa_fwd_fp16", "fa_fwd_bf16"):
        getattr(lib, name).argtypes = fwd_args
        getattr(lib, name).restype = i
    lib.fa_fwd_ws.argtypes = fwd_args + [i, vp, ctypes.c_size_t]
    lib.fa_fwd_ws.restype = i
    lib.fa_fwd_window.argtypes = fwd_args[:13] + [i, i, vp, i, vp, ctypes.c_size_t]
    lib.fa_fwd_window.restype = i
    ll = ctypes.c_longlong
    lib.fa_fwd_bias.argtypes = fwd_args[:13] + [vp, ll, ll, ll, vp, i]
    lib.fa_fwd_bias.restype = i
    lib.fa_fwd_bias_window.argtypes = fwd_args[:13] + [vp, ll, ll, ll, i, i, vp, i]
    lib.fa_fwd_bias_window.restype = i
    lib.fa_fwd_bias_ws.argtypes = fwd_args[:13] + [vp, ll, ll, ll, i, i, vp, i, vp,
                                                    ctypes.c_size_t]
    lib.fa_fwd_bias_ws.restype = i
    lib.fa_bwd.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, i, vp, i, vp, ctypes.c_size_t]
    lib.fa_bwd.restype = i
    lib.fa_bwd_window.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, i, i, i, vp, i, vp, ctypes.c_size_t]
    lib.fa_bwd_window.restype = i
    lib.fa_bwd_bias.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, i, vp, ll, ll, ll, vp, i, vp,
                                           ctypes.c_size_t]
    lib.fa_bwd_bias.restype = i
    lib.fa_bwd_bias_window.argtypes = [vp] * 9 + [i, i, i, i, i, i, f, i, vp, ll, ll, ll, i, i, vp,
                                                  i, vp, ctypes.c_size_t]
    lib.fa_bwd_bias_window.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_noalloc.argtypes = fwd_args + [i]
    lib.fa_fwd_noalloc.restype = i
    lib.fa_fwd_noalloc_scratch_bytes.argtypes = []
    lib.fa_fwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_unfused.argtypes = fwd_args + [i, vp, ctypes.c_size_t]
    lib.fa_fwd_unfused.restype = i
    lib.fa_fwd_unfused_workspace_size.argtypes = [i, i, i, i]
    lib.fa_fwd_unfused_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_workspace_size.argtypes = [i]
    lib.fa_fwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_set_max_ctas.argtypes = [i]
    lib.fa_set_max_ctas.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_device_status.argtypes = [i]
    lib.fa_device_status.restype = i
    lib.fa_device_timeout_site.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    lib.fa_device_timeout_site.restype = i
    lib.fa_debug_wait_timeout.argtypes = [vp]
    lib.fa_debug_wait_timeout.restype = i
    lib.fa_debug_exp2_fma.argtypes = [vp, vp, i, vp]
    lib.fa_debug_exp2_fma.restype = i
    lib.fa_fwd_num_tiles.argtypes = [i, i, i, i]
    lib.fa_fwd_num_tiles.restype = ctypes.c_longlong
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().fa_status_string(int(code)).decode()


def device_status(reset: bool = False) -> int:
    """FA_OK, or FA_ERR_DEVICE_TIMEOUT if a kernel gave up on a wait (synchronises the device)."""
    return int(load_library().fa_device_status(1 if reset else 0))


def timeout_site():
    """(cta, warp, mbarrier shared address, parity) of the first timed-out wait, or None."""
    v = ctypes.c_ulonglong(0)
    rc = load_library().fa_device_timeout_site(ctypes.byref(v))
    if rc != FA_OK:
        raise FaError(rc, "fa_device_timeout_site")
    x = v.value
    if x == 0:
        return None
    return (x >> 48, (x >> 40) & 0xFF, (x >> 8) & 0xFFFFF, x & 1)


def exp2_fma(x):
    """2^x by the softmax's FMA-pipe approximation (diagnostics); x: float32 CUDA tensor."""
    import torch
    x = x.contiguous()
    y = torch.empty_like(x)
    rc = load_library().fa_debug_exp2_fma(x.data_ptr(), y.data_ptr(), x.numel(),
                                          torch.cuda.current_stream(x.device).cuda_stream or None)
    if rc != FA_OK:
        raise FaError(rc, "fa_debug_exp2_fma")
    return y


def num_tiles(B: int, Hq: int, Nq: int, D: int) -> int:
    return int(load_library().fa_fwd_num_tiles(B, Hq, Nq, D))


def set_max_ctas(n: int) -> int:
    """Cap the CTAs a launch uses (0 = one per SM); returns the previous cap."""
    return int(load_library().fa_set_max_ctas(int(n)))


_workspaces = {}


def workspace(device, stream_handle: int):
    """Zero-filled workspace for fa_fwd_ws, one per (device, stream), large enough for any D."""
    import torch
    key = (device.index, int(stream_handle or 0))
    ws = _workspaces.get(key)
    if ws is None:
        lib = load_library()
        with torch.cuda.device(device):
            size = max(int(lib.fa_fwd_workspace_size(d)) for d in (64, 128, 256))
        if size == 0:
            raise FaError(8, "fa_fwd_workspace_size")
        ws = torch.zeros(size, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def fa_fwd_raw(q: int, k: int, v: int, o: int, lse: Optional[int], B: int, Hq: int, Hkv: int,
               Nq: int, Nk: int, D: int, scale: float, causal: bool, stream: int,
               dtype: int) -> int:
    """The C entry point with plain integers for pointers; returns the status code."""
    return int(load_library().fa_fwd(q, k, v, o, lse or None, B, Hq, Hkv, Nq, Nk, D,
                                     ctypes.c_float(scale), 1 if causal else 0, stream or None,
                                     dtype))


def fa_fwd(q, k, v, o=None, lse=None, scale: Optional[float] = None, causal: bool = False,
           return_lse: bool = True, stream=None, use_workspace: bool = True,
           window: Tuple[int, int] = (-1, -1), bias=None) -> Tuple[object, Optional[object]]:
    """Fused attention forward on the current CUDA stream.

    q: [B, Hq, Nq, D], k/v: [B, Hkv, Nk, D] contiguous CUDA tensors, fp16 or bf16.
    o: optional output like q; lse: optional float32 [B, Hq, Nq] output.
    scale defaults to 1/sqrt(D).  use_workspace: call fa_fwd_ws with a cached
    per-(device, stream) workspace (load balance), else fa_fwd.  window:
    (left, right) key window, -1 = unbounded (fa_fwd_window when either is set).
    bias: additive score bias (fa_fwd_bias_ws, with the workspace when
    use_workspace), a CUDA tensor of q's dtype that broadcasts to
    [B, Hq, Nq, Nk] (size-1 dims broadcast); a window may come with it.
    Returns (o, lse or None).
    """
    import torch

    lib = load_library()
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("q, k, v must be float16 or bfloat16")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("expected q [B,Hq,Nq,D] and k, v [B,Hkv,Nk,D]")
    B, Hq, Nq, D = q.shape
    Bk, Hkv, Nk, Dk = k.shape
    if (Bk, Dk) != (B, D):
        raise ValueError("batch and head_dim of q and k differ")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if o is None:
        o = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    dtype = FA_BF16 if q.dtype == torch.bfloat16 else FA_FP16
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
            lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, Nk, D,
            ctypes.c_float(scale), 1 if causal else 0, stream or None, dtype)
    wl, wr = (int(x) for x in window)
    if bias is not None:
        bt, sb, sh, sq = _bias_view(bias, q.dtype, B, Hq, Nq, Nk)
        ws = workspace(q.device, stream) if use_workspace else None
        rc = lib.fa_fwd_bias_ws(*args[:13], bt.data_ptr(), sb, sh, sq, wl, wr, args[13], dtype,
                                ws.data_ptr() if ws is not None else None,
                                ws.numel() if ws is not None else 0)
        if rc != FA_OK:
            raise FaError(rc, "fa_fwd_bias_ws")
        return o, lse
    if (wl, wr) != (-1, -1):
        ws = workspace(q.device, stream) if use_workspace else None
        rc = lib.fa_fwd_window(*args[:13], wl, wr, args[13], dtype,
                               ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0)
    elif use_workspace:
        ws = workspace(q.device, stream)
        rc = lib.fa_fwd_ws(*args, ws.data_ptr(), ws.numel())
    else:
        rc = lib.fa_fwd(*args)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd")
    return o, lse


def fa_fwd_unfused(q, k, v, o=None, lse=None, scale: Optional[float] = None,
                   causal: bool = False, stream=None, workspace=None):
    """Standard three-step attention (S and P through device memory), for comparison.

    Same tensors and arguments as fa_fwd; workspace: optional uint8 CUDA tensor
    of at least fa_fwd_unfused_workspace_size bytes (allocated here when None).
    Returns (o, lse).
    """
    import torch

    lib = load_library()
    if q.dtype not in (torch.float16, torch.bfloat16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype, float16 or bfloat16")
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    nbytes = int(lib.fa_fwd_unfused_workspace_size(B, Hq, Nq, Nk))
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    dtype = FA_BF16 if q.dtype == torch.bfloat16 else FA_FP16
    rc = lib.fa_fwd_unfused(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            B, Hq, Hkv, Nq, Nk, D, ctypes.c_float(scale), 1 if causal else 0,
                            stream or None, dtype, workspace.data_ptr(), workspace.numel())
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_unfused")
    return o, lse


def fa_bwd(q, k, v, o, lse, dout, scale: Optional[float] = None, causal: bool = False,
           dq=None, dk=None, dv=None, stream=None, workspace=None,
           window: Tuple[int, int] = (-1, -1), bias=None):
    """Gradients of the attention forward pass (three kernels on the current stream).

    q, o, dout: [B, Hq, Nq, D]; k, v: [B, Hkv, Nk, D] contiguous CUDA tensors of
    one dtype (fp16 or bf16); lse: float32 [B, Hq, Nq] from fa_fwd.  D must be
    64, 128 or 256.  Optional outputs dq (like q), dk, dv (like k); optional
    workspace: a uint8 CUDA tensor of at least fa_bwd_workspace_size bytes
    (allocated here when None).  window: (left, right) key window of the
    forward pass (fa_bwd_window), -1 = unbounded.  bias: the forward pass's
    additive score bias (fa_bwd_bias_window, with or without a window).
    Returns (dq, dk, dv).
    """
    import torch

    lib = load_library()
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("q, k, v must be float16 or bfloat16")
    for name, t in (("k", k), ("v", v), ("o", o), ("dout", dout)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must have the dtype of q")
    if lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if o.shape != q.shape or dout.shape != q.shape or v.shape != k.shape or \
            tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("expected q, o, dout [B,Hq,Nq,D], k, v [B,Hkv,Nk,D], lse [B,Hq,Nq]")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout), ("lse", lse)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = int(lib.fa_bwd_workspace_size(B, Hq, Nq))
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    dtype = FA_BF16 if q.dtype == torch.bfloat16 else FA_FP16
    wl, wr = (int(x) for x in window)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    if bias is not None:
        bt, sb, sh, sq = _bias_view(bias, q.dtype, B, Hq, Nq, Nk)
        rc = lib.fa_bwd_bias_window(*ptrs, B, Hq, Hkv, Nq, Nk, D, ctypes.c_float(scale),
                                    1 if causal else 0, bt.data_ptr(), sb, sh, sq, wl, wr,
                                    stream or None, dtype, workspace.data_ptr(), workspace.numel())
        if rc != FA_OK:
            raise FaError(rc, "fa_bwd_bias_window")
        return dq, dk, dv
    rc = lib.fa_bwd_window(*ptrs, B, Hq, Hkv, Nq, Nk, D, ctypes.c_float(scale), 1 if causal else 0,
                           wl, wr, stream or None, dtype, workspace.data_ptr(), workspace.numel())
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def _bias_view(bias, dtype, B, Hq, Nq, Nk):
    """(tensor, stride_b, stride_h, stride_q) in elements for fa_fwd_bias.

    Broadcast (size-1) dims get stride 0.  Keys must be contiguous and the other
    strides multiples of 8 elements (16 bytes); otherwise the bias is copied
    into a buffer whose rows are padded to a multiple of 8 keys.
    """
    import torch

    if bias.dtype != dtype or not bias.is_cuda:
        raise TypeError("bias must be a CUDA tensor with the dtype of q")
    while bias.dim() < 4:
        bias = bias.unsqueeze(0)
    full = (B, Hq, Nq, Nk)
    if bias.dim() != 4 or any(n not in (1, f) for n, f in zip(bias.shape, full)) or bias.shape[3] != Nk:
        raise ValueError("bias must broadcast to [B, Hq, Nq, Nk] with last dim Nk")
    st = [0 if bias.shape[d] == 1 else bias.stride(d) for d in range(3)]
    if bias.stride(3) != 1 or any(x % 8 for x in st) or bias.data_ptr() % 16:
        nk_pad = (Nk + 7) // 8 * 8
        padded = torch.zeros(tuple(bias.shape[:3]) + (nk_pad,), dtype=dtype, device=bias.device)
        padded[..., :Nk] = bias
        bias = padded[..., :Nk]
        st = [0 if bias.shape[d] == 1 else bias.stride(d) for d in range(3)]
    return bias, st[0], st[1], st[2]
