"""Python binding of ``libfa_sm100.so`` (declared in ``include/fa.h``).

Argument marshalling only: every step of the forward and backward pass runs in the
library's CUDA kernels.  PyTorch provides device memory and the current stream.  There
is no fallback: if the library cannot be loaded, or a call returns an error status,
:class:`FAError` is raised.

Entry points mirror the C ABI names:

* :func:`fa_fwd` / :func:`fa_bwd` - pointer-level calls (device pointers as ints);
* :func:`fa_fwd_window` / :func:`fa_bwd_window` - the same for local attention (key j
  visible to query i iff i - left <= j <= i + right, -1 = unlimited);
* :func:`fwd` / :func:`bwd` - tensor conveniences that allocate outputs with torch
  (``window=(left, right)`` selects local attention);
* :func:`fa_bwd_workspace_bytes`, :func:`fa_device_status`, :func:`fa_status_string`.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa_sm100.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_GQA = 3
FA_ERR_ALIGN = 4
FA_ERR_WORKSPACE = 5
FA_ERR_CUDA = 6
FA_ERR_DEVICE_TIMEOUT = 7
FA_ERR_SCRATCH_LIMIT = 8
FA_NOALLOC_SCRATCH_BYTES = 64 << 20

_lib = None
_lock = threading.Lock()


class FAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: status {code} ({fa_status_string(code)})")


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load the library (building it with nvcc first if it is absent)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            if not build_if_missing:
                raise FAError(FA_ERR_CUDA, f"library missing: {LIB_PATH}")
            from . import build as _build
            _build.build()
        lib = ctypes.CDLL(LIB_PATH)
        vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_fwd.restype = ci
        lib.fa_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
        lib.fa_bwd_workspace_bytes.restype = sz
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                               ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_bwd.restype = ci
        lib.fa_fwd_window.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_fwd_window.restype = ci
        lib.fa_bwd_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                      ci, ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_bwd_window.restype = ci
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                       ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_bwd_noalloc.restype = ci
        lib.fa_device_status.argtypes = [vp]
        lib.fa_device_status.restype = ci
        lib.fa_status_string.argtypes = [ci]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_version.argtypes = []
        lib.fa_version.restype = ci
        lib.fa_watchdog_selftest.argtypes = [ci, vp]
        lib.fa_watchdog_selftest.restype = ci
        lib.fa_kernel_timing.argtypes = [ci]
        lib.fa_kernel_timing.restype = ci
        lib.fa_kernel_time_ms.argtypes = [ci, ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_int)]
        lib.fa_kernel_time_ms.restype = ci
        _lib = lib
        return lib


def fa_status_string(code: int) -> str:
    return load().fa_status_string(int(code)).decode()


def _check(rc: int, where: str) -> None:
    if rc != FA_OK:
        raise FAError(rc, where)


# ----------------------------------------------------------------------------- C ABI

def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, stream) -> None:
    _check(load().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, int(causal), float(scale), stream),
           "fa_fwd")


def fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, d, window_left, window_right, scale,
                  stream) -> None:
    _check(load().fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, d, int(window_left),
                                int(window_right), float(scale), stream), "fa_fwd_window")


def fa_bwd_workspace_bytes(B, Hq, Hkv, N, d) -> int:
    return int(load().fa_bwd_workspace_bytes(B, Hq, Hkv, N, d))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N, d,
           causal, scale, stream) -> None:
    _check(load().fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                         B, Hq, Hkv, N, d, int(causal), float(scale), stream), "fa_bwd")


def fa_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N,
                  d, window_left, window_right, scale, stream) -> None:
    _check(load().fa_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                B, Hq, Hkv, N, d, int(window_left), int(window_right),
                                float(scale), stream), "fa_bwd_window")


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, causal, scale,
                   stream) -> None:
    """fa_bwd for callers that cannot allocate device memory: the scratch is a static
    64 MiB device buffer inside the library (see include/fa.h for the size limit and the
    rule that calls overlapping on the GPU race on that buffer)."""
    _check(load().fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d,
                                 int(causal), float(scale), stream), "fa_bwd_noalloc")


def fa_device_status(stream=None) -> int:
    return int(load().fa_device_status(stream))


def fa_watchdog_selftest(limit_us: int, stream=None) -> None:
    _check(load().fa_watchdog_selftest(int(limit_us), stream), "fa_watchdog_selftest")


def fa_kernel_timing(enable: bool) -> None:
    _check(load().fa_kernel_timing(1 if enable else 0), "fa_kernel_timing")


def fa_kernel_time_ms(which: int):
    """(summed device ms, launches) of the forward (0) or backward main (1) kernel."""
    ms = ctypes.c_float()
    n = ctypes.c_int()
    _check(load().fa_kernel_time_ms(int(which), ctypes.byref(ms), ctypes.byref(n)),
           "fa_kernel_time_ms")
    return float(ms.value), int(n.value)


# ----------------------------------------------------------------------------- tensors

def _stream_handle(t):
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _dims(q, k):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)}")
    return B, Hq, Hkv, N, d


def _need(t, name):
    import torch
    if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def _window(causal, window):
    if window is None:
        return None
    if causal:
        raise ValueError("give either causal=True or window=(left, right), not both")
    left, right = (int(w) for w in window)
    return left, right


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
        window=None):
    """O, LSE = attention(q, k, v); q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16 on one GPU.
    ``window=(left, right)``: local attention, key j visible to query i iff
    i - left <= j <= i + right (-1 = unlimited on that side)."""
    import torch
    win = _window(causal, window)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    B, Hq, Hkv, N, d = _dims(q, k)
    if v.shape != k.shape:
        raise ValueError("v must match k")
    scale = default_scale(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    if win is None:
        fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
               B, Hq, Hkv, N, d, causal, scale, _stream_handle(q))
    else:
        fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                      B, Hq, Hkv, N, d, win[0], win[1], scale, _stream_handle(q))
    return o, l


def bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
        workspace=None, dq=None, dk=None, dv=None, window=None):
    """dQ, dK, dV of <O, dO> given the forward's O and LSE (same causal / window)."""
    import torch
    win = _window(causal, window)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n)
    B, Hq, Hkv, N, d = _dims(q, k)
    scale = default_scale(d) if scale is None else scale
    nbytes = fa_bwd_workspace_bytes(B, Hq, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), B, Hq, Hkv, N, d)
    if win is None:
        fa_bwd(*ptrs, causal, scale, _stream_handle(q))
    else:
        fa_bwd_window(*ptrs, win[0], win[1], scale, _stream_handle(q))
    return dq, dk, dv
