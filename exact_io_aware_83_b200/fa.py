"""Python binding of ``libfa_sm100.so`` (declared in ``include/fa.h``).

Argument marshalling only: every step of the forward and backward pass runs in the
library's CUDA kernels.  PyTorch provides device memory and the current stream.  There
is no fallback: if the library cannot be loaded, or a call returns an error status,
:class:`FAError` is raised.

Entry points mirror the C ABI names:

* :func:`fa_fwd` / :func:`fa_bwd` - pointer-level calls (device pointers as ints);
* :func:`fa_fwd_window` / :func:`fa_bwd_window` - the same for local attention (key j
  visible to query i iff i - left <= j <= i + right, -1 = unlimited);
* :func:`fa_fwd_varlen` / :func:`fa_bwd_varlen` - packed variable-length sequences
  ([total, H, d] rows, [B+1] offsets; query and key lengths may differ, the band being
  aligned to the end of each sequence);
* :func:`fa_fwd_dropout` / :func:`fa_bwd_dropout` - attention dropout with a
  Philox4x32-10 keep mask regenerated in the backward;
* :func:`fa_fwd_blocksparse` / :func:`fa_bwd_blocksparse` - block-sparse attention over a
  per-head 0/1 mask of 128 x 128 blocks (with or without the causal mask);
* :func:`fa_decode` / :func:`fa_merge` - a few new query rows against a long key/value
  cache, split over the cache, and the merge of partial results;
* :func:`fwd` / :func:`bwd` / :func:`fwd_varlen` / :func:`bwd_varlen` / :func:`decode` /
  :func:`merge` - tensor conveniences that allocate outputs with torch
  (``window=(left, right)`` selects local attention, ``dropout_p`` / ``seed`` dropout,
  ``block_mask`` block-sparse attention);
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
FA_ERR_SEQLENS = 9
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
        lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                                      ci, ci, ci, cf, vp]
        lib.fa_fwd_varlen.restype = ci
        lib.fa_bwd_varlen_workspace_bytes.argtypes = [ci, ci, ci]
        lib.fa_bwd_varlen_workspace_bytes.restype = sz
        lib.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp,
                                      ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_bwd_varlen.restype = ci
        u64 = ctypes.c_ulonglong
        lib.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, u64, cf, vp]
        lib.fa_fwd_dropout.restype = ci
        lib.fa_bwd_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                       ci, ci, ci, ci, ci, ci, cf, u64, cf, vp]
        lib.fa_bwd_dropout.restype = ci
        lib.fa_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_fwd_blocksparse.restype = ci
        lib.fa_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                           ci, ci, ci, ci, ci, ci, cf, vp]
        lib.fa_bwd_blocksparse.restype = ci
        lib.fa_decode_num_splits.argtypes = [ci, ci, ci, ci, ci, ci]
        lib.fa_decode_num_splits.restype = ci
        lib.fa_decode_workspace_bytes.argtypes = [ci, ci, ci, ci, ci, ci, ci]
        lib.fa_decode_workspace_bytes.restype = sz
        lib.fa_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, ci, ci, ci, ci, ci, ci, ci, ci,
                                  cf, vp]
        lib.fa_decode.restype = ci
        lib.fa_merge.argtypes = [vp, vp, vp, vp, ci, ci, ci, vp]
        lib.fa_merge.restype = ci
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
        lib.fa_set_fwd_scheduler.argtypes = [ci]
        lib.fa_set_fwd_scheduler.restype = ci
        lib.fa_get_fwd_scheduler.argtypes = []
        lib.fa_get_fwd_scheduler.restype = ci
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


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, Hq, Hkv, total_q, total_k, max_q, max_k, d,
                  window_left, window_right, scale, stream) -> None:
    _check(load().fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, Hq, Hkv, total_q, total_k, max_q,
                                max_k, d, int(window_left), int(window_right), float(scale),
                                stream), "fa_fwd_varlen")


def fa_bwd_varlen_workspace_bytes(Hq, total_q, d) -> int:
    return int(load().fa_bwd_varlen_workspace_bytes(Hq, total_q, d))


def fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, cu_q, cu_k, B,
                  Hq, Hkv, total_q, total_k, max_q, max_k, d, window_left, window_right, scale,
                  stream) -> None:
    _check(load().fa_bwd_varlen(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                cu_q, cu_k, B, Hq, Hkv, total_q, total_k, max_q, max_k, d,
                                int(window_left), int(window_right), float(scale), stream),
           "fa_bwd_varlen")


def fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, dropout_p, seed, scale,
                   stream) -> None:
    _check(load().fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, N, d, int(causal), float(dropout_p),
                                 int(seed) & 0xFFFFFFFFFFFFFFFF, float(scale), stream),
           "fa_fwd_dropout")


def fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, N,
                   d, causal, dropout_p, seed, scale, stream) -> None:
    _check(load().fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                 B, Hq, Hkv, N, d, int(causal), float(dropout_p),
                                 int(seed) & 0xFFFFFFFFFFFFFFFF, float(scale), stream),
           "fa_bwd_dropout")


def fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, Hq, Hkv, N, d, causal, scale,
                       stream) -> None:
    _check(load().fa_fwd_blocksparse(q, k, v, o, lse, block_mask, B, Hq, Hkv, N, d, int(causal),
                                     float(scale), stream),
           "fa_fwd_blocksparse")


def fa_bwd_blocksparse(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, block_mask,
                       B, Hq, Hkv, N, d, causal, scale, stream) -> None:
    _check(load().fa_bwd_blocksparse(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                                     block_mask, B, Hq, Hkv, N, d, int(causal), float(scale),
                                     stream),
           "fa_bwd_blocksparse")


def fa_decode_num_splits(B, Hq, Hkv, Nq, Nk, d) -> int:
    return int(load().fa_decode_num_splits(B, Hq, Hkv, Nq, Nk, d))


def fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_splits) -> int:
    return int(load().fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_splits))


def fa_decode(q, k, v, o, lse, seqlens_k, workspace, workspace_bytes, B, Hq, Hkv, Nq, Nk, d,
              causal, num_splits, scale, stream) -> None:
    _check(load().fa_decode(q, k, v, o, lse, seqlens_k, workspace, workspace_bytes, B, Hq, Hkv,
                            Nq, Nk, d, int(causal), int(num_splits), float(scale), stream),
           "fa_decode")


def fa_merge(o_parts, lse_parts, o, lse, num_parts, rows, d, stream) -> None:
    _check(load().fa_merge(o_parts, lse_parts, o, lse, int(num_parts), int(rows), int(d),
                           stream), "fa_merge")


def fa_device_status(stream=None) -> int:
    return int(load().fa_device_status(stream))


def fa_watchdog_selftest(limit_us: int, stream=None) -> None:
    _check(load().fa_watchdog_selftest(int(limit_us), stream), "fa_watchdog_selftest")


def fa_kernel_timing(enable: bool) -> None:
    _check(load().fa_kernel_timing(1 if enable else 0), "fa_kernel_timing")


def fa_set_fwd_scheduler(persistent: bool) -> bool:
    """Choose the dense forward's tile scheduler (True: persistent CTAs with dynamic unit
    assignment, False: one CTA per unit); returns the previous choice."""
    prev = load().fa_set_fwd_scheduler(1 if persistent else 0)
    if prev < 0:
        _check(prev, "fa_set_fwd_scheduler")
    return bool(prev)


def fa_get_fwd_scheduler() -> bool:
    """True when the dense forward uses the persistent scheduler."""
    return bool(load().fa_get_fwd_scheduler())


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


def _block_mask(block_mask, B, Hq, N, win, dropout_p):
    import torch
    if block_mask is None:
        return None
    nb = (N + 127) // 128
    if block_mask.dtype == torch.bool:
        block_mask = block_mask.view(torch.uint8)  # one byte, 0 or 1, per block
    if (not block_mask.is_cuda or block_mask.dtype != torch.uint8 or not block_mask.is_contiguous()
            or tuple(block_mask.shape) != (B, Hq, nb, nb)):
        raise ValueError(f"block_mask must be a contiguous uint8 CUDA tensor [{B}, {Hq}, {nb}, {nb}]")
    if win is not None or dropout_p:
        raise ValueError("block_mask combines with causal only (no window, no dropout)")
    return block_mask


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
        window=None, dropout_p: float = 0.0, seed: int = 0, block_mask=None):
    """O, LSE = attention(q, k, v); q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16 on one GPU.
    ``window=(left, right)``: local attention, key j visible to query i iff
    i - left <= j <= i + right (-1 = unlimited on that side).  ``dropout_p`` > 0: attention
    dropout with the Philox4x32-10 mask of ``seed`` (full or causal attention).
    ``block_mask``: block-sparse attention, uint8 (or bool) [B, Hq, ceil(N/128), ceil(N/128)]
    on the GPU, nonzero = the 128 x 128 block is computed (with or without ``causal``)."""
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
    bm = _block_mask(block_mask, B, Hq, N, win, dropout_p)
    if bm is not None:
        fa_fwd_blocksparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                           bm.data_ptr(), B, Hq, Hkv, N, d, causal, scale, _stream_handle(q))
    elif dropout_p:
        if win is not None:
            raise ValueError("dropout is supported with full or causal attention only")
        fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                       B, Hq, Hkv, N, d, causal, dropout_p, seed, scale, _stream_handle(q))
    elif win is None:
        fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
               B, Hq, Hkv, N, d, causal, scale, _stream_handle(q))
    else:
        fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                      B, Hq, Hkv, N, d, win[0], win[1], scale, _stream_handle(q))
    return o, l


def bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
        workspace=None, dq=None, dk=None, dv=None, window=None, dropout_p: float = 0.0,
        seed: int = 0, block_mask=None):
    """dQ, dK, dV of <O, dO> given the forward's O and LSE (same causal / window /
    dropout / block_mask)."""
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
    bm = _block_mask(block_mask, B, Hq, N, win, dropout_p)
    if bm is not None:
        fa_bwd_blocksparse(*ptrs[:11], bm.data_ptr(), *ptrs[11:], causal, scale, _stream_handle(q))
    elif dropout_p:
        if win is not None:
            raise ValueError("dropout is supported with full or causal attention only")
        fa_bwd_dropout(*ptrs, causal, dropout_p, seed, scale, _stream_handle(q))
    elif win is None:
        fa_bwd(*ptrs, causal, scale, _stream_handle(q))
    else:
        fa_bwd_window(*ptrs, win[0], win[1], scale, _stream_handle(q))
    return dq, dk, dv


def decode(q, k, v, seqlens_k=None, causal: bool = False, scale: float | None = None,
           num_splits: int | None = None, out=None, lse=None, workspace=None):
    """Attention of q [B, Hq, Nq, d] against a cache k, v [B, Hkv, Nk, d] (bf16, one GPU),
    of which the first seqlens_k[b] keys are valid (int32 [B] on the GPU, or None: all).
    Causal: the Nq queries are the last Nq positions.  Returns (O, LSE); rows that see
    no key get O = 0 and LSE = -inf."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("expected q [B,Hq,Nq,d] and k, v [B,Hkv,Nk,d]")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)}")
    lens_ptr = None
    if seqlens_k is not None:
        if (not seqlens_k.is_cuda or seqlens_k.dtype != torch.int32 or seqlens_k.numel() != B
                or not seqlens_k.is_contiguous()):
            raise ValueError("seqlens_k must be a contiguous int32 CUDA tensor of B entries")
        lens_ptr = seqlens_k.data_ptr()
    scale = default_scale(d) if scale is None else scale
    if num_splits is None:
        num_splits = fa_decode_num_splits(B, Hq, Hkv, Nq, Nk, d)
        if num_splits < 1:
            raise FAError(FA_ERR_UNSUPPORTED, "fa_decode_num_splits")
    nbytes = fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_splits)
    if workspace is None and nbytes > 0:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    ws_ptr = None if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(), lens_ptr,
              ws_ptr, ws_bytes, B, Hq, Hkv, Nq, Nk, d, causal, num_splits, scale,
              _stream_handle(q))
    return o, l


def merge(o_parts, lse_parts, out=None, lse=None):
    """Combine partial results over disjoint key sets: o_parts [S, ..., d] fp32 (each part
    normalised), lse_parts [S, ...] fp32 -> (O bf16 [..., d], LSE fp32 [...])."""
    import torch
    if (not o_parts.is_cuda or o_parts.dtype != torch.float32 or not o_parts.is_contiguous()
            or not lse_parts.is_cuda or lse_parts.dtype != torch.float32
            or not lse_parts.is_contiguous() or tuple(lse_parts.shape) != tuple(o_parts.shape[:-1])):
        raise ValueError("o_parts [S, ..., d] and lse_parts [S, ...] must be contiguous fp32 CUDA tensors")
    S, d = o_parts.shape[0], o_parts.shape[-1]
    rows = lse_parts[0].numel()
    o = torch.empty(o_parts.shape[1:], dtype=torch.bfloat16, device=o_parts.device) if out is None else out
    l = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device) if lse is None else lse
    fa_merge(o_parts.data_ptr(), lse_parts.data_ptr(), o.data_ptr(), l.data_ptr(), S, rows, d,
             _stream_handle(o_parts))
    return o, l


def _varlen_args(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, window):
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n)
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or q.shape[2] != k.shape[2]:
        raise ValueError("expected q [total_q, Hq, d] and k, v [total_k, Hkv, d]")
    for c, n in ((cu_seqlens_q, "cu_seqlens_q"), (cu_seqlens_k, "cu_seqlens_k")):
        if not c.is_cuda or c.dtype != torch.int32 or not c.is_contiguous() or c.dim() != 1:
            raise ValueError(f"{n} must be a contiguous int32 CUDA vector of B + 1 offsets")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 >= 2 offsets")
    if window is not None and causal:
        raise ValueError("give either causal=True or window=(left, right), not both")
    left, right = (int(w) for w in window) if window is not None else (-1, 0 if causal else -1)
    return (cu_seqlens_q.numel() - 1, q.shape[1], k.shape[1], q.shape[0], k.shape[0],
            int(max_seqlen_q), int(max_seqlen_k), q.shape[2], left, right)


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
               causal: bool = False, scale: float | None = None, window=None, out=None, lse=None):
    """Attention over packed sequences: q [total_q, Hq, d], k/v [total_k, Hkv, d] bf16,
    cu_seqlens_* int32 [B+1] on the GPU.  Returns O [total_q, Hq, d] and LSE [total_q, Hq].
    causal / window bands are aligned to the end of each sequence."""
    import torch
    B, Hq, Hkv, tq, tk, mq, mk, d, left, right = _varlen_args(
        q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, window)
    scale = default_scale(d) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((tq, Hq), dtype=torch.float32, device=q.device) if lse is None else lse
    fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                  cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, Hq, Hkv, tq, tk, mq, mk, d,
                  left, right, scale, _stream_handle(q))
    return o, l


def bwd_varlen(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
               causal: bool = False, scale: float | None = None, window=None, workspace=None,
               dq=None, dk=None, dv=None):
    """dQ, dK, dV of <O, dO> for packed sequences (same arguments as fwd_varlen)."""
    import torch
    B, Hq, Hkv, tq, tk, mq, mk, d, left, right = _varlen_args(
        q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal, window)
    _need(o, "o")
    _need(dout, "dout")
    scale = default_scale(d) if scale is None else scale
    nbytes = fa_bwd_varlen_workspace_bytes(Hq, tq, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                  dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                  workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                  cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, Hq, Hkv, tq, tk, mq, mk, d,
                  left, right, scale, _stream_handle(q))
    return dq, dk, dv
