"""ctypes front end of the fp64 attention oracle (``attention_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, the smoke check and the benchmark's
CPU-baseline leg may import this package; the CUDA library and its binding never do.

Every function takes and returns numpy float64 arrays in the ``[B, H, N, d]`` layout
(LSE / Delta: ``[B, Hq, N]``).  Inputs given in bf16 are upcast exactly by the caller.

Pins (checked by ``tests/test_oracle_pins.py`` against closed forms, the toy example
of the "Consideration"/FlashAttention article page, finite differences and invariants):
``oracle_fwd``, ``oracle_bwd``, their key-window, variable-length, block-sparse and dropout forms,
``oracle_decode``, ``oracle_merge`` and ``online_softmax_stats`` all have pins; none is
"parity unpinned".  The dropout generator itself (Philox4x32-10) is pinned word for word
against an independent implementation (PyTorch's ATen Philox engine, compiled from its
header by the test) and by statistics (keep rate, uniformity, independence).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_VARIANT = "portable"


def use_build(variant: str) -> None:
    """Select the shared object the functions below call: "portable" (-O2, the one the
    tests pin) or "native" (-O3 -march=native for this host, used to time the oracle as
    a CPU baseline; it computes bit-identical results)."""
    global _LIB, _VARIANT
    if variant not in ("portable", "native"):
        raise ValueError(variant)
    if variant != _VARIANT:
        _LIB, _VARIANT = None, variant


def build_flags() -> str:
    """Compiler flags of the build currently selected."""
    return " ".join(_build.NATIVE_FLAGS if _VARIANT == "native" else ["-O2", "-ffp-contract=off", "-fopenmp"])


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build_native() if _VARIANT == "native" else _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ci = ctypes.c_int
        lib.oracle_fwd.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, ci, ctypes.c_double]
        lib.oracle_fwd.restype = ci
        lib.oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                   ci, ci, ci, ci, ci, ci, ctypes.c_double]
        lib.oracle_bwd.restype = ci
        lib.oracle_fwd_window.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, ci, ci,
                                          ctypes.c_double]
        lib.oracle_fwd_window.restype = ci
        lib.oracle_bwd_window.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                          ci, ci, ci, ci, ci, ci, ci, ctypes.c_double]
        lib.oracle_bwd_window.restype = ci
        ip = ctypes.POINTER(ctypes.c_int)
        lib.oracle_decode.argtypes = [dp, dp, dp, ip, dp, dp, ci, ci, ci, ci, ci, ci, ci,
                                      ctypes.c_double]
        lib.oracle_decode.restype = ci
        lib.oracle_merge.argtypes = [dp, dp, ci, ctypes.c_longlong, ci, dp, dp]
        lib.oracle_merge.restype = ci
        lib.oracle_fwd_varlen.argtypes = [dp, dp, dp, ip, ip, dp, dp, ci, ci, ci, ci, ci, ci,
                                          ci, ci, ctypes.c_double]
        lib.oracle_fwd_varlen.restype = ci
        lib.oracle_bwd_varlen.argtypes = [dp, dp, dp, dp, ip, ip, dp, dp, dp, ci, ci, ci, ci,
                                          ci, ci, ci, ci, ctypes.c_double]
        lib.oracle_bwd_varlen.restype = ci
        u8p = ctypes.POINTER(ctypes.c_ubyte)
        u64 = ctypes.c_uint64
        lib.oracle_dropout_mask.argtypes = [u8p, ci, ci, ctypes.c_double, u64]
        lib.oracle_dropout_mask.restype = ci
        lib.oracle_fwd_dropout.argtypes = [dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, ci,
                                           ctypes.c_double, ctypes.c_double, u64]
        lib.oracle_fwd_dropout.restype = ci
        lib.oracle_bwd_dropout.argtypes = [dp, dp, dp, dp, dp, dp, dp, ci, ci, ci, ci, ci, ci,
                                           ctypes.c_double, ctypes.c_double, u64]
        lib.oracle_bwd_dropout.restype = ci
        lib.oracle_fwd_blocksparse.argtypes = [dp, dp, dp, u8p, dp, dp, ci, ci, ci, ci, ci, ci,
                                               ctypes.c_double]
        lib.oracle_fwd_blocksparse.restype = ci
        lib.oracle_bwd_blocksparse.argtypes = [dp, dp, dp, dp, u8p, dp, dp, dp, ci, ci, ci, ci,
                                               ci, ci, ctypes.c_double]
        lib.oracle_bwd_blocksparse.restype = ci
        u32p = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        lib.oracle_philox4x32_10.restype = ci
        lib.oracle_online_softmax_stats.argtypes = [dp, ci, ci, dp, dp]
        lib.oracle_online_softmax_stats.restype = ci
        _LIB = lib
    return _LIB


def _as_f64(a) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def set_threads(n: int) -> None:
    """Set the OpenMP thread count used by later oracle calls in this process."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))
    try:
        gomp = ctypes.CDLL("libgomp.so.1")
        gomp.omp_set_num_threads(ctypes.c_int(int(n)))
    except OSError:
        pass


def _shapes(q, k):
    B, Hq, N, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, Nk, dk) != (B, N, d):
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape}")
    return B, Hq, Hkv, N, d


def attention_fwd(q, k, v, causal: bool, scale: float):
    """O = softmax(scale Q K^T [+ causal mask]) V and the natural-log LSE per row."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, Hkv, N, d = _shapes(q, k)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                           B, Hq, Hkv, N, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd failed with {rc}")
    return o, lse


def attention_bwd(q, k, v, dout, causal: bool, scale: float):
    """Exact gradient of <O, dO>: returns dq, dk, dv, lse, delta."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, Hq, Hkv, N, d = _shapes(q, k)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    delta = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                           _ptr(dv), _ptr(lse), _ptr(delta), B, Hq, Hkv, N, d,
                           int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd failed with {rc}")
    return dq, dk, dv, lse, delta


def attention_fwd_window(q, k, v, left: int, right: int, scale: float):
    """Local attention: key j is visible to query i iff i - left <= j <= i + right
    (a negative bound is unlimited; causal is right = 0)."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, Hkv, N, d = _shapes(q, k)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                  B, Hq, Hkv, N, d, int(left), int(right), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd_window failed with {rc}")
    return o, lse


def attention_bwd_window(q, k, v, dout, left: int, right: int, scale: float):
    """Gradient of <O, dO> for local attention: returns dq, dk, dv, lse, delta."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, Hq, Hkv, N, d = _shapes(q, k)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    delta = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                  _ptr(dv), _ptr(lse), _ptr(delta), B, Hq, Hkv, N, d,
                                  int(left), int(right), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd_window failed with {rc}")
    return dq, dk, dv, lse, delta


def attention_decode(q, k, v, lens, causal: bool, scale: float):
    """Nq queries [B,Hq,Nq,d] against the first lens[b] of Nk cached keys [B,Hkv,Nk,d]
    (lens None: all).  Causal: the queries are the last Nq positions (bottom-right).
    Rows that see no key get O = 0, LSE = -inf."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
    lens_arr = None
    if lens is not None:
        lens_arr = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(B))
    o = np.empty_like(q)
    lse = np.empty((B, Hq, Nq), dtype=np.float64)
    lp = None if lens_arr is None else lens_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    rc = _lib().oracle_decode(_ptr(q), _ptr(k), _ptr(v), lp, _ptr(o), _ptr(lse), B, Hq, Hkv,
                              Nq, Nk, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_decode failed with {rc}")
    return o, lse


def _cu(cu):
    a = np.ascontiguousarray(np.asarray(cu, dtype=np.int32).reshape(-1))
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def attention_fwd_varlen(q, k, v, cu_q, cu_k, left: int, right: int, scale: float):
    """Packed sequences: q [total_q, Hq, d], k/v [total_k, Hkv, d], cu_* [B+1] row offsets.
    The band i + dlt - left <= j <= i + dlt + right (dlt = Lk - Lq, -1 = unlimited) is
    aligned to the end of each sequence.  Returns o [total_q, Hq, d], lse [total_q, Hq]."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    tq, Hq, d = q.shape
    tk, Hkv, dk = k.shape
    if dk != d or v.shape != k.shape:
        raise ValueError("shape mismatch")
    cq, cqp = _cu(cu_q)
    ck, ckp = _cu(cu_k)
    if cq.size != ck.size:
        raise ValueError("cu_q and cu_k must have B+1 entries each")
    o = np.empty_like(q)
    lse = np.empty((tq, Hq), dtype=np.float64)
    rc = _lib().oracle_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), cqp, ckp, _ptr(o), _ptr(lse),
                                  cq.size - 1, Hq, Hkv, tq, tk, d, int(left), int(right),
                                  float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd_varlen failed with {rc}")
    return o, lse


def attention_bwd_varlen(q, k, v, dout, cu_q, cu_k, left: int, right: int, scale: float):
    """Gradient of <O, dO> for packed sequences; returns dq, dk, dv."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    tq, Hq, d = q.shape
    tk, Hkv, _ = k.shape
    cq, cqp = _cu(cu_q)
    ck, ckp = _cu(cu_k)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    rc = _lib().oracle_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), cqp, ckp, _ptr(dq),
                                  _ptr(dk), _ptr(dv), cq.size - 1, Hq, Hkv, tq, tk, d,
                                  int(left), int(right), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd_varlen failed with {rc}")
    return dq, dk, dv


def philox4x32_10(ctr, key):
    """The oracle's Philox4x32-10: four uint32 output words for counter ``ctr`` (4 words)
    and key ``key`` (2 words)."""
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32).reshape(4))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32).reshape(2))
    out = np.empty(4, dtype=np.uint32)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    rc = _lib().oracle_philox4x32_10(c.ctypes.data_as(u32p), k.ctypes.data_as(u32p),
                                     out.ctypes.data_as(u32p))
    if rc != 0:
        raise RuntimeError(f"oracle_philox4x32_10 failed with {rc}")
    return out


def dropout_keep_mask(BH: int, N: int, p: float, seed: int):
    """uint8 [BH, N, N]: 1 where the probability of (query head bh, row i, key j) is kept."""
    keep = np.empty((BH, N, N), dtype=np.uint8)
    rc = _lib().oracle_dropout_mask(keep.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte)), BH, N,
                                    float(p), int(seed) & 0xFFFFFFFFFFFFFFFF)
    if rc != 0:
        raise RuntimeError(f"oracle_dropout_mask failed with {rc}")
    return keep


def attention_fwd_dropout(q, k, v, causal: bool, scale: float, p: float, seed: int):
    """O = (P * Z / (1 - p)) V with the Philox4x32-10 keep mask Z; LSE without dropout."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, Hkv, N, d = _shapes(q, k)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N,
                                   d, int(bool(causal)), float(scale), float(p),
                                   int(seed) & 0xFFFFFFFFFFFFFFFF)
    if rc != 0:
        raise RuntimeError(f"oracle_fwd_dropout failed with {rc}")
    return o, lse


def attention_bwd_dropout(q, k, v, dout, causal: bool, scale: float, p: float, seed: int):
    """dq, dk, dv of <O, dO> for attention_fwd_dropout with the same seed."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, Hq, Hkv, N, d = _shapes(q, k)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _lib().oracle_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, Hq, Hkv, N, d, int(bool(causal)), float(scale),
                                   float(p), int(seed) & 0xFFFFFFFFFFFFFFFF)
    if rc != 0:
        raise RuntimeError(f"oracle_bwd_dropout failed with {rc}")
    return dq, dk, dv


def _bmask(bmask, B, Hq, N):
    nb = (N + 127) // 128
    m = np.ascontiguousarray(np.asarray(bmask, dtype=np.uint8))
    if m.shape != (B, Hq, nb, nb):
        raise ValueError(f"block mask must be [B, Hq, {nb}, {nb}]")
    return m, m.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte))


def attention_fwd_blocksparse(q, k, v, bmask, causal: bool, scale: float):
    """Attention restricted to the enabled 128 x 128 blocks of bmask [B, Hq, nb, nb]
    (and to j <= i with causal).  Rows without keys: O = 0, LSE = -inf."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, Hkv, N, d = _shapes(q, k)
    m, mp = _bmask(bmask, B, Hq, N)
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    rc = _lib().oracle_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), mp, _ptr(o), _ptr(lse), B, Hq,
                                       Hkv, N, d, int(bool(causal)), float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_fwd_blocksparse failed with {rc}")
    return o, lse


def attention_bwd_blocksparse(q, k, v, dout, bmask, causal: bool, scale: float):
    """dq, dk, dv of <O, dO> for block-sparse attention."""
    q, k, v, dout = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, Hq, Hkv, N, d = _shapes(q, k)
    m, mp = _bmask(bmask, B, Hq, N)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    rc = _lib().oracle_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), mp, _ptr(dq),
                                       _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, int(bool(causal)),
                                       float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle_bwd_blocksparse failed with {rc}")
    return dq, dk, dv


def merge(o_parts, lse_parts):
    """Combine S partial results over disjoint key sets: o_parts [S, ..., d] (each part
    normalised), lse_parts [S, ...] -> (o [..., d], lse [...])."""
    op = _as_f64(o_parts)
    lp = _as_f64(lse_parts)
    S = op.shape[0]
    d = op.shape[-1]
    if lp.shape != op.shape[:-1]:
        raise ValueError("lse_parts must be o_parts without its last axis")
    rows = int(np.prod(op.shape[1:-1])) if op.ndim > 2 else 1
    o = np.empty(op.shape[1:], dtype=np.float64)
    lse = np.empty(lp.shape[1:], dtype=np.float64)
    rc = _lib().oracle_merge(_ptr(op), _ptr(lp), S, rows, d, _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"oracle_merge failed with {rc}")
    return o, lse


def online_softmax_stats(scores, block: int):
    """(m, l) of the blocked online-softmax recurrence over a 1-D score row."""
    s = _as_f64(scores).reshape(-1)
    m = ctypes.c_double()
    l = ctypes.c_double()
    rc = _lib().oracle_online_softmax_stats(_ptr(s), s.size, int(block), ctypes.byref(m),
                                            ctypes.byref(l))
    if rc != 0:
        raise RuntimeError(f"oracle_online_softmax_stats failed with {rc}")
    return m.value, l.value
