"""Host-only checks of the C ABI: the library builds for sm_100a, loads without a GPU,
exports every entry point that include/fa.h declares, and rejects invalid arguments with
the documented status codes before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from exact_io_aware_83_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

FAKE = 0x10000  # never dereferenced: every case below fails validation first


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_fwd_window", "fa_bwd_window", "fa_decode",
                     "fa_fwd_varlen", "fa_bwd_varlen", "fa_fwd_dropout", "fa_bwd_dropout",
                     "fa_decode_num_splits", "fa_decode_workspace_bytes", "fa_merge",
                     "fa_bwd_workspace_bytes", "fa_device_status", "fa_status_string",
                     "fa_version", "fa_fwd_blocksparse", "fa_bwd_blocksparse"):
        assert required in names


def test_library_exports_every_declared_symbol():
    fa.load()
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing


def test_status_strings_and_version():
    assert fa.load().fa_version() == 102
    for code in range(8):
        assert fa.fa_status_string(code) not in ("", "unknown status")
    assert fa.fa_status_string(99) == "unknown status"


def _fwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, N=16, d=128,
                causal=0, scale=0.125, stream=None)
    args.update(kw)
    return fa.load().fa_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"],
                            args["Hq"], args["Hkv"], args["N"], args["d"], args["causal"],
                            args["scale"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(lse=None), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_GQA),
    (dict(o=FAKE + 8), fa.FA_ERR_ALIGN),
    (dict(lse=FAKE + 4), fa.FA_ERR_ALIGN),
    (dict(B=1 << 16, Hq=1 << 8, Hkv=1, N=1 << 8), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_argument_errors(kw, code):
    assert _fwd(**kw) == code


def _bwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
                ws=FAKE, ws_bytes=1 << 30, B=1, Hq=2, Hkv=1, N=16, d=128, causal=1, scale=0.125,
                stream=None)
    args.update(kw)
    a = args
    return fa.load().fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"],
                            a["dk"], a["dv"], a["ws"], a["ws_bytes"], a["B"], a["Hq"], a["Hkv"],
                            a["N"], a["d"], a["causal"], a["scale"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(dout=None), fa.FA_ERR_INVALID_ARG),
    (dict(dv=None), fa.FA_ERR_INVALID_ARG),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(Hq=4, Hkv=3), fa.FA_ERR_GQA),
    (dict(ws=None), fa.FA_ERR_WORKSPACE),
    (dict(ws_bytes=100), fa.FA_ERR_WORKSPACE),
    (dict(dk=FAKE + 2), fa.FA_ERR_ALIGN),
])
def test_bwd_argument_errors(kw, code):
    assert _bwd(**kw) == code


def _fwd_w(left, right, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, N=16, d=128,
             scale=0.125)
    a.update(kw)
    return fa.load().fa_fwd_window(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                                   a["Hkv"], a["N"], a["d"], left, right, a["scale"], None)


def _bwd_w(left, right, **kw):
    a = dict(B=1, Hq=2, Hkv=1, N=16, d=128, ws_bytes=1 << 30)
    a.update(kw)
    return fa.load().fa_bwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                   a["ws_bytes"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], left,
                                   right, 0.125, None)


@pytest.mark.parametrize("left,right,kw,code", [
    (-2, 0, {}, fa.FA_ERR_INVALID_ARG),
    (0, -2, {}, fa.FA_ERR_INVALID_ARG),
    (-(1 << 31), -1, {}, fa.FA_ERR_INVALID_ARG),
    (4, 4, dict(q=None), fa.FA_ERR_INVALID_ARG),
    (4, 4, dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (4, 4, dict(Hq=3, Hkv=2), fa.FA_ERR_GQA),
    (4, 4, dict(o=FAKE + 8), fa.FA_ERR_ALIGN),
    (4, 4, dict(B=1, Hq=1, Hkv=1, N=(1 << 30) + 1), fa.FA_ERR_UNSUPPORTED),
])
def test_fwd_window_argument_errors(left, right, kw, code):
    assert _fwd_w(left, right, **kw) == code


@pytest.mark.parametrize("left,right,kw,code", [
    (-5, 3, {}, fa.FA_ERR_INVALID_ARG),
    (3, -3, {}, fa.FA_ERR_INVALID_ARG),
    (3, 3, dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (3, 3, dict(ws_bytes=100), fa.FA_ERR_WORKSPACE),
])
def test_bwd_window_argument_errors(left, right, kw, code):
    assert _bwd_w(left, right, **kw) == code


def test_binding_rejects_causal_together_with_a_window():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fwd(q, q, q, causal=True, window=(4, 0))


def _dec(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, lens=None, ws=FAKE, ws_bytes=1 << 30,
             B=2, Hq=8, Hkv=2, Nq=1, Nk=1000, d=128, causal=0, splits=4, scale=0.125)
    a.update(kw)
    return fa.load().fa_decode(a["q"], a["k"], a["v"], a["o"], a["lse"], a["lens"], a["ws"],
                               a["ws_bytes"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"],
                               a["d"], a["causal"], a["splits"], a["scale"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=0), fa.FA_ERR_INVALID_ARG),
    (dict(causal=3), fa.FA_ERR_INVALID_ARG),
    (dict(splits=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=1025), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(Hq=8, Hkv=3), fa.FA_ERR_GQA),
    (dict(Hq=8, Hkv=1, Nq=17), fa.FA_ERR_UNSUPPORTED),          # 136 query rows per K/V head
    (dict(Hq=8, Hkv=1, Nq=9, d=256), fa.FA_ERR_UNSUPPORTED),    # 72 > 64 for d = 256
    (dict(ws=None), fa.FA_ERR_WORKSPACE),
    (dict(ws_bytes=64), fa.FA_ERR_WORKSPACE),
    (dict(o=FAKE + 8), fa.FA_ERR_ALIGN),
    (dict(lens=FAKE + 2), fa.FA_ERR_ALIGN),
])
def test_decode_argument_errors(kw, code):
    assert _dec(**kw) == code


def test_decode_workspace_and_splits():
    B, Hq, Hkv, Nq, Nk, d = 2, 8, 2, 3, 1000, 128
    rows = B * Hq * Nq
    pad = lambda x: (x + 255) // 256 * 256
    assert fa.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, 1) == 0
    assert fa.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, 5) == pad(5 * rows * d * 4) + pad(5 * rows * 4)
    assert fa.fa_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, 0) == 0
    assert fa.fa_decode_workspace_bytes(B, Hq, 3, Nq, Nk, d, 2) == 0
    # Without a device the split choice assumes 148 SMs (one CTA each): 4 units -> 37
    # splits, capped by the 8 key blocks (at least two per split) -> 4.
    assert fa.fa_decode_num_splits(B, Hq, Hkv, Nq, Nk, d) == 4
    assert fa.fa_decode_num_splits(B, Hq, Hkv, Nq, 1 << 20, d) == 37
    assert fa.fa_decode_num_splits(64, Hq, Hkv, Nq, 1 << 20, d) == 1
    # d = 64 with up to 16 query rows per K/V head runs two CTAs per SM (296 slots).
    assert fa.fa_decode_num_splits(B, Hq, Hkv, Nq, 1 << 20, 64) == 74
    assert fa.fa_decode_num_splits(B, 16, 2, 5, 1 << 20, 64) == 37
    assert fa.fa_decode_num_splits(B, Hq, 3, Nq, Nk, d) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(o=None), fa.FA_ERR_INVALID_ARG),
    (dict(parts=0), fa.FA_ERR_INVALID_ARG),
    (dict(rows=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(lse=FAKE + 4), fa.FA_ERR_ALIGN),
])
def test_merge_argument_errors(kw, code):
    a = dict(op=FAKE, lp=FAKE, o=FAKE, lse=FAKE, parts=3, rows=10, d=128)
    a.update(kw)
    assert fa.load().fa_merge(a["op"], a["lp"], a["o"], a["lse"], a["parts"], a["rows"], a["d"],
                              None) == code


@pytest.mark.parametrize("p_drop,causal,code", [
    (-0.1, 0, fa.FA_ERR_INVALID_ARG), (1.0, 0, fa.FA_ERR_INVALID_ARG),
    (float("nan"), 0, fa.FA_ERR_INVALID_ARG), (0.1, 2, fa.FA_ERR_INVALID_ARG),
])
def test_dropout_argument_errors(p_drop, causal, code):
    lib = fa.load()
    assert lib.fa_fwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1, 16, 128, causal, p_drop, 7,
                              0.125, None) == code
    assert lib.fa_bwd_dropout(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                              1, 2, 1, 16, 128, causal, p_drop, 7, 0.125, None) == code


def _sparse(mask, Hq, Hkv, N, d, causal):
    lib = fa.load()
    rf = lib.fa_fwd_blocksparse(FAKE, FAKE, FAKE, FAKE, FAKE, mask, 1, Hq, Hkv, N, d, causal, 0.125,
                                None)
    rb = lib.fa_bwd_blocksparse(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                                mask, 1, Hq, Hkv, N, d, causal, 0.125, None)
    return rf, rb


@pytest.mark.parametrize("mask,Hq,Hkv,N,d,causal,code", [
    (None, 2, 1, 16, 128, 0, fa.FA_ERR_INVALID_ARG),              # no mask
    (FAKE, 2, 1, 16, 128, 2, fa.FA_ERR_INVALID_ARG),              # causal not 0/1
    (FAKE, 2, 1, 4096 * 128 + 1, 64, 0, fa.FA_ERR_UNSUPPORTED),   # more than 4096 blocks a side
    (FAKE, 64, 1, 32768, 256, 1, fa.FA_ERR_UNSUPPORTED),          # d = 256 bitmap: 64 x 8 words
    (FAKE, 2, 3, 16, 128, 0, fa.FA_ERR_GQA),
])
def test_blocksparse_argument_errors(mask, Hq, Hkv, N, d, causal, code):
    assert _sparse(mask, Hq, Hkv, N, d, causal) == (code, code)


@pytest.mark.skipif(torch.cuda.is_available(), reason="valid-argument path needs no GPU")
def test_blocksparse_limits_that_fit_reach_the_device_check():
    # 64 query heads per K/V head over 256 blocks: 2 KB of bitmap fits for d = 128, and a
    # 4096-block side is the longest sequence taken.
    assert _sparse(FAKE, 64, 1, 32768, 128, 1) == (fa.FA_ERR_CUDA, fa.FA_ERR_CUDA)
    assert _sparse(FAKE, 2, 1, 4096 * 128, 64, 0) == (fa.FA_ERR_CUDA, fa.FA_ERR_CUDA)


def test_workspace_size():
    B, Hq, N, d = 2, 4, 100, 128
    rows = B * Hq * N
    pad = lambda x: (x + 255) // 256 * 256
    assert fa.fa_bwd_workspace_bytes(B, Hq, 2, N, d) == pad(rows * 4) + pad(rows * d * 4)
    assert fa.fa_bwd_workspace_bytes(B, Hq, 3, N, d) == 0
    assert fa.fa_bwd_workspace_bytes(B, Hq, 2, N, 48) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="valid-argument path needs no GPU")
def test_valid_arguments_without_a_device_report_cuda_error():
    # Every argument is valid, so the call reaches the device check and stops there.
    assert _fwd() == fa.FA_ERR_CUDA
    assert _bwd() == fa.FA_ERR_CUDA
    assert _fwd_w(3, 0) == fa.FA_ERR_CUDA
    assert _bwd_w(-1, 7) == fa.FA_ERR_CUDA
    assert _dec() == fa.FA_ERR_CUDA
    assert fa.load().fa_merge(FAKE, FAKE, FAKE, FAKE, 2, 4, 64, None) == fa.FA_ERR_CUDA


def test_binding_checks_the_block_mask():
    m = torch.zeros(1, 2, 3, 3, dtype=torch.uint8)
    with pytest.raises(ValueError):      # not on the GPU
        fa._block_mask(m, 1, 2, 300, None, 0.0)
    with pytest.raises(ValueError):      # wrong dtype
        fa._block_mask(m.float(), 1, 2, 300, None, 0.0)
    with pytest.raises(ValueError):      # wrong shape (nb = 3 for N = 300)
        fa._block_mask(torch.zeros(1, 2, 2, 2, dtype=torch.uint8), 1, 2, 300, None, 0.0)
    assert fa._block_mask(None, 1, 2, 300, None, 0.0) is None


def test_binding_rejects_cpu_tensors():
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fwd(q, q, q)
