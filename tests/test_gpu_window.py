"""GPU parity of local (sliding-window) attention against the fp64 oracle.

Key j is visible to query i iff i - left <= j <= i + right (-1 = unlimited on that side);
the "FlashAttention1" Q&A's scaling question (item 4) proposes pairing the method with
local attention.  Same tolerances as the dense tests (the O bound with the allowance for
the bf16 probabilities computed over each row's window), |LSE - LSE_ref| <= 1e-3,
relative Frobenius error <= 2e-2 for dQ, dK, dV, guard bands intact, no NaN/Inf.  Exact checks: the windows that equal full and causal
attention reproduce fa_fwd / fa_bwd bit for bit, and a zero-width window returns V itself.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw
from test_gpu_parity import (GRAD_TOL, LSE_TOL, SENT_BF16, SENT_F32, _f64, _finite, _guarded,
                             _guards_intact, _rel_fro, o_tolerance, p_allowance)

pytestmark = pytest.mark.gpu


def run_fwd_w(q, k, v, window, scale):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    B, Hq, N, d = q.shape
    ob, o = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    lb, lse = _guarded((B, Hq, N), torch.float32, SENT_F32)
    fa.fwd(qd, kd, vd, window=window, scale=scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    assert _guards_intact(ob, SENT_BF16), "write outside O"
    assert _guards_intact(lb, SENT_F32), "write outside LSE"
    return o.cpu(), lse.cpu()


def run_bwd_w(q, k, v, o, lse, do, window, scale):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dqb, dq = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    dkb, dk = _guarded(k.shape, torch.bfloat16, SENT_BF16)
    dvb, dv = _guarded(v.shape, torch.bfloat16, SENT_BF16)
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    fa.bwd(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), window=window,
           scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    for buf, name in ((dqb, "dQ"), (dkb, "dK"), (dvb, "dV")):
        assert _guards_intact(buf, SENT_BF16), f"write outside {name}"
    return dq.cpu(), dk.cpu(), dv.cpu()


def check_fwd_w(o, lse, q, k, v, window, scale):
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    o_ref, lse_ref = oracle.attention_fwd_window(q64, k64, v64, window[0], window[1], scale)
    _finite(o, lse)
    diff = np.abs(_f64(o) - o_ref)
    keys = np.arange(q.shape[2])
    left, right = window

    def visible(b, h, i):
        return (((keys >= i - left) if left >= 0 else True) & ((keys <= i + right) if right >= 0 else True)
                & np.ones(len(keys), dtype=bool))

    excess = float(np.max(diff - o_tolerance(o_ref, p_allowance(q64, k64, v64, o_ref, lse_ref, scale, visible))))
    err_l = float(np.max(np.abs(lse.double().numpy() - lse_ref)))
    assert excess <= 0.0, f"|O-O_ref| above tolerance by {excess}"
    assert err_l <= LSE_TOL, f"max|LSE-LSE_ref| = {err_l}"


def check_bwd_w(dq, dk, dv, q, k, v, do, window, scale):
    dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd_window(_f64(q), _f64(k), _f64(v), _f64(do),
                                                         window[0], window[1], scale)
    _finite(dq, dk, dv)
    for name, x, ref in (("dQ", dq, dq_r), ("dK", dk, dk_r), ("dV", dv, dv_r)):
        x = _f64(x)
        if np.abs(ref).max() < 1e-12:
            # zero-width windows: every probability is 1, so dS = 0 and dQ = dK = 0
            assert np.abs(x).max() <= 1e-2, f"{name} should vanish"
            continue
        err = _rel_fro(x, ref)
        assert err <= GRAD_TOL, f"{name} relative Frobenius error {err}"


# Windows chosen around the 128-key (64 for d = 256) block edges: inside one block, exactly
# one block, straddling two, one side only, and both sides.
WINDOWS = [(0, 0), (1, 0), (127, 0), (128, 0), (200, 0), (64, 64), (300, 17), (0, 200),
           (5, -1), (-1, 5), (129, 129)]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [257, 700])
@pytest.mark.parametrize("window", WINDOWS)
def test_window_fwd_bwd(d, N, window):
    q, k, v, do = draw(1, 2, 1, N, d, seed=4000 + N + d + 7 * window[0] + window[1])
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd_w(q, k, v, window, scale)
    check_fwd_w(o, lse, q, k, v, window, scale)
    dq, dk, dv = run_bwd_w(q, k, v, o, lse, do, window, scale)
    check_bwd_w(dq, dk, dv, q, k, v, do, window, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [1, 2, 130])
def test_zero_width_window_returns_v(d, N):
    # Each row sees only its own key: P = [1], so O_i = v_i exactly and LSE_i = scale q_i.k_i.
    q, k, v, do = draw(1, 2, 2, N, d, seed=5000 + N + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd_w(q, k, v, (0, 0), scale)
    assert torch.equal(o, v)
    lse_ref = (_f64(q) * _f64(k)).sum(-1) * scale
    assert np.abs(lse.double().numpy() - lse_ref).max() <= LSE_TOL
    dq, dk, dv = run_bwd_w(q, k, v, o, lse, do, (0, 0), scale)
    check_bwd_w(dq, dk, dv, q, k, v, do, (0, 0), scale)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_unlimited_windows_equal_dense_calls_bitwise(d):
    N = 300
    q, k, v, do = draw(1, 4, 2, N, d, seed=6000 + d)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    for causal, window in ((False, (-1, -1)), (True, (-1, 0)), (True, (N - 1, 0)),
                           (False, (N + 5, 10 ** 9))):
        o1, l1 = fa.fwd(qd, kd, vd, causal=causal, scale=scale)
        o2, l2 = fa.fwd(qd, kd, vd, window=window, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2), window
        g1 = fa.bwd(qd, kd, vd, o1, l1, dod, causal=causal, scale=scale)
        g2 = fa.bwd(qd, kd, vd, o1, l1, dod, window=window, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2]), window
        assert _rel_fro(_f64(g1[0]), _f64(g2[0])) < 1e-3


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1), (4, 4)])
@pytest.mark.parametrize("window", [(100, 0), (50, 50), (300, 0)])
def test_window_heads_and_groups(Hq, Hkv, window):
    # (8, 2): a CTA owns the same query block of two heads; (3, 1) and (4, 4): two query
    # blocks of one head, whose key-block ranges differ under a window.
    q, k, v, do = draw(2, Hq, Hkv, 520, 128, seed=7000 + Hq * 10 + Hkv + window[0])
    scale = 0.0883883461356163
    o, lse = run_fwd_w(q, k, v, window, scale)
    check_fwd_w(o, lse, q, k, v, window, scale)
    dq, dk, dv = run_bwd_w(q, k, v, o, lse, do, window, scale)
    check_bwd_w(dq, dk, dv, q, k, v, do, window, scale)


@pytest.mark.parametrize("d", [128, 256])
def test_window_stress_large_scores(d):
    # Large scores move the running max between blocks; with a left bound, a row's first
    # visible key can sit in the tile's second or third block, after blocks it cannot see.
    q, k, v, do = draw(1, 2, 2, 640, d, seed=78, q_std=4.0)
    scale = 0.35 if d == 128 else 0.25
    for window in ((300, 0), (200, 100), (129, 3)):
        o, lse = run_fwd_w(q, k, v, window, scale)
        check_fwd_w(o, lse, q, k, v, window, scale)
        dq, dk, dv = run_bwd_w(q, k, v, o, lse, do, window, scale)
        check_bwd_w(dq, dk, dv, q, k, v, do, window, scale)


def test_window_full_size_8k():
    # Sliding-window causal attention over 8k tokens (1024 keys per row, including the
    # row's own), 16 heads: one (b, head) slice compared row by row with the oracle, and
    # the gradient invariants sum_j dK_j = 0, sum_j dV_j = sum_i dO_i checked everywhere.
    B, H, N, d, window = 1, 16, 8192, 128, (1023, 0)
    q, k, v, do = draw(B, H, H, N, d, seed=8080)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.fwd(qd, kd, vd, window=window, scale=scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, window=window, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    o, lse, dq, dk, dv = (t.cpu() for t in (o, lse, dq, dk, dv))
    _finite(o, lse, dq, dk, dv)
    h = H - 1
    sl = slice(h, h + 1)
    check_fwd_w(o[:, sl], lse[:, sl], q[:, sl], k[:, sl], v[:, sl], window, scale)
    check_bwd_w(dq[:, sl], dk[:, sl], dv[:, sl], q[:, sl], k[:, sl], v[:, sl], do[:, sl], window,
                scale)
    dk64, dv64, do64 = _f64(dk), _f64(dv), _f64(do)
    assert np.abs(dk64.sum(axis=2)).max() <= 2e-2 * np.abs(dk64).sum(axis=2).max()
    do_sum = do64.sum(axis=2)
    assert np.abs(dv64.sum(axis=2) - do_sum).max() <= 2e-2 * np.abs(do_sum).max() + 1.0
