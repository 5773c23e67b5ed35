"""GPU parity of attention dropout (forward and backward) against the fp64 oracle.

The keep mask is a pure function of (seed, head, row, key) (Philox4x32-10, 16-bit values
against an integer threshold), so the kernel's mask must equal the oracle's bit for bit; that is checked
directly with Q = 0 and V = I (then O = P Z / (1 - p) exposes Z), and through dV with
dO = I.  Outputs and gradients use the dense tolerances.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw
from test_gpu_parity import (GRAD_TOL, LSE_TOL, _f64, _rel_fro, causal_visible, o_tolerance,
                             p_allowance)

pytestmark = pytest.mark.gpu


def run(q, k, v, do, causal, scale, p, seed):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = fa.fwd(qd, kd, vd, causal=causal, scale=scale, dropout_p=p, seed=seed)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, do.cuda(), causal=causal, scale=scale, dropout_p=p,
                        seed=seed)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


def check(res, q, k, v, do, causal, scale, p, seed):
    o, lse, dq, dk, dv = res
    q64, k64, v64 = _f64(q), _f64(k), _f64(v)
    o_r, lse_r = oracle.attention_fwd_dropout(q64, k64, v64, causal, scale, p, seed)
    assert np.isfinite(_f64(o)).all()
    # the allowance's weights: the keep mask times the inverse keep probability
    B, Hq, N, _ = q.shape
    keep = oracle.dropout_keep_mask(B * Hq, N, p, seed).astype(np.float64)
    inv_keep = 65536.0 / (65536.0 - math.floor(p * 65536.0))
    allow = p_allowance(q64, k64, v64, o_r, lse_r, scale, causal_visible(N, causal),
                        weight=lambda b, h, i: keep[b * Hq + h, i] * inv_keep)
    assert float(np.max(np.abs(_f64(o) - o_r) - o_tolerance(o_r, allow))) <= 0.0
    assert float(np.abs(lse.double().numpy() - lse_r).max()) <= LSE_TOL
    refs = oracle.attention_bwd_dropout(_f64(q), _f64(k), _f64(v), _f64(do), causal, scale, p, seed)
    for name, x, ref in zip(("dQ", "dK", "dV"), (dq, dk, dv), refs):
        if np.abs(ref).max() < 1e-12:
            assert np.abs(_f64(x)).max() <= 1e-2, name
            continue
        err = _rel_fro(_f64(x), ref)
        assert err <= GRAD_TOL, f"{name} relative Frobenius error {err}"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 129, 384])
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_against_oracle(d, causal, N, p):
    q, k, v, do = draw(1, 2, 1, N, d, seed=900 + N + d)
    scale = 1.0 / math.sqrt(d)
    seed = 0x1234_5678_9ABC_DEF0 + N
    check(run(q, k, v, do, causal, scale, p, seed), q, k, v, do, causal, scale, p, seed)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1)])
def test_dropout_heads_and_groups(Hq, Hkv):
    q, k, v, do = draw(2, Hq, Hkv, 300, 128, seed=950 + Hq)
    check(run(q, k, v, do, True, 0.088, 0.2, 42), q, k, v, do, True, 0.088, 0.2, 42)


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_mask_is_bitwise_the_oracle_mask(causal):
    # Q = 0 makes P uniform over the visible keys; V = I (N = d = 128) turns O into
    # P Z / (1 - p), so O != 0 is exactly the keep mask.  With dO = I, dV = (P Z / (1 - p))^T.
    N, d, H, p, seed = 128, 128, 3, 0.3, 987654321
    q = torch.zeros(1, H, N, d, dtype=torch.bfloat16)
    k = torch.randn(1, H, N, d).to(torch.bfloat16)
    eye = torch.eye(N, d).to(torch.bfloat16).expand(1, H, N, d).contiguous()
    res = run(q, k, eye, eye, causal, 0.1, p, seed)
    keep = oracle.dropout_keep_mask(H, N, p, seed).astype(bool)
    if causal:
        keep &= np.tril(np.ones((N, N), dtype=bool))[None]
    o, dv = _f64(res[0])[0], _f64(res[4])[0]
    np.testing.assert_array_equal(o != 0, keep)
    np.testing.assert_array_equal(dv.transpose(0, 2, 1) != 0, keep)


def test_dropout_is_deterministic_and_seeded():
    q, k, v, do = draw(1, 4, 4, 256, 128, seed=3)
    a = run(q, k, v, do, False, 0.088, 0.25, 11)
    b = run(q, k, v, do, False, 0.088, 0.25, 11)
    c = run(q, k, v, do, False, 0.088, 0.25, 12)
    assert torch.equal(a[0], b[0]) and torch.equal(a[3], b[3]) and torch.equal(a[4], b[4])
    assert not torch.equal(a[0], c[0])
    # p = 0 is the plain kernels.
    z = run(q, k, v, do, False, 0.088, 0.0, 11)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=0.088)
    torch.cuda.synchronize()
    assert torch.equal(z[0], o.cpu()) and torch.equal(z[1], lse.cpu())
