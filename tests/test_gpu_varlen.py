"""GPU parity of packed variable-length attention (forward and backward) against the
fp64 oracle.

Layout: q, o, dq [total_q, Hq, d]; k, v, dk, dv [total_k, Hkv, d]; lse [total_q, Hq];
int32 offsets [B + 1].  Query and key lengths may differ, the causal / window band being
aligned to the end of each sequence.  Tolerances as for the dense tests; rows that see no
key must give O = 0 and LSE = -inf exactly; rows outside every sequence stay untouched.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw, draw_packed, packed_lengths
from test_gpu_parity import (GRAD_TOL, LSE_TOL, SENT_BF16, SENT_F32, _f64, _guarded,
                             _guards_intact, _rel_fro, o_tolerance)

pytestmark = pytest.mark.gpu


def run_varlen(q, k, v, do, cu_q, cu_k, causal, window, scale, backward=True):
    tq, Hq, d = q.shape
    tk, Hkv, _ = k.shape
    mq = int((cu_q[1:] - cu_q[:-1]).max())
    mk = int((cu_k[1:] - cu_k[:-1]).max())
    cq, ck = cu_q.cuda(), cu_k.cuda()
    ob, o = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    lb, lse = _guarded((tq, Hq), torch.float32, SENT_F32)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    fa.fwd_varlen(qd, kd, vd, cq, ck, mq, mk, causal=causal, window=window, scale=scale, out=o,
                  lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    assert _guards_intact(ob, SENT_BF16) and _guards_intact(lb, SENT_F32)
    res = [o.cpu(), lse.cpu()]
    if backward:
        dqb, dq = _guarded(q.shape, torch.bfloat16, SENT_BF16)
        dkb, dk = _guarded(k.shape, torch.bfloat16, SENT_BF16)
        dvb, dv = _guarded(v.shape, torch.bfloat16, SENT_BF16)
        fa.bwd_varlen(qd, kd, vd, o, lse, do.cuda(), cq, ck, mq, mk, causal=causal, window=window,
                      scale=scale, dq=dq, dk=dk, dv=dv)
        torch.cuda.synchronize()
        assert fa.fa_device_status(None) == fa.FA_OK
        for buf, name in ((dqb, "dQ"), (dkb, "dK"), (dvb, "dV")):
            assert _guards_intact(buf, SENT_BF16), f"write outside {name}"
        res += [dq.cpu(), dk.cpu(), dv.cpu()]
    return res


def band(causal, window):
    if window is not None:
        return window
    return (-1, 0) if causal else (-1, -1)


def check_varlen(res, q, k, v, do, cu_q, cu_k, causal, window, scale):
    left, right = band(causal, window)
    o, lse = res[0], res[1]
    o_ref, lse_ref = oracle.attention_fwd_varlen(_f64(q), _f64(k), _f64(v), cu_q.numpy(),
                                                 cu_k.numpy(), left, right, scale)
    lse64 = lse.double().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse64), empty), "rows without keys differ"
    assert np.all(_f64(o)[empty] == 0.0)
    assert np.isfinite(_f64(o)).all()
    assert float(np.max(np.abs(_f64(o) - o_ref) - o_tolerance(o_ref))) <= 0.0
    if (~empty).any():
        assert float(np.abs(lse64[~empty] - lse_ref[~empty]).max()) <= LSE_TOL
    if len(res) == 2:
        return
    refs = oracle.attention_bwd_varlen(_f64(q), _f64(k), _f64(v), _f64(do), cu_q.numpy(),
                                       cu_k.numpy(), left, right, scale)
    for name, x, ref in zip(("dQ", "dK", "dV"), res[2:], refs):
        x = _f64(x)
        assert np.isfinite(x).all(), name
        if np.abs(ref).max() < 1e-12:
            assert np.abs(x).max() <= 1e-2, name
            continue
        err = _rel_fro(x, ref)
        assert err <= GRAD_TOL, f"{name} relative Frobenius error {err}"


SELF_LENS = [1, 127, 128, 129, 300, 0, 513, 64]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", [(False, None), (True, None), (False, (100, 0)),
                                           (False, (64, 64))])
def test_varlen_self_attention(d, causal, window):
    q, k, v, do, cq, ck = draw_packed(SELF_LENS, SELF_LENS, 4, 2, d, seed=200 + d)
    scale = 1.0 / math.sqrt(d)
    res = run_varlen(q, k, v, do, cq, ck, causal, window, scale)
    check_varlen(res, q, k, v, do, cq, ck, causal, window, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal,window", [(False, None), (True, None), (False, (40, 3))])
def test_varlen_unequal_lengths(d, causal, window):
    # Queries shorter and longer than their keys; Lq > Lk leaves the first causal rows
    # without keys (O = 0, LSE = -inf), and one sequence has no keys at all.
    lq = [5, 200, 130, 1, 260, 3, 77]
    lk = [300, 64, 257, 1000, 129, 0, 77]
    q, k, v, do, cq, ck = draw_packed(lq, lk, 6, 3, d, seed=300 + d)
    scale = 1.0 / math.sqrt(d)
    res = run_varlen(q, k, v, do, cq, ck, causal, window, scale)
    check_varlen(res, q, k, v, do, cq, ck, causal, window, scale)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1), (2, 2)])
def test_varlen_heads_and_groups(Hq, Hkv):
    lens = [257, 33, 400]
    q, k, v, do, cq, ck = draw_packed(lens, lens, Hq, Hkv, 128, seed=400 + Hq)
    res = run_varlen(q, k, v, do, cq, ck, True, None, 0.0883883461356163)
    check_varlen(res, q, k, v, do, cq, ck, True, None, 0.0883883461356163)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_one_sequence_equals_the_dense_call(d):
    # A single sequence packed as [N, H, d] runs the same tiles as the dense [1, H, N, d]
    # call: the forward is bitwise identical, dK and dV too (d = 64, 128).
    N, H = 384, 4
    q, k, v, do = draw(1, H, H, N, d, seed=17)
    scale = 1.0 / math.sqrt(d)
    pack = lambda t: t[0].transpose(0, 1).contiguous().cuda()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    cu = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    for causal in (False, True):
        o1, l1 = fa.fwd(qd, kd, vd, causal=causal, scale=scale)
        o2, l2 = fa.fwd_varlen(pack(q), pack(k), pack(v), cu, cu, N, N, causal=causal, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(o1[0].transpose(0, 1), o2)
        assert torch.equal(l1[0].transpose(0, 1), l2)
        g1 = fa.bwd(qd, kd, vd, o1, l1, dod, causal=causal, scale=scale)
        g2 = fa.bwd_varlen(pack(q), pack(k), pack(v), o2, l2, pack(do), cu, cu, N, N,
                           causal=causal, scale=scale)
        torch.cuda.synchronize()
        if d == 256:
            # Dense d = 256 runs its backward as CTA pairs (64-row steps, P^T exchanged as
            # bf16); packed sequences take the single-CTA d-split kernel: equal to rounding.
            for a1, a2 in zip(g1, g2):
                assert _rel_fro(_f64(a1[0].transpose(0, 1)), _f64(a2)) < 1e-2
            continue
        assert torch.equal(g1[1][0].transpose(0, 1), g2[1])
        assert torch.equal(g1[2][0].transpose(0, 1), g2[2])
        assert _rel_fro(_f64(g1[0][0].transpose(0, 1)), _f64(g2[0])) < 1e-3


def test_rows_outside_every_sequence_are_untouched():
    # Offsets that skip rows: rows 0-9 and 500-519 belong to no sequence.
    q, k, v, do, _, _ = draw_packed([520], [520], 2, 2, 128, seed=21)
    cq = torch.tensor([10, 200, 500], dtype=torch.int32, device="cuda")
    o = torch.full(q.shape, SENT_BF16, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((520, 2), SENT_F32, dtype=torch.float32, device="cuda")
    fa.fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq, cq, 300, 300, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    for rows in (slice(0, 10), slice(500, 520)):
        assert torch.all(o[rows] == SENT_BF16) and torch.all(lse[rows] == SENT_F32)
    res = [o.cpu(), lse.cpu()]
    cqn = np.array([0, 190, 490])
    check_varlen([res[0][10:500], res[1][10:500]], q[10:500], k[10:500], v[10:500], None,
                 torch.tensor(cqn, dtype=torch.int32), torch.tensor(cqn, dtype=torch.int32),
                 True, None, 1.0 / math.sqrt(128))


@pytest.mark.parametrize("bad", ["decreasing", "past_total", "too_long"])
def test_inconsistent_offsets_are_reported(bad):
    # The kernels check the offsets before touching any row and report FA_ERR_SEQLENS;
    # nothing faults and the context stays usable.
    q, k, v, _, _, _ = draw_packed([300], [300], 2, 2, 128, seed=23)
    cu, max_len = {"decreasing": ([0, 200, 100], 200), "past_total": ([0, 200, 400], 200),
                   "too_long": ([0, 250, 300], 100)}[bad]   # 250 rows > one 128-row block
    cq = torch.tensor(cu, dtype=torch.int32, device="cuda")
    fa.fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cq, cq, max_len, max_len, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_ERR_SEQLENS
    assert fa.fa_device_status(None) == fa.FA_OK  # read-and-clear
    # The context still works.
    o, _ = fa.fwd_varlen(q.cuda(), k.cuda(), v.cuda(), torch.tensor([0, 300], dtype=torch.int32,
                         device="cuda").contiguous(), torch.tensor([0, 300], dtype=torch.int32,
                         device="cuda"), 300, 300, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK


def test_varlen_full_size_ragged_batch():
    # 24 sequences of long-tailed length (mean 1500, up to 8192), 16 heads, d = 128,
    # causal: two sampled sequences compared with the oracle, invariants everywhere.
    lens = packed_lengths(24, 1500, seed=31)
    H, d = 16, 128
    q, k, v, do, cq, ck = draw_packed(lens, lens, H, H, d, seed=32)
    scale = 1.0 / math.sqrt(d)
    o, lse, dq, dk, dv = run_varlen(q, k, v, do, cq, ck, True, None, scale)
    for b in (int(np.argmax(lens)), 3):
        s0, s1 = int(cq[b]), int(cq[b + 1])
        sub = lambda t: t[s0:s1].contiguous()
        cu1 = torch.tensor([0, s1 - s0], dtype=torch.int32)
        check_varlen([sub(o), sub(lse), sub(dq), sub(dk), sub(dv)], sub(q), sub(k), sub(v),
                     sub(do), cu1, cu1, True, None, scale)
