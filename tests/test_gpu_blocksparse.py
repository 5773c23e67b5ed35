"""GPU parity of block-sparse attention against the fp64 oracle.

Key j is visible to query i iff block (i // 128, j // 128) of the query head's 0/1 mask is
enabled (and j <= i with causal); the deep-dive page's closing paragraph names block-sparse
FlashAttention.  Tolerances as for the dense tests: |O - O_ref| <= max(1e-2, one bf16
spacing of O_ref), |LSE - LSE_ref| <= 1e-3, relative Frobenius error <= 2e-2 for dQ, dK,
dV, guard bands intact, no NaN/Inf.  Exact checks: an all-ones mask reproduces fa_fwd and
fa_bwd's dK, dV bit for bit (same blocks in the same order), an all-zeros mask gives O = 0,
LSE = -inf and zero gradients, and rows or keys whose blocks are all disabled give zeros.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw, draw_block_mask
from test_gpu_parity import (GRAD_TOL, LSE_TOL, SENT_BF16, SENT_F32, _f64, _guarded, _guards_intact,
                             _rel_fro, o_tolerance)

pytestmark = pytest.mark.gpu


def run_fwd_bs(q, k, v, mask, causal, scale):
    B, Hq, N, d = q.shape
    ob, o = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    lb, lse = _guarded((B, Hq, N), torch.float32, SENT_F32)
    fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, out=o, lse=lse,
           block_mask=mask.cuda())
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    assert _guards_intact(ob, SENT_BF16), "write outside O"
    assert _guards_intact(lb, SENT_F32), "write outside LSE"
    return o.cpu(), lse.cpu()


def run_bwd_bs(q, k, v, o, lse, do, mask, causal, scale):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dqb, dq = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    dkb, dk = _guarded(k.shape, torch.bfloat16, SENT_BF16)
    dvb, dv = _guarded(v.shape, torch.bfloat16, SENT_BF16)
    ws = torch.full((fa.fa_bwd_workspace_bytes(B, Hq, Hkv, N, d),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    fa.bwd(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), causal=causal,
           scale=scale, workspace=ws, dq=dq, dk=dk, dv=dv, block_mask=mask.cuda())
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    for buf, name in ((dqb, "dQ"), (dkb, "dK"), (dvb, "dV")):
        assert _guards_intact(buf, SENT_BF16), f"write outside {name}"
    return dq.cpu(), dk.cpu(), dv.cpu()


def check_fwd_bs(o, lse, q, k, v, mask, causal, scale):
    o_ref, lse_ref = oracle.attention_fwd_blocksparse(_f64(q), _f64(k), _f64(v), mask.numpy(),
                                                      causal, scale)
    lse64 = lse.double().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse64), empty), "rows without keys differ"
    assert np.all(_f64(o)[empty] == 0.0), "rows without keys must give O = 0"
    assert np.isfinite(_f64(o)).all() and np.isfinite(lse64[~empty]).all()
    excess = float(np.max(np.abs(_f64(o) - o_ref) - o_tolerance(o_ref)))
    assert excess <= 0.0, f"|O-O_ref| above tolerance by {excess}"
    if (~empty).any():
        err = float(np.max(np.abs(lse64[~empty] - lse_ref[~empty])))
        assert err <= LSE_TOL, f"max|LSE-LSE_ref| = {err}"


def _pairless(mask, B, Hq, Hkv, N, causal):
    """Query rows [B, Hq, N] that see no key and key rows [B, Hkv, N] that no query sees."""
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = mask.numpy()[:, :, i // 128, j // 128] != 0      # [B, Hq, N, N]
    if causal:
        vis &= (j <= i)[None, None]
    q_none = ~vis.any(axis=3)
    k_seen = vis.any(axis=2).reshape(B, Hkv, Hq // Hkv, N).any(axis=2)
    return q_none, ~k_seen


def check_bwd_bs(dq, dk, dv, q, k, v, do, mask, causal, scale):
    dq_r, dk_r, dv_r = oracle.attention_bwd_blocksparse(_f64(q), _f64(k), _f64(v), _f64(do),
                                                        mask.numpy(), causal, scale)
    B, Hq, N, _ = q.shape
    q_none, k_none = _pairless(mask, B, Hq, k.shape[1], N, causal)
    for name, x, ref, none in (("dQ", dq, dq_r, q_none), ("dK", dk, dk_r, k_none),
                               ("dV", dv, dv_r, k_none)):
        x = _f64(x)
        assert np.isfinite(x).all(), f"{name} not finite"
        # rows the mask leaves without any pair have exactly zero gradient (a row that sees a
        # single key has dQ = 0 only up to rounding: dP and Delta are summed differently)
        assert np.all(x[none] == 0.0), f"{name}: rows without pairs must be 0"
        if np.abs(ref).max() == 0.0:
            continue
        err = _rel_fro(x, ref)
        assert err <= GRAD_TOL, f"{name} relative Frobenius error {err}"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [257, 700])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("density", [0.3, 0.7])
def test_blocksparse_fwd_bwd(d, N, causal, density):
    q, k, v, do = draw(1, 4, 2, N, d, seed=9000 + N + d + int(causal) + int(10 * density))
    mask = draw_block_mask(1, 4, N, density, seed=N + d + int(100 * density))
    scale = 1.0 / math.sqrt(d)
    o, lse = run_fwd_bs(q, k, v, mask, causal, scale)
    check_fwd_bs(o, lse, q, k, v, mask, causal, scale)
    dq, dk, dv = run_bwd_bs(q, k, v, o, lse, do, mask, causal, scale)
    check_bwd_bs(dq, dk, dv, q, k, v, do, mask, causal, scale)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (3, 1), (4, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_heads_and_groups(Hq, Hkv, causal):
    # (8, 2): a forward CTA owns the same query block of two heads whose masks differ;
    # (3, 1) and (4, 4): two query blocks of one head.  The backward walks every head of
    # the group over each key block.
    q, k, v, do = draw(2, Hq, Hkv, 520, 128, seed=9100 + Hq * 10 + Hkv + int(causal))
    mask = draw_block_mask(2, Hq, 520, 0.5, seed=Hq * 7 + Hkv)
    scale = 0.0883883461356163
    o, lse = run_fwd_bs(q, k, v, mask, causal, scale)
    check_fwd_bs(o, lse, q, k, v, mask, causal, scale)
    dq, dk, dv = run_bwd_bs(q, k, v, o, lse, do, mask, causal, scale)
    check_bwd_bs(dq, dk, dv, q, k, v, do, mask, causal, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_all_ones_mask_equals_dense_calls_bitwise(d):
    N = 300
    q, k, v, do = draw(1, 4, 2, N, d, seed=9200 + d)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    nb = (N + 127) // 128
    ones = torch.ones(1, 4, nb, nb, dtype=torch.uint8, device="cuda")
    for causal in (False, True):
        o1, l1 = fa.fwd(qd, kd, vd, causal=causal)
        o2, l2 = fa.fwd(qd, kd, vd, causal=causal, block_mask=ones)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        g1 = fa.bwd(qd, kd, vd, o1, l1, dod, causal=causal)
        g2 = fa.bwd(qd, kd, vd, o1, l1, dod, causal=causal, block_mask=ones)
        torch.cuda.synchronize()
        if d == 256:
            # The dense d = 256 backward runs as CTA pairs (64-row query steps, P^T sent as
            # bf16 to the CTA that forms dS^T), the block-sparse one as the single-CTA
            # d-split kernel, so they agree to rounding, not bit for bit.
            for a1, a2 in zip(g1, g2):
                assert _rel_fro(_f64(a1), _f64(a2)) < 1e-2
            continue
        assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
        # dQ sums the key blocks' fp32 partials with reduce-adds in whatever order the
        # CTAs finish, so two runs of the same kernel agree only up to rounding.
        assert _rel_fro(_f64(g1[0]), _f64(g2[0])) < 1e-3


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [1, 130])
def test_all_zeros_mask(d, N):
    q, k, v, do = draw(1, 2, 1, N, d, seed=9300 + d + N)
    nb = (N + 127) // 128
    zeros = torch.zeros(1, 2, nb, nb, dtype=torch.uint8)
    o, lse = run_fwd_bs(q, k, v, zeros, False, 0.1)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    dq, dk, dv = run_bwd_bs(q, k, v, o, lse, do, zeros, False, 0.1)
    assert torch.all(dq == 0) and torch.all(dk == 0) and torch.all(dv == 0)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_structured_masks(d):
    # Block-diagonal, one empty query row of blocks, one empty key column of blocks, and a
    # mask that keeps only blocks above the diagonal (nothing left once causal).
    N = 640
    nb = 5
    q, k, v, do = draw(1, 2, 2, N, d, seed=9400 + d)
    masks = []
    m = torch.zeros(1, 2, nb, nb, dtype=torch.uint8)
    m[:, :, range(nb), range(nb)] = 1
    masks.append(m)
    m = torch.ones(1, 2, nb, nb, dtype=torch.uint8)
    m[:, 0, 2, :] = 0
    m[:, 1, :, 3] = 0
    masks.append(m)
    masks.append(torch.triu(torch.ones(nb, nb, dtype=torch.uint8), 1).expand(1, 2, nb, nb).contiguous())
    scale = 1.0 / math.sqrt(d)
    for mask in masks:
        for causal in (False, True):
            o, lse = run_fwd_bs(q, k, v, mask, causal, scale)
            check_fwd_bs(o, lse, q, k, v, mask, causal, scale)
            dq, dk, dv = run_bwd_bs(q, k, v, o, lse, do, mask, causal, scale)
            check_bwd_bs(dq, dk, dv, q, k, v, do, mask, causal, scale)


@pytest.mark.parametrize("d", [128, 256])
def test_blocksparse_stress_large_scores(d):
    # Large scores move the running max between the enabled blocks, which are not
    # adjacent: the rescale of O must follow the visited blocks, not the block index.
    q, k, v, do = draw(1, 2, 2, 896, d, seed=9500 + d, q_std=4.0)
    mask = draw_block_mask(1, 2, 896, 0.4, seed=55)
    scale = 0.35 if d == 128 else 0.25
    for causal in (False, True):
        o, lse = run_fwd_bs(q, k, v, mask, causal, scale)
        check_fwd_bs(o, lse, q, k, v, mask, causal, scale)
        dq, dk, dv = run_bwd_bs(q, k, v, o, lse, do, mask, causal, scale)
        check_bwd_bs(dq, dk, dv, q, k, v, do, mask, causal, scale)


def test_blocksparse_full_size_8k():
    # 8k tokens, 16 heads, a quarter of the causal blocks enabled (the diagonal always):
    # one head compared row by row with the oracle, and the invariant sum_j dK_j = 0
    # checked for every head.
    B, H, N, d = 1, 16, 8192, 128
    q, k, v, do = draw(B, H, H, N, d, seed=9600)
    mask = draw_block_mask(B, H, N, 0.25, seed=96, diagonal=True)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, dod, md = q.cuda(), k.cuda(), v.cuda(), do.cuda(), mask.cuda()
    o, lse = fa.fwd(qd, kd, vd, causal=True, scale=scale, block_mask=md)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=True, scale=scale, block_mask=md)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    o, lse, dq, dk, dv = (t.cpu() for t in (o, lse, dq, dk, dv))
    h = 5
    sl = slice(h, h + 1)
    check_fwd_bs(o[:, sl], lse[:, sl], q[:, sl], k[:, sl], v[:, sl], mask[:, sl].contiguous(), True, scale)
    check_bwd_bs(dq[:, sl], dk[:, sl], dv[:, sl], q[:, sl], k[:, sl], v[:, sl], do[:, sl],
                 mask[:, sl].contiguous(), True, scale)
    dk64 = _f64(dk)
    assert np.abs(dk64.sum(axis=2)).max() <= 2e-2 * np.abs(dk64).sum(axis=2).max()
