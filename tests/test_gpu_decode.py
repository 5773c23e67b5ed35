"""GPU parity of decode (a few new query rows against a long key/value cache, split over
the cache) and of the merge of partial results, against the fp64 oracle.

Tolerances as for the dense forward: |O - O_ref| <= max(1e-2, one bf16 spacing of
O_ref), |LSE - LSE_ref| <= 1e-3, and rows that see no key must give O = 0 and LSE = -inf
exactly.  Guard bands around O and LSE must stay untouched.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw_decode
from test_gpu_parity import LSE_TOL, SENT_BF16, SENT_F32, _f64, _guarded, _guards_intact, o_tolerance

pytestmark = pytest.mark.gpu


def run_decode(q, k, v, lens, causal, scale, num_splits):
    B, Hq, Nq, d = q.shape
    ob, o = _guarded(q.shape, torch.bfloat16, SENT_BF16)
    lb, lse = _guarded((B, Hq, Nq), torch.float32, SENT_F32)
    lens_d = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
    fa.decode(q.cuda(), k.cuda(), v.cuda(), seqlens_k=lens_d, causal=causal, scale=scale,
              num_splits=num_splits, out=o, lse=lse)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    assert _guards_intact(ob, SENT_BF16), "write outside O"
    assert _guards_intact(lb, SENT_F32), "write outside LSE"
    return o.cpu(), lse.cpu()


def check_decode(o, lse, q, k, v, lens, causal, scale):
    o_ref, lse_ref = oracle.attention_decode(_f64(q), _f64(k), _f64(v), lens, causal, scale)
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


# (Hq, Hkv, Nq): query rows per K/V head R = Hq / Hkv * Nq of 1, 4, 8, 16, 32, 40, 64, 128.
SHAPES = [(4, 4, 1), (8, 2, 1), (32, 4, 1), (8, 2, 4), (8, 1, 4), (16, 2, 5), (8, 1, 8), (8, 1, 16)]


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Hq,Hkv,Nq", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_decode_shapes(d, Hq, Hkv, Nq, causal):
    if d == 256 and Hq // Hkv * Nq > 64:
        pytest.skip("d = 256 takes at most 64 query rows per K/V head")
    Nk = 700
    q, k, v = draw_decode(2, Hq, Hkv, Nq, Nk, d, seed=100 + d + Hq + Nq)
    lens = [Nk, 389]
    scale = 1.0 / math.sqrt(d)
    for splits in (1, 3):
        o, lse = run_decode(q, k, v, lens, causal, scale, splits)
        check_decode(o, lse, q, k, v, lens, causal, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Nk,lens", [(1, None), (1, [0, 1]), (129, [0, 129]), (128, [5, 127]),
                                      (1000, [1, 999]), (4097, [4097, 2048]), (300, [2, 3])])
@pytest.mark.parametrize("splits", [1, 2, 7, None])
def test_decode_lengths_and_splits(d, Nk, lens, splits):
    # Lengths at block edges, empty caches, more splits than blocks (empty key ranges),
    # and the library's own split count.
    q, k, v = draw_decode(2, 8, 2, 3, Nk, d, seed=Nk + d)
    scale = 1.0 / math.sqrt(d)
    for causal in (False, True):
        o, lse = run_decode(q, k, v, lens, causal, scale, splits)
        check_decode(o, lse, q, k, v, lens, causal, scale)


def test_decode_with_square_queries_matches_the_forward():
    # Nq = Nk (the queries are the whole sequence): decode and fa_fwd compute the same
    # attention, bottom-right and top-left alignment agreeing.
    q, k, v = draw_decode(1, 2, 2, 100, 100, 128, seed=9)
    for causal in (False, True):
        o1, l1 = run_decode(q, k, v, None, causal, 0.1, 1)
        o2, l2 = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=0.1)
        torch.cuda.synchronize()
        assert float((o1.float() - o2.cpu().float()).abs().max()) <= 1e-2
        assert float((l1 - l2.cpu()).abs().max()) <= 1e-3


def test_decode_large_scores_move_the_max():
    # Q ~ N(0, 4^2) and a large scale: the running max moves between key blocks, which
    # exercises the rescale of O^T and of the probability sums.
    q, k, v = draw_decode(1, 8, 1, 2, 3000, 128, seed=11, q_std=4.0)
    for splits in (1, 4):
        o, lse = run_decode(q, k, v, None, True, 0.35, splits)
        check_decode(o, lse, q, k, v, None, True, 0.35)


def test_decode_full_size_sampled():
    # 64k-token caches, 32 query heads over 8 K/V heads, one new token, ragged lengths:
    # the oracle checks every row of two sampled (b, K/V head) groups.
    B, Hq, Hkv, Nq, Nk, d = 4, 32, 8, 1, 65536, 128
    q, k, v = draw_decode(B, Hq, Hkv, Nq, Nk, d, seed=12)
    lens = [65536, 40000, 1, 65000]
    scale = 1.0 / math.sqrt(d)
    o, lse = run_decode(q, k, v, lens, False, scale, None)
    g = Hq // Hkv
    for b, kh in ((0, 0), (3, Hkv - 1), (1, 3)):
        hs = slice(kh * g, (kh + 1) * g)
        check_decode(o[b:b + 1, hs], lse[b:b + 1, hs], q[b:b + 1, hs].contiguous(),
                     k[b:b + 1, kh:kh + 1].contiguous(), v[b:b + 1, kh:kh + 1].contiguous(),
                     [lens[b]], False, scale)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("S", [1, 2, 5, 33])
def test_merge_against_oracle(d, S):
    g = torch.Generator().manual_seed(S * 1000 + d)
    rows = 300
    o_parts = torch.randn(S, rows, d, generator=g)
    lse_parts = torch.randn(S, rows, generator=g) * 3.0
    lse_parts[0, :50] = -math.inf                 # some empty parts
    if S > 1:
        lse_parts[:, 50:60] = -math.inf           # rows with every part empty
    ob, o = _guarded((rows, d), torch.bfloat16, SENT_BF16)
    lb, lse = _guarded((rows,), torch.float32, SENT_F32)
    fa.merge(o_parts.cuda(), lse_parts.cuda(), out=o, lse=lse)
    torch.cuda.synchronize()
    assert _guards_intact(ob, SENT_BF16) and _guards_intact(lb, SENT_F32)
    o_ref, lse_ref = oracle.merge(o_parts.double().numpy(), lse_parts.double().numpy())
    lse64 = lse.cpu().double().numpy()
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse64), empty)
    assert np.abs(lse64[~empty] - lse_ref[~empty]).max() <= 1e-5
    o64 = _f64(o.cpu())
    assert np.all(o64[empty] == 0.0)
    assert float(np.max(np.abs(o64 - o_ref) - o_tolerance(o_ref))) <= 0.0
