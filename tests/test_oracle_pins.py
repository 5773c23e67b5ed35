"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign, a swapped index, K used where V belongs, the wrong K/V head for a query head,
the causal mask on the wrong side, a missing scale) fails at least one test:

* closed forms: Q = 0 (uniform softmax), V = 1 (rows of P sum to one), a one-hot
  dominant score, N = 1;
* the toy 4x4 example printed on the "Consideration is All You Want" page, with values
  derived by hand (tests/golden/p5_toy_scores.txt);
* the online-softmax recurrence of the "FlashAttention1" Q&A page and a tiled forward
  that merges blocks with the rescaling described on the "flash attention deep dive"
  page ("Intuition"), against the oracle's two-pass rows;
* scipy's logsumexp for the LSE;
* central finite differences of L = <O, dO> for the gradient;
* Delta_i = <dO_i, O_i>, sum_j dK_j = 0, sum_j dV_j = sum_i dO_i;
* grouped-query attention equals multi-head attention with repeated K/V;
* local attention against a brute-force masked softmax and its full/causal special cases;
* decode (queries at the end of a longer cache) against a bottom-right-masked softmax on
  the full score matrix, the square forward, and single-key / no-key closed forms;
* the merge of partial results against attention over the union of the key ranges, and
  closed forms (one part, equal weights, weights 1/4 and 3/4, all parts empty);
* packed variable-length batches against the dense oracle per sequence (equal lengths),
  the decode oracle per sequence (unequal lengths, bottom-right band), a brute-force
  masked softmax for banded windows, and central finite differences;
* block-sparse: an all-ones mask is dense attention, a block-diagonal mask is independent
  chunks, random masks (with an empty block row) equal a brute-force masked softmax, and
  central finite differences;
* dropout: p = 0 is plain attention, the forward equals the reweighted masked softmax
  built from the keep mask, it is unbiased over seeds, its gradient matches central
  differences, and the keep mask has the right rate for six p and no visible correlation
  between neighbouring keys, rows, heads or seeds;
* the dropout generator: the oracle's Philox4x32-10 equals, word for word, PyTorch's
  ATen Philox engine (an independent implementation of the same published generator,
  compiled here from its C++ header), and the keep mask is exactly the stated selection
  of 16-bit halves of that engine's output.
"""
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p5_toy_scores.txt")


def _load_golden():
    scores, vals = [], {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) == 4:
                scores.append([float(x) for x in parts])
            else:
                vals[parts[0]] = float(parts[1])
    return np.array(scores), vals


def _embed_scores(S):
    """Q = I, K = S^T, V = I, scale 1: then Q K^T = S and O = P."""
    n = S.shape[0]
    q = np.eye(n)[None, None]
    k = S.T.copy()[None, None]
    v = np.eye(n)[None, None]
    return q, k, v


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------------------- forward


def test_toy_example_non_causal():
    S, gv = _load_golden()
    q, k, v = _embed_scores(S)
    o, lse = oracle.attention_fwd(q, k, v, causal=False, scale=1.0)
    np.testing.assert_allclose(lse[0, 0], gv["lse_full"], rtol=0, atol=1e-13)
    p_of = {s: gv[f"p_of_{s}"] for s in (1, 2, 3, 4)}
    expect = np.vectorize(lambda s: p_of[int(s)])(S)
    np.testing.assert_allclose(o[0, 0], expect, rtol=0, atol=1e-13)


def test_toy_example_causal():
    S, gv = _load_golden()
    q, k, v = _embed_scores(S)
    o, lse = oracle.attention_fwd(q, k, v, causal=True, scale=1.0)
    np.testing.assert_allclose(
        lse[0, 0], [gv[f"lse_causal_{r}"] for r in "ABCD"], rtol=0, atol=1e-13)
    # Row A keeps only key A; row B: softmax(2, 1) over keys A, B; keys after the
    # query get exactly zero weight.
    assert o[0, 0, 0, 0] == 1.0 and np.all(o[0, 0, 0, 1:] == 0.0)
    np.testing.assert_allclose(o[0, 0, 1, :2], [math.e / (math.e + 1), 1 / (math.e + 1)],
                               atol=1e-15)
    assert np.all(o[0, 0, 1, 2:] == 0.0) and np.all(o[0, 0, 2, 3:] == 0.0)


def test_toy_example_online_recurrence_2x2_tiles():
    S, gv = _load_golden()
    m, l = oracle.online_softmax_stats(S[0], block=2)
    assert m == gv["row_A_tile2_m"]
    assert abs(l - gv["row_A_tile2_l"]) < 1e-14
    assert abs(m + math.log(l) - gv["lse_full"]) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_values(causal):
    B, Hq, Hkv, N, d = 2, 4, 2, 9, 5
    r = _rng(1)
    q = np.zeros((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    o, lse = oracle.attention_fwd(q, k, v, causal, scale=0.3)
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            for i in range(N):
                J = i + 1 if causal else N
                np.testing.assert_allclose(o[b, h, i], v[b, h // g, :J].mean(0), atol=1e-14)
                assert abs(lse[b, h, i] - math.log(J)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    r = _rng(2)
    q = 3 * r.standard_normal((1, 2, 33, 8))
    k = r.standard_normal((1, 2, 33, 8))
    v = np.ones((1, 2, 33, 8))
    o, _ = oracle.attention_fwd(q, k, v, causal, scale=0.5)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_one_hot_dominant_score_selects_value_row(causal):
    # K = I (N <= d) and q_i = alpha e_t(i): s_ij = scale*alpha*[j == t(i)].  With
    # scale*alpha = 800 every other weight is exp(-800), which underflows in fp64, so
    # O_i = v_t(i) and LSE_i = 800 exactly.
    N, d = 6, 8
    r = _rng(3)
    t = [int(r.integers(0, (i + 1) if causal else N)) for i in range(N)]
    q = np.zeros((1, 1, N, d))
    for i, ti in enumerate(t):
        q[0, 0, i, ti] = 1600.0
    k = np.zeros((1, 1, N, d))
    k[0, 0, :, :N] = np.eye(N)
    v = r.standard_normal((1, 1, N, d))
    o, lse = oracle.attention_fwd(q, k, v, causal, scale=0.5)
    for i, ti in enumerate(t):
        np.testing.assert_array_equal(o[0, 0, i], v[0, 0, ti])
        assert lse[0, 0, i] == 800.0


def test_single_token_causal():
    r = _rng(4)
    q, k, v = (r.standard_normal((1, 1, 1, 4)) for _ in range(3))
    o, lse = oracle.attention_fwd(q, k, v, True, scale=0.7)
    np.testing.assert_array_equal(o[0, 0, 0], v[0, 0, 0])
    assert abs(lse[0, 0, 0] - 0.7 * float(q[0, 0, 0] @ k[0, 0, 0])) < 1e-15


@pytest.mark.parametrize("causal", [False, True])
def test_lse_matches_scipy_logsumexp(causal):
    r = _rng(5)
    N, d, scale = 40, 16, 0.25
    q = 4 * r.standard_normal((1, 1, N, d))
    k = r.standard_normal((1, 1, N, d))
    v = r.standard_normal((1, 1, N, d))
    _, lse = oracle.attention_fwd(q, k, v, causal, scale)
    for i in range(N):
        J = i + 1 if causal else N
        s = scale * (k[0, 0, :J] @ q[0, 0, i])
        assert abs(lse[0, 0, i] - scipy.special.logsumexp(s)) < 1e-12


@pytest.mark.parametrize("block", [1, 2, 3, 7, 128, 1000])
def test_online_softmax_stats_equal_two_pass(block):
    r = _rng(6)
    for scale in (1.0, 30.0):
        s = scale * r.standard_normal(300)
        m, l = oracle.online_softmax_stats(s, block)
        assert m == s.max()
        assert abs((m + math.log(l)) - scipy.special.logsumexp(s)) < 1e-12


def _tiled_forward(q, k, v, causal, scale, Br, Bc):
    """Block-by-block forward: running max, running sum and a running numerator that is
    rescaled by exp(old max - new max) whenever a key block raises the max; tiles wholly
    above the diagonal are skipped and the diagonal tile is masked element-wise."""
    N, d = q.shape
    o = np.zeros((N, d))
    lse = np.zeros(N)
    for r0 in range(0, N, Br):
        rows = range(r0, min(r0 + Br, N))
        m = np.full(len(rows), -np.inf)
        l = np.zeros(len(rows))
        acc = np.zeros((len(rows), d))
        for c0 in range(0, N, Bc):
            if causal and c0 > rows[-1]:
                break  # tile entirely above the diagonal
            cols = np.arange(c0, min(c0 + Bc, N))
            s = scale * (q[list(rows)] @ k[cols].T)
            if causal:
                s = np.where(cols[None, :] <= np.array(list(rows))[:, None], s, -np.inf)
            bm = s.max(axis=1)
            mn = np.maximum(m, bm)
            alpha = np.where(np.isneginf(m), 0.0, np.exp(m - mn))
            p = np.exp(s - mn[:, None])
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v[cols]
            m = mn
        o[list(rows)] = acc / l[:, None]
        lse[list(rows)] = m + np.log(l)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Br,Bc", [(1, 1), (2, 2), (3, 5), (16, 16), (128, 128)])
def test_tiled_online_forward_equals_oracle(causal, Br, Bc):
    r = _rng(7)
    N, d, scale = 37, 8, 0.35
    q = 4 * r.standard_normal((N, d))
    k = r.standard_normal((N, d))
    v = r.standard_normal((N, d))
    o_t, lse_t = _tiled_forward(q, k, v, causal, scale, Br, Bc)
    o, lse = oracle.attention_fwd(q[None, None], k[None, None], v[None, None], causal, scale)
    np.testing.assert_allclose(o[0, 0], o_t, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], lse_t, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------- backward


def _loss(q, k, v, do, causal, scale):
    o, _ = oracle.attention_fwd(q, k, v, causal, scale)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 2), (5, 3), (7, 4)])
def test_gradients_match_central_differences(causal, N, d):
    r = _rng(100 + N * 10 + d + int(causal))
    B, Hq, Hkv, scale = 1, 2, 1, 0.6
    q = r.standard_normal((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    dq, dk, dv, _, _ = oracle.attention_bwd(q, k, v, do, causal, scale)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp = x.copy()
            xp[idx] += h
            xm = x.copy()
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, causal, scale)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, causal, scale)
            num[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(grad - num) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6 or np.linalg.norm(grad - num) < 1e-8, (name, err)


@pytest.mark.parametrize("causal", [False, True])
def test_delta_equals_do_dot_o_and_lse_matches_forward(causal):
    r = _rng(8)
    B, Hq, Hkv, N, d, scale = 2, 4, 2, 23, 8, 0.3
    q = r.standard_normal((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    o, lse_f = oracle.attention_fwd(q, k, v, causal, scale)
    _, _, _, lse_b, delta = oracle.attention_bwd(q, k, v, do, causal, scale)
    np.testing.assert_allclose(delta, np.sum(o * do, axis=-1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_b, lse_f, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_column_sum_invariants(causal):
    r = _rng(9)
    B, Hq, Hkv, N, d, scale = 2, 6, 2, 19, 8, 0.4
    q = 2 * r.standard_normal((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    _, dk, dv, _, _ = oracle.attention_bwd(q, k, v, do, causal, scale)
    g = Hq // Hkv
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    group_do = do.reshape(B, Hkv, g, N, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), group_do, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_mha_with_repeated_kv(causal):
    r = _rng(10)
    B, Hq, Hkv, N, d, scale = 2, 8, 2, 17, 8, 0.3
    g = Hq // Hkv
    q = r.standard_normal((B, Hq, N, d))
    k = r.standard_normal((B, Hkv, N, d))
    v = r.standard_normal((B, Hkv, N, d))
    do = r.standard_normal((B, Hq, N, d))
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    o1, l1 = oracle.attention_fwd(q, k, v, causal, scale)
    o2, l2 = oracle.attention_fwd(q, kr, vr, causal, scale)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-14)
    dq1, dk1, dv1, _, _ = oracle.attention_bwd(q, k, v, do, causal, scale)
    dq2, dk2, dv2, _, _ = oracle.attention_bwd(q, kr, vr, do, causal, scale)
    np.testing.assert_allclose(dq1, dq2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk1, dk2.reshape(B, Hkv, g, N, d).sum(2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv1, dv2.reshape(B, Hkv, g, N, d).sum(2), rtol=1e-12, atol=1e-12)


def test_causal_differs_from_full_only_through_the_mask():
    # Row N-1 of a causal attention sees every key, so it equals the non-causal row.
    r = _rng(11)
    q, k, v = (r.standard_normal((1, 1, 12, 4)) for _ in range(3))
    oc, lc = oracle.attention_fwd(q, k, v, True, 0.5)
    of, lf = oracle.attention_fwd(q, k, v, False, 0.5)
    np.testing.assert_array_equal(oc[0, 0, -1], of[0, 0, -1])
    assert lc[0, 0, -1] == lf[0, 0, -1]
    assert not np.allclose(oc[0, 0, 0], of[0, 0, 0])


def test_invalid_arguments_are_rejected():
    q = np.zeros((1, 3, 4, 2))
    k = np.zeros((1, 2, 4, 2))
    with pytest.raises(RuntimeError):
        oracle.attention_fwd(q, k, k, False, 1.0)  # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.attention_fwd(q, np.zeros((1, 1, 5, 2)), np.zeros((1, 1, 5, 2)), False, 1.0)


# ---------------------------------------------------------------------------- key windows
# Local attention keeps key j for query i iff i - left <= j <= i + right (a negative bound
# is unlimited; causal attention is right = 0).


def _brute_window(q, k, v, left, right, scale):
    """Masked two-pass softmax over a full score matrix (small sizes only)."""
    N = q.shape[0]
    s = scale * (q @ k.T)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = np.ones((N, N), dtype=bool)
    if left >= 0:
        vis &= j >= i - left
    if right >= 0:
        vis &= j <= i + right
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p / l) @ v, (m + np.log(l))[:, 0]


@pytest.mark.parametrize("left,right", [(-1, -1), (-1, 0), (3, 0), (0, 0), (5, 2), (2, -1),
                                        (0, 4), (100, 100)])
def test_window_forward_equals_masked_softmax(left, right):
    r = _rng(20 + left + 3 * right)
    N, d, scale = 29, 8, 0.4
    q = 3 * r.standard_normal((N, d))
    k = r.standard_normal((N, d))
    v = r.standard_normal((N, d))
    o, lse = oracle.attention_fwd_window(q[None, None], k[None, None], v[None, None], left,
                                         right, scale)
    o_b, lse_b = _brute_window(q, k, v, left, right, scale)
    np.testing.assert_allclose(o[0, 0], o_b, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], lse_b, rtol=1e-13, atol=1e-13)


def test_window_special_cases():
    r = _rng(31)
    q, k, v = (r.standard_normal((2, 2, 17, 4)) for _ in range(3))
    # Unlimited window = full attention; right = 0 with no left limit = causal.
    for causal, (left, right) in ((False, (-1, -1)), (True, (-1, 0))):
        o1, l1 = oracle.attention_fwd(q, k, v, causal, 0.5)
        o2, l2 = oracle.attention_fwd_window(q, k, v, left, right, 0.5)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(l1, l2)
    # A zero-width window keeps only the diagonal: O_i = v_i, LSE_i = s_ii.
    o, lse = oracle.attention_fwd_window(q, k, v, 0, 0, 0.5)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse, 0.5 * np.einsum("bhnd,bhnd->bhn", q, k), atol=1e-15)


@pytest.mark.parametrize("left,right", [(2, 0), (1, 2), (-1, 1)])
def test_window_gradients_match_central_differences(left, right):
    r = _rng(40 + left + right)
    N, d, scale = 6, 3, 0.6
    q = r.standard_normal((1, 2, N, d))
    k = r.standard_normal((1, 1, N, d))
    v = r.standard_normal((1, 1, N, d))
    do = r.standard_normal((1, 2, N, d))
    dq, dk, dv, _, _ = oracle.attention_bwd_window(q, k, v, do, left, right, scale)

    def loss(q_, k_, v_):
        o, _ = oracle.attention_fwd_window(q_, k_, v_, left, right, scale)
        return float(np.sum(o * do))

    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v, name: xp}
            args_m = {"q": q, "k": k, "v": v, name: xm}
            num[idx] = (loss(args_p["q"], args_p["k"], args_p["v"])
                        - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        err = np.linalg.norm(grad - num) / max(np.linalg.norm(num), 1e-30)
        assert err < 1e-6, (name, err)


# ---------------------------------------------------------------------------- decode / merge

def _brute_decode(q, k, v, lens, causal, scale):
    """Bottom-right-aligned masked softmax on the full score matrix, with numpy."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        n = Nk if lens is None else lens[b]
        for h in range(Hq):
            s = scale * q[b, h] @ k[b, h // g, :n].T               # [Nq, n]
            if causal:
                pos = n - Nq + np.arange(Nq)                        # absolute query positions
                s = np.where(np.arange(n)[None, :] <= pos[:, None], s, -np.inf)
            for t in range(Nq):
                if not np.isfinite(s[t]).any():
                    continue
                lse[b, h, t] = scipy.special.logsumexp(s[t])
                o[b, h, t] = np.exp(s[t] - lse[b, h, t]) @ v[b, h // g, :n]
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq,Nk,lens", [(1, 9, None), (3, 9, [9, 4]), (4, 6, [2, 6]),
                                         (5, 5, [0, 5]), (2, 7, [1, 7])])
def test_decode_equals_bottom_right_masked_softmax(causal, Nq, Nk, lens):
    r = _rng(31 + Nq * 7 + Nk)
    q = r.normal(size=(2, 4, Nq, 8))
    k = r.normal(size=(2, 2, Nk, 8))
    v = r.normal(size=(2, 2, Nk, 8))
    o, lse = oracle.attention_decode(q, k, v, lens, causal, 0.4)
    o_ref, lse_ref = _brute_decode(q, k, v, lens, causal, 0.4)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_decode_with_nq_equal_nk_is_the_square_forward(causal):
    # When the queries are the whole sequence, bottom-right and top-left alignment agree.
    r = _rng(41)
    q, k, v = r.normal(size=(2, 4, 11, 6)), r.normal(size=(2, 2, 11, 6)), r.normal(size=(2, 2, 11, 6))
    o1, l1 = oracle.attention_decode(q, k, v, None, causal, 0.3)
    o2, l2 = oracle.attention_fwd(q, k, v, causal, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_decode_special_cases():
    r = _rng(43)
    q, k, v = r.normal(size=(2, 2, 1, 5)), r.normal(size=(2, 1, 8, 5)), r.normal(size=(2, 1, 8, 5))
    # One query: the causal mask hides nothing.
    o1, l1 = oracle.attention_decode(q, k, v, [8, 3], True, 0.5)
    o2, l2 = oracle.attention_decode(q, k, v, [8, 3], False, 0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # lens[b] valid keys equal a cache that holds only those keys.
    o3, l3 = oracle.attention_decode(q[1:], k[1:, :, :3], v[1:, :, :3], None, False, 0.5)
    np.testing.assert_allclose(o2[1:], o3, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l2[1:], l3, rtol=0, atol=1e-14)
    # A single visible key: O is that key's value row, LSE its scaled score.
    o4, l4 = oracle.attention_decode(q, k, v, [1, 1], False, 0.5)
    np.testing.assert_allclose(o4[:, :, 0], np.broadcast_to(v[:, :, 0], (2, 2, 5)), atol=1e-15)
    np.testing.assert_allclose(l4[:, :, 0], 0.5 * np.einsum("bhd,bd->bh", q[:, :, 0], k[:, 0, 0]),
                               atol=1e-14)
    # No visible key: O = 0, LSE = -inf.
    o5, l5 = oracle.attention_decode(q, k, v, [0, 2], False, 0.5)
    assert np.all(o5[0] == 0) and np.all(np.isneginf(l5[0]))
    with pytest.raises(RuntimeError):
        oracle.attention_decode(q, k, v, [9, 1], False, 0.5)   # more keys than the cache


@pytest.mark.parametrize("bounds", [[0, 4, 9, 16], [0, 1, 2, 16], [0, 16], [0, 5, 5, 12, 16]])
def test_merge_of_disjoint_key_ranges_is_full_attention(bounds):
    # Attention over each key range separately, merged, equals attention over all keys; an
    # empty range (LSE = -inf) contributes nothing.
    r = _rng(47)
    q, k, v = r.normal(size=(1, 3, 4, 7)), r.normal(size=(1, 3, 16, 7)), r.normal(size=(1, 3, 16, 7))
    parts_o, parts_l = [], []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b == a:
            parts_o.append(np.full_like(q, 123.0))   # must be ignored: its weight is zero
            parts_l.append(np.full(q.shape[:-1], -np.inf))
        else:
            o_s, l_s = oracle.attention_decode(q, k[:, :, a:b], v[:, :, a:b], None, False, 0.35)
            parts_o.append(o_s)
            parts_l.append(l_s)
    o, lse = oracle.merge(np.stack(parts_o), np.stack(parts_l))
    o_ref, lse_ref = oracle.attention_decode(q, k, v, None, False, 0.35)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-13)


def test_merge_closed_forms():
    r = _rng(53)
    o1 = r.normal(size=(1, 3, 4))
    l1 = r.normal(size=(1, 3))
    # One part: identity.
    o, lse = oracle.merge(o1, l1)
    np.testing.assert_array_equal(o, o1[0])
    np.testing.assert_array_equal(lse, l1[0])
    # Two parts with equal LSE: the mean, and LSE + ln 2.
    o2 = r.normal(size=(1, 3, 4))
    o, lse = oracle.merge(np.concatenate([o1, o2]), np.concatenate([l1, l1]))
    np.testing.assert_allclose(o, 0.5 * (o1[0] + o2[0]), atol=1e-15)
    np.testing.assert_allclose(lse, l1[0] + math.log(2.0), atol=1e-15)
    # LSEs 0 and ln 3: weights 1/4 and 3/4.
    l2 = np.zeros((1, 3))
    l3 = np.full((1, 3), math.log(3.0))
    o, lse = oracle.merge(np.concatenate([o1, o2]), np.concatenate([l2, l3]))
    np.testing.assert_allclose(o, 0.25 * o1[0] + 0.75 * o2[0], atol=1e-15)
    np.testing.assert_allclose(lse, math.log(4.0), atol=1e-15)
    # All parts empty.
    o, lse = oracle.merge(np.concatenate([o1, o2]), np.full((2, 3), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    # Order of the parts does not matter.
    oa, la = oracle.merge(np.concatenate([o1, o2]), np.concatenate([l1, l3]))
    ob, lb = oracle.merge(np.concatenate([o2, o1]), np.concatenate([l3, l1]))
    np.testing.assert_allclose(oa, ob, atol=1e-15)
    np.testing.assert_allclose(la, lb, atol=1e-15)


# ---------------------------------------------------------------------------- variable length

def _pack(rng, lens, H, d):
    """[total, H, d] packed rows and the [B+1] offsets."""
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return rng.normal(size=(int(cu[-1]), H, d)), cu


def _seq(x, cu, b):
    """Rows of sequence b as a dense [1, H, L, d] array."""
    return np.ascontiguousarray(x[cu[b]:cu[b + 1]].transpose(1, 0, 2)[None])


@pytest.mark.parametrize("left,right", [(-1, -1), (-1, 0), (3, 1), (0, 0)])
def test_varlen_with_equal_lengths_is_the_dense_oracle_per_sequence(left, right):
    r = _rng(61)
    lens = [5, 1, 9]
    q, cu = _pack(r, lens, 4, 6)
    k, _ = _pack(r, lens, 2, 6)
    v, _ = _pack(r, lens, 2, 6)
    do, _ = _pack(r, lens, 4, 6)
    o, lse = oracle.attention_fwd_varlen(q, k, v, cu, cu, left, right, 0.45)
    dq, dk, dv = oracle.attention_bwd_varlen(q, k, v, do, cu, cu, left, right, 0.45)
    for b in range(len(lens)):
        o_b, l_b = oracle.attention_fwd_window(_seq(q, cu, b), _seq(k, cu, b), _seq(v, cu, b),
                                               left, right, 0.45)
        np.testing.assert_allclose(_seq(o, cu, b), o_b, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[cu[b]:cu[b + 1]].T[None], l_b, rtol=0, atol=1e-13)
        g = oracle.attention_bwd_window(_seq(q, cu, b), _seq(k, cu, b), _seq(v, cu, b),
                                        _seq(do, cu, b), left, right, 0.45)
        for x, ref in ((dq, g[0]), (dk, g[1]), (dv, g[2])):
            np.testing.assert_allclose(_seq(x, cu, b), ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_with_unequal_lengths_is_decode_per_sequence(causal):
    # Lq != Lk: the band is aligned to the end of the sequence, which is exactly the
    # decode oracle's bottom-right convention (Lq > Lk leaves early causal rows empty).
    r = _rng(67)
    lq, lk = [3, 7, 2, 4], [8, 7, 0, 2]
    q, cq = _pack(r, lq, 4, 5)
    k, ck = _pack(r, lk, 2, 5)
    v, _ = _pack(r, lk, 2, 5)
    o, lse = oracle.attention_fwd_varlen(q, k, v, cq, ck, -1, 0 if causal else -1, 0.6)
    for b in range(4):
        if lk[b] == 0:
            assert np.all(_seq(o, cq, b) == 0) and np.all(np.isneginf(lse[cq[b]:cq[b + 1]]))
            continue
        o_b, l_b = oracle.attention_decode(_seq(q, cq, b), _seq(k, ck, b), _seq(v, ck, b), None,
                                           causal, 0.6)
        np.testing.assert_allclose(_seq(o, cq, b), o_b, rtol=0, atol=1e-13)
        got = lse[cq[b]:cq[b + 1]].T[None]
        np.testing.assert_array_equal(np.isneginf(got), np.isneginf(l_b))
        fin = np.isfinite(l_b)
        np.testing.assert_allclose(got[fin], l_b[fin], rtol=0, atol=1e-13)


def _brute_varlen(q, k, v, cq, ck, left, right, scale):
    o = np.zeros_like(q)
    lse = np.full(q.shape[:2], -np.inf)
    Hq, Hkv = q.shape[1], k.shape[1]
    for b in range(len(cq) - 1):
        Lq, Lk = cq[b + 1] - cq[b], ck[b + 1] - ck[b]
        i = np.arange(Lq)[:, None] + (Lk - Lq)
        j = np.arange(Lk)[None, :]
        vis = np.ones((Lq, Lk), dtype=bool)
        if left >= 0:
            vis &= j >= i - left
        if right >= 0:
            vis &= j <= i + right
        for h in range(Hq):
            s = scale * q[cq[b]:cq[b + 1], h] @ k[ck[b]:ck[b + 1], h // (Hq // Hkv)].T
            s = np.where(vis, s, -np.inf)
            for t in range(Lq):
                if vis[t].any():
                    lse[cq[b] + t, h] = scipy.special.logsumexp(s[t])
                    o[cq[b] + t, h] = np.exp(s[t] - lse[cq[b] + t, h]) @ v[ck[b]:ck[b + 1], h // (Hq // Hkv)]
    return o, lse


@pytest.mark.parametrize("left,right", [(2, 0), (1, 3), (-1, 2), (4, -1), (0, 0)])
def test_varlen_window_equals_masked_softmax(left, right):
    r = _rng(71)
    lq, lk = [6, 2, 9], [4, 5, 9]
    q, cq = _pack(r, lq, 2, 4)
    k, ck = _pack(r, lk, 1, 4)
    v, _ = _pack(r, lk, 1, 4)
    o, lse = oracle.attention_fwd_varlen(q, k, v, cq, ck, left, right, 0.7)
    o_ref, lse_ref = _brute_varlen(q, k, v, cq, ck, left, right, 0.7)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)


def test_varlen_gradients_match_central_differences():
    r = _rng(73)
    lq, lk = [3, 4], [5, 2]
    q, cq = _pack(r, lq, 2, 3)
    k, ck = _pack(r, lk, 1, 3)
    v, _ = _pack(r, lk, 1, 3)
    do = r.normal(size=q.shape)
    left, right, scale = 2, 1, 0.8

    def loss(q_, k_, v_):
        o_, _ = oracle.attention_fwd_varlen(q_, k_, v_, cq, ck, left, right, scale)
        return float((o_ * do).sum())

    dq, dk, dv = oracle.attention_bwd_varlen(q, k, v, do, cq, ck, left, right, scale)
    eps = 1e-6
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


def test_varlen_invalid_offsets_are_rejected():
    r = _rng(79)
    q, cq = _pack(r, [2, 3], 1, 4)
    with pytest.raises(RuntimeError):
        oracle.attention_fwd_varlen(q, q, q, [0, 3, 2], cq, -1, -1, 1.0)   # decreasing
    with pytest.raises(RuntimeError):
        oracle.attention_fwd_varlen(q, q, q, cq, [0, 2, 9], -1, -1, 1.0)   # past the end


# ---------------------------------------------------------------------------- dropout

@pytest.mark.parametrize("causal", [False, True])
def test_dropout_with_p_zero_is_plain_attention(causal):
    r = _rng(83)
    q, k, v, do = (r.normal(size=(1, 4, 9, 5)) for _ in range(4))
    k, v = k[:, :2], v[:, :2]
    o1, l1 = oracle.attention_fwd_dropout(q, k, v, causal, 0.5, 0.0, 77)
    o2, l2 = oracle.attention_fwd(q, k, v, causal, 0.5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    g1 = oracle.attention_bwd_dropout(q, k, v, do, causal, 0.5, 0.0, 77)
    g2 = oracle.attention_bwd(q, k, v, do, causal, 0.5)[:3]
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)


@pytest.mark.parametrize("p", [0.05, 0.1, 0.25, 0.5, 0.75, 0.9])
def test_dropout_keep_rate_tracks_one_minus_p(p):
    # The keep rate as a function of p is the complement of the 16-bit values' CDF: it
    # must follow 1 - p within 5 standard errors over 4 x 256 x 256 elements.
    keep = oracle.dropout_keep_mask(4, 256, p, seed=2024)
    n = keep.size
    assert abs(keep.mean() - (1 - p)) < 5 * math.sqrt(p * (1 - p) / n)


def test_dropout_mask_has_no_visible_correlation():
    keep = oracle.dropout_keep_mask(2, 256, 0.5, seed=99).astype(np.float64) - 0.5
    n = keep[:, :, 1:].size
    bound = 5 * 0.25 / math.sqrt(n)          # 5 standard errors of a covariance of +-1/2 bits
    assert abs((keep[:, :, 1:] * keep[:, :, :-1]).mean()) < bound    # neighbouring keys
    assert abs((keep[:, 1:, :] * keep[:, :-1, :]).mean()) < bound    # neighbouring rows
    assert abs((keep[1] * keep[0]).mean()) < 5 * 0.25 / math.sqrt(keep[0].size)  # heads
    other = oracle.dropout_keep_mask(2, 256, 0.5, seed=100).astype(np.float64) - 0.5
    assert abs((keep * other).mean()) < 5 * 0.25 / math.sqrt(keep.size)         # seeds
    # Same seed, same mask: the generator is a pure function of (seed, head, row, key).
    again = oracle.dropout_keep_mask(2, 256, 0.5, seed=99).astype(np.float64) - 0.5
    np.testing.assert_array_equal(keep, again)


_ATEN_PHILOX_SRC = r"""
#include <cstdint>
#include <ATen/core/PhiloxRNGEngine.h>
// n generator calls: counter ctr[4 i .. 4 i + 3], key key[2 i .. 2 i + 1] -> out[4 i ..].
// The engine's state is (key = seed, counter = (offset lo, offset hi, subsequence lo,
// subsequence hi)); its first four outputs are the four words of one block.
extern "C" void aten_philox4x32_10(int n, const uint32_t *ctr, const uint32_t *key, uint32_t *out) {
  for (int i = 0; i < n; ++i) {
    const uint32_t *c = ctr + 4 * i, *k = key + 2 * i;
    at::Philox4_32 eng(k[0] | (static_cast<uint64_t>(k[1]) << 32),
                       c[2] | (static_cast<uint64_t>(c[3]) << 32),
                       c[0] | (static_cast<uint64_t>(c[1]) << 32));
    for (int w = 0; w < 4; ++w) out[4 * i + w] = eng();
  }
}
"""


@pytest.fixture(scope="module")
def aten_philox(tmp_path_factory):
    """PyTorch's header-only ATen Philox4x32-10 engine compiled into a tiny shared object:
    an implementation of the generator that shares nothing with the oracle."""
    import ctypes
    import subprocess
    import torch
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    d = tmp_path_factory.mktemp("aten_philox")
    src, lib = d / "aten_philox.cpp", d / "libaten_philox.so"
    src.write_text(_ATEN_PHILOX_SRC)
    cuda_inc = os.environ.get("CUDA_HOME", "/usr/local/cuda") + "/include"
    subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", f"-I{inc}", f"-I{cuda_inc}",
                    str(src), "-o", str(lib)], check=True)
    so = ctypes.CDLL(str(lib))
    u32p = ctypes.POINTER(ctypes.c_uint32)

    def run(ctr, key):
        ctr = np.ascontiguousarray(ctr, dtype=np.uint32).reshape(-1, 4)
        key = np.ascontiguousarray(key, dtype=np.uint32).reshape(-1, 2)
        out = np.empty_like(ctr)
        so.aten_philox4x32_10(ctypes.c_int(len(ctr)), ctr.ctypes.data_as(u32p),
                              key.ctypes.data_as(u32p), out.ctypes.data_as(u32p))
        return out

    return run


def test_philox_equals_the_aten_engine_word_for_word(aten_philox):
    # Seeded random counters and keys over the whole 32-bit range, plus the extremes.
    r = _rng(2011)
    ctr = r.integers(0, 2 ** 32, size=(2000, 4), dtype=np.uint64).astype(np.uint32)
    key = r.integers(0, 2 ** 32, size=(2000, 2), dtype=np.uint64).astype(np.uint32)
    ctr[0], key[0] = 0, 0
    ctr[1], key[1] = 0xFFFFFFFF, 0xFFFFFFFF
    ctr[2] = [7, 0, 0, 0]          # small counters as the dropout mask uses them
    ctr[3] = [0, 5, 3, 0]
    want = aten_philox(ctr, key)
    got = np.stack([oracle.philox4x32_10(c, k) for c, k in zip(ctr, key)])
    np.testing.assert_array_equal(got, want)
    # and the generator is not trivially the identity or constant
    assert len({tuple(w) for w in got}) == len(got)


def test_dropout_mask_is_the_stated_halves_of_the_generator(aten_philox):
    # keep(bh, i, j) iff the 16-bit value j % 8 of Philox(counter (j / 8, i, bh, 0), key
    # (seed low, seed high)) - the low half of word (j % 8) / 2 for even j, the high half
    # for odd j - is >= floor(p 2^16); here the values come from the ATen engine.
    BH, N, p, seed = 3, 41, 0.3, 0x1234ABCD9876F00D
    thr = math.floor(p * 65536)
    bh, i, j8 = np.meshgrid(np.arange(BH), np.arange(N), np.arange((N + 7) // 8), indexing="ij")
    ctr = np.stack([j8.ravel(), i.ravel(), bh.ravel(), np.zeros(bh.size, dtype=np.int64)], axis=1)
    key = np.tile([seed & 0xFFFFFFFF, seed >> 32], (len(ctr), 1))
    words = aten_philox(ctr, key).reshape(BH, N, (N + 7) // 8, 4).astype(np.int64)
    halves = np.stack([words & 0xFFFF, words >> 16], axis=-1).reshape(BH, N, -1)  # value m = 2w + half
    want = (halves[:, :, :N] >= thr).astype(np.uint8)
    np.testing.assert_array_equal(oracle.dropout_keep_mask(BH, N, p, seed), want)


def test_dropout_forward_is_the_masked_reweighted_softmax():
    # Brute force from the keep mask: O = (softmax(S) * Z / (1 - p)) V, LSE unchanged.
    r = _rng(89)
    q, k, v = r.normal(size=(1, 2, 7, 4)), r.normal(size=(1, 2, 7, 4)), r.normal(size=(1, 2, 7, 4))
    p, seed = 0.3, 5
    o, lse = oracle.attention_fwd_dropout(q, k, v, True, 0.8, p, seed)
    keep = oracle.dropout_keep_mask(2, 7, p, seed)
    for h in range(2):
        s = 0.8 * q[0, h] @ k[0, h].T
        s = np.where(np.tril(np.ones((7, 7), dtype=bool)), s, -np.inf)
        P = np.exp(s - scipy.special.logsumexp(s, axis=1, keepdims=True))
        # kept values are scaled by the inverse of the exact keep probability 1 - thr / 2^16
        inv_keep = 65536.0 / (65536.0 - math.floor(p * 65536.0))
        np.testing.assert_allclose(o[0, h], (P * keep[h] * inv_keep) @ v[0, h], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], scipy.special.logsumexp(s, axis=1), atol=1e-13)


def test_dropout_is_unbiased_over_seeds():
    # E_Z[O] = O without dropout: the mean over 400 seeds lies within 5 standard errors.
    r = _rng(97)
    q, k, v = r.normal(size=(1, 1, 6, 3)), r.normal(size=(1, 1, 6, 3)), r.normal(size=(1, 1, 6, 3))
    outs = np.stack([oracle.attention_fwd_dropout(q, k, v, False, 0.7, 0.4, s)[0]
                     for s in range(400)])
    ref, _ = oracle.attention_fwd(q, k, v, False, 0.7)
    se = outs.std(axis=0) / math.sqrt(len(outs))
    assert np.all(np.abs(outs.mean(axis=0) - ref) <= 5 * se + 1e-12)


def test_dropout_gradients_match_central_differences():
    r = _rng(101)
    q, k, v, do = (r.normal(size=(1, 2, 5, 3)) for _ in range(4))
    k, v = k[:, :1], v[:, :1]
    p, seed, scale = 0.35, 123, 0.9
    for causal in (False, True):
        dq, dk, dv = oracle.attention_bwd_dropout(q, k, v, do, causal, scale, p, seed)
        loss = lambda q_, k_, v_: float(
            (oracle.attention_fwd_dropout(q_, k_, v_, causal, scale, p, seed)[0] * do).sum())
        eps = 1e-6
        for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][idx] += eps
                args_m[which][idx] -= eps
                num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------------------- block-sparse

@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_all_ones_is_dense_attention(causal):
    r = _rng(103)
    q, k, v = r.normal(size=(1, 2, 300, 4)), r.normal(size=(1, 1, 300, 4)), r.normal(size=(1, 1, 300, 4))
    ones = np.ones((1, 2, 3, 3), dtype=np.uint8)
    o1, l1 = oracle.attention_fwd_blocksparse(q, k, v, ones, causal, 0.5)
    o2, l2 = oracle.attention_fwd(q, k, v, causal, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)
    # Blocks above the diagonal do not matter under the causal mask.
    tril = np.tril(np.ones((3, 3), dtype=np.uint8))[None, None].repeat(2, axis=1)
    if causal:
        o3, l3 = oracle.attention_fwd_blocksparse(q, k, v, tril, True, 0.5)
        np.testing.assert_array_equal(o3, o1)
        np.testing.assert_array_equal(l3, l1)


def test_blocksparse_block_diagonal_is_independent_chunks():
    # Only diagonal blocks: each 128-row chunk attends to itself alone.
    r = _rng(107)
    q, k, v = r.normal(size=(1, 1, 300, 3)), r.normal(size=(1, 1, 300, 3)), r.normal(size=(1, 1, 300, 3))
    diag = np.eye(3, dtype=np.uint8)[None, None]
    o, lse = oracle.attention_fwd_blocksparse(q, k, v, diag, False, 0.7)
    for c0, c1 in ((0, 128), (128, 256), (256, 300)):
        o_c, l_c = oracle.attention_fwd(q[:, :, c0:c1], k[:, :, c0:c1], v[:, :, c0:c1], False, 0.7)
        np.testing.assert_allclose(o[:, :, c0:c1], o_c, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, c0:c1], l_c, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_equals_masked_softmax(causal):
    r = _rng(109 + causal)
    N = 300
    q, k, v = r.normal(size=(1, 2, N, 3)), r.normal(size=(1, 1, N, 3)), r.normal(size=(1, 1, N, 3))
    bm = (r.random(size=(1, 2, 3, 3)) < 0.5).astype(np.uint8)
    bm[0, 1, 1, :] = 0           # a block row with no keys: rows 128..255 of head 1 see nothing
    bm[0, 0, :, 0] = 1
    o, lse = oracle.attention_fwd_blocksparse(q, k, v, bm, causal, 0.6)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    for h in range(2):
        vis = bm[0, h][i // 128, j // 128].astype(bool)
        if causal:
            vis &= j <= i
        s = np.where(vis, 0.6 * q[0, h] @ k[0, 0].T, -np.inf)
        for t in range(N):
            if not vis[t].any():
                assert np.isneginf(lse[0, h, t]) and np.all(o[0, h, t] == 0)
                continue
            L = scipy.special.logsumexp(s[t])
            assert abs(lse[0, h, t] - L) < 1e-12
            np.testing.assert_allclose(o[0, h, t], np.exp(s[t] - L) @ v[0, 0], rtol=0, atol=1e-12)


def test_blocksparse_gradients_match_central_differences():
    r = _rng(113)
    N = 140
    q, k, v, do = (r.normal(size=(1, 1, N, 2)) for _ in range(4))
    bm = np.array([[[[1, 0], [1, 1]]]], dtype=np.uint8)
    dq, dk, dv = oracle.attention_bwd_blocksparse(q, k, v, do, bm, False, 0.9)
    loss = lambda q_, k_, v_: float((oracle.attention_fwd_blocksparse(q_, k_, v_, bm, False, 0.9)[0] * do).sum())
    eps = 1e-6
    rng = np.random.default_rng(0)
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        # a sample of entries from both block rows and both block columns
        for n in list(rng.integers(0, N, 6)) + [0, 127, 128, N - 1]:
            for c in range(2):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[which][0, 0, n, c] += eps
                args_m[which][0, 0, n, c] -= eps
                num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
                assert abs(g[0, 0, n, c] - num) <= 1e-6 * max(1.0, abs(num)), (which, n, c)


# ---------------------------------------------------------------------------- timing build

def test_native_timing_build_computes_the_same_bits():
    # The -O3 -march=native build that times the oracle as a CPU baseline must be the
    # same computation: no contraction into FMAs and no reassociation, so equal bits.
    r = _rng(404)
    q, k, v, do = (r.normal(size=(1, 4, 70, 16)) for _ in range(4))
    k, v = k[:, :2], v[:, :2]
    want = oracle.attention_fwd(q, k, v, True, 0.3) + oracle.attention_bwd(q, k, v, do, True, 0.3)
    oracle.use_build("native")
    try:
        got = oracle.attention_fwd(q, k, v, True, 0.3) + oracle.attention_bwd(q, k, v, do, True, 0.3)
    finally:
        oracle.use_build("portable")
    for a, b in zip(want, got):
        np.testing.assert_array_equal(a, b)
