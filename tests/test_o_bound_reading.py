"""Why the O bound leaves 1e-2 for |O| >= 2: a constructed two-key row (CPU, no GPU).

The tensor core takes the probabilities of P V as bf16 when V is bf16, so every kernel of
this kind rounds each probability to 8 significant bits before the product.  This test
builds one row where even the most favourable such computation - the exact row maximum
as exponent offset (so the largest probability, 1, is exact), the exact sum of the rounded
weights as normaliser, and a correctly rounded bf16 output - misses the exact O by more
than 1e-2, with |O| in [2, 4) and |v| <= 4.  It also checks that the derived bound of the
parity tests (1e-2 below |O| = 2, from 2 up the larger of 1e-2 and half a bf16 spacing
plus the probability-rounding allowance) covers that computation.

Row: scores (0, c) with c = 0.6015625 * (-1.1328125) (bf16 operands, exact product), so
the second probability exp(c) = 0.50588 rounds to bf16 with relative error 0.0038 (close
to the worst, 2^-8); values (-3.96875, 1.34375) put O at -2.184.
"""
import math

import numpy as np
import torch

import oracle
from test_gpu_parity import O_TOL, causal_visible, o_tolerance, p_allowance

A, B = 0.6015625, -1.1328125      # q[0] and k_1[0]; the score of key 0 is 0
V0, V1 = -3.96875, 1.34375       # the two keys' values in column 0


def two_key_row(d=64):
    """q [1,1,2,d], k, v [1,1,2,d] (bf16-exact values): two identical query rows against two
    keys with scores (0, A*B) at scale 1, values (V0, V1) in column 0."""
    q = np.zeros((1, 1, 2, d))
    q[0, 0, :, 0] = A
    k = np.zeros((1, 1, 2, d))
    k[0, 0, 1, 0] = B
    v = np.zeros((1, 1, 2, d))
    v[0, 0, :, 0] = (V0, V1)
    v[0, 0, :, 1] = (0.5, -0.25)  # a second, harmless column
    return q, k, v


def _bf16(x):
    return torch.tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def test_inputs_are_bf16_exact():
    q, k, v = two_key_row()
    for t in (q, k, v):
        np.testing.assert_array_equal(_bf16(t), t)


def test_ideal_bf16_probability_kernel_misses_1e2_and_the_derived_bound_covers_it():
    q, k, v = two_key_row()
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, False, 1.0)
    s = np.array([0.0, A * B])
    p = np.exp(s - s.max())                  # exact offset: the largest probability is 1
    pt = _bf16(p)                            # what the tensor core multiplies
    o_pre = (pt @ v[0, 0, :, 0]) / pt.sum()  # exact normaliser of the rounded weights
    o_ideal = float(_bf16(o_pre))            # correctly rounded bf16 output
    err = abs(o_ideal - o_ref[0, 0, 0, 0])
    assert 2.0 <= abs(o_ref[0, 0, 0, 0]) < 4.0
    assert abs(pt[1] - p[1]) / p[1] > 2.0 ** -9   # more than the top-of-binade bound
    assert err > O_TOL, f"the ideal computation's error {err} should exceed 1e-2"
    tol = o_tolerance(o_ref, p_allowance(q, k, v, o_ref, lse_ref, 1.0, causal_visible(2, False)))
    assert err <= tol[0, 0, 0, 0], f"derived bound {tol[0, 0, 0, 0]} does not cover {err}"
    # and below |O| = 2 the bound stays 1e-2
    assert tol[0, 0, 0, 1] == O_TOL
