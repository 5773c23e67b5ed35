"""fa_bwd_noalloc: the backward pass for callers that may not allocate device memory.

Some callers cannot call cudaMalloc (or a caching allocator) where they run the backward
pass - code under a fixed, pre-reserved memory budget, latency-critical paths where an
allocation might block or fail, hooks that must not touch the framework's allocator.
fa_bwd_noalloc takes no workspace; its scratch is a static device buffer inside the
library, shared by every call and holding whatever the previous call left there.

These tests call it through the C ABI and compare it with the ordinary fa_bwd given a
caller-allocated workspace.  Both run the same kernels, so dK and dV must be bit-equal;
dQ is accumulated with fp32 reduce-adds whose order varies from run to run, so it must
agree to 1e-3 relative (Frobenius).  The inputs of consecutive calls differ, and one case
runs a larger problem first so that the smaller one starts on stale scratch contents.
One case is also held to the oracle at the parity tolerance.

This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes on its own in a fresh process, where its first call
performs the one-time buffer lookup.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2    # relative Frobenius error against the oracle
DQ_RUN_TOL = 1e-3  # dQ between two runs of the same kernels (fp32 reduce order)


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def _grads_noalloc(q, k, v, o, lse, do, causal, scale):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream().cuda_stream
    fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                      B, Hq, Hkv, N, d, causal, scale, stream)
    return dq, dk, dv


def _compare(shape, causal, seed):
    """One no-alloc call against fa_bwd on fresh inputs; returns the inputs and results."""
    B, Hq, Hkv, N, d = shape
    scale = 1.0 / math.sqrt(d)
    host = draw(B, Hq, Hkv, N, d, seed=seed)
    q, k, v, do = (t.cuda() for t in host)
    o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    ref = fa.bwd(q, k, v, o, lse, do, causal=causal, scale=scale)
    got = _grads_noalloc(q, k, v, o, lse, do, causal, scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    for name, x in zip(("dQ", "dK", "dV"), got):
        assert torch.isfinite(x.float()).all(), name
    assert torch.equal(got[1], ref[1]), "dK differs from fa_bwd"
    assert torch.equal(got[2], ref[2]), "dV differs from fa_bwd"
    err = _rel(got[0], ref[0])
    assert err <= DQ_RUN_TOL, f"dQ differs from fa_bwd by {err}"
    return host, got, scale


@pytest.mark.parametrize("shape,causal", [((2, 4, 2, 384, 128), True),
                                          ((1, 2, 2, 300, 64), False),
                                          ((1, 2, 1, 200, 256), True)])
def test_noalloc_matches_workspace_entry_point_twice(shape, causal):
    for seed in (41, 42):  # two calls in a row, different inputs
        _compare(shape, causal, seed + shape[-1])


def test_noalloc_after_a_larger_problem_left_the_scratch_dirty():
    # The larger call fills more of the shared buffer (Delta and the dQ accumulator of
    # 2 x 8 x 1024 rows); the smaller one that follows reuses its start.
    _compare((2, 8, 4, 1024, 128), True, 7)
    _compare((1, 3, 1, 257, 128), True, 8)


def test_noalloc_matches_the_oracle():
    host, got, scale = _compare((1, 4, 2, 333, 128), True, 9)
    q, k, v, do = (t.float().double().numpy() for t in host)
    refs = oracle.attention_bwd(q, k, v, do, True, scale)[:3]
    for name, x, r in zip(("dQ", "dK", "dV"), got, refs):
        err = float(np.linalg.norm(x.double().cpu().numpy() - r) / np.linalg.norm(r))
        assert err <= GRAD_TOL, f"{name}: relative Frobenius error {err}"


def test_noalloc_rejects_problems_beyond_the_static_buffer():
    # d = 128: 4 B per Delta row + 512 B per dQ row; 2 x 16 x 8192 rows need ~135 MB.
    assert fa.fa_bwd_workspace_bytes(2, 16, 16, 8192, 128) > fa.FA_NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as err:
        fa.fa_bwd_noalloc(*([x.data_ptr()] * 9), 2, 16, 16, 8192, 128, True, 0.088, None)
    assert err.value.code == fa.FA_ERR_SCRATCH_LIMIT
