"""fa_bwd_noalloc: the backward pass for callers that may not allocate device memory.

Some callers cannot call cudaMalloc (or a caching allocator) where they run the backward
pass - code under a fixed, pre-reserved memory budget, latency-critical paths where an
allocation might block or fail, hooks that must not touch the framework's allocator.
fa_bwd_noalloc takes no workspace; its scratch is a static device buffer inside the
library.  These tests call it through the C ABI, twice in a row, and compare every
gradient with the ordinary fa_bwd given a caller-allocated workspace, within the parity
tolerance (relative Frobenius error <= 2e-2).  This file is collected last so that a run
stopping at the first failure has already run every other test; it also passes on its
own in a fresh process, where its first call performs the one-time buffer lookup.
"""
import math

import numpy as np
import pytest
import torch

from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw

pytestmark = pytest.mark.gpu

GRAD_TOL = 2e-2


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def _grads_with_workspace(q, k, v, o, lse, do, causal, scale):
    return fa.bwd(q, k, v, o, lse, do, causal=causal, scale=scale)


def _grads_noalloc(q, k, v, o, lse, do, causal, scale):
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream().cuda_stream
    fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                      do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                      B, Hq, Hkv, N, d, causal, scale, stream)
    return dq, dk, dv


@pytest.mark.parametrize("shape,causal", [((2, 4, 2, 384, 128), True),
                                          ((1, 2, 2, 300, 64), False)])
def test_noalloc_matches_workspace_entry_point_twice(shape, causal):
    B, Hq, Hkv, N, d = shape
    scale = 1.0 / math.sqrt(d)
    for call, seed in enumerate((41, 42)):  # two calls in a row, different inputs
        q, k, v, do = (t.cuda() for t in draw(B, Hq, Hkv, N, d, seed=seed + d))
        o, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
        ref = _grads_with_workspace(q, k, v, o, lse, do, causal, scale)
        got = _grads_noalloc(q, k, v, o, lse, do, causal, scale)
        torch.cuda.synchronize()
        assert fa.fa_device_status(None) == fa.FA_OK
        for name, x, r in zip(("dQ", "dK", "dV"), got, ref):
            assert torch.isfinite(x.float()).all(), (call, name)
            err = _rel(x, r)
            assert err <= GRAD_TOL, f"call {call}: {name} differs from fa_bwd by {err}"


def test_noalloc_rejects_problems_beyond_the_static_buffer():
    # d = 128: 4 B per Delta row + 512 B per dQ row; 2 x 16 x 8192 rows need ~135 MB.
    assert fa.fa_bwd_workspace_bytes(2, 16, 16, 8192, 128) > fa.FA_NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError) as err:
        fa.fa_bwd_noalloc(*([x.data_ptr()] * 9), 2, 16, 16, 8192, 128, True, 0.088, None)
    assert err.value.code == fa.FA_ERR_SCRATCH_LIMIT
