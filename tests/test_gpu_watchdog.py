"""Device-side failure detection without a GPU fault: a bounded pipeline wait that can
never complete (nothing arrives at its barrier) must expire, report
FA_ERR_DEVICE_TIMEOUT through the status word, and leave the context usable."""
import math
import time

import pytest
import torch

from exact_io_aware_83_b200 import fa
from exact_io_aware_83_b200.inputs import draw

pytestmark = pytest.mark.gpu


def test_expired_wait_sets_status_and_context_survives():
    assert fa.fa_device_status(None) == fa.FA_OK
    t0 = time.time()
    fa.fa_watchdog_selftest(20000)  # 20 ms limit
    assert fa.fa_device_status(None) == fa.FA_ERR_DEVICE_TIMEOUT
    assert time.time() - t0 < 10.0
    assert fa.fa_device_status(None) == fa.FA_OK  # reading clears the word
    # The context still runs attention correctly afterwards.
    q, k, v = (t.cuda() for t in draw(1, 2, 1, 200, 128, seed=3, with_dout=False))
    o, lse = fa.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None) == fa.FA_OK
    assert torch.isfinite(o.float()).all()


def test_selftest_rejects_bad_limits():
    for bad in (0, -5, 10 ** 8):
        with pytest.raises(fa.FAError):
            fa.fa_watchdog_selftest(bad)
