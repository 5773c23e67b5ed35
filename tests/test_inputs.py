"""Host checks of the seeded input generators and of the pair counts behind the FLOP
totals that the benchmark reports (brute force over every (query, key) pair)."""
import numpy as np
import pytest
import torch

from exact_io_aware_83_b200.inputs import (WORKLOADS, Workload, blocksparse_pairs,
                                           draw_block_mask)


def _visible(mask_bh, N, causal):
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    vis = mask_bh[i // 128, j // 128] != 0
    return vis & (j <= i) if causal else vis


@pytest.mark.parametrize("N", [1, 127, 128, 300, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_pairs_brute_force(N, causal):
    m = draw_block_mask(2, 3, N, 0.5, seed=N)
    want = sum(int(_visible(m[b, h].numpy(), N, causal).sum()) for b in range(2) for h in range(3))
    assert blocksparse_pairs(m, N, causal) == want


def test_block_mask_is_seeded_and_keeps_the_diagonal():
    a = draw_block_mask(1, 4, 1000, 0.1, seed=5, diagonal=True)
    b = draw_block_mask(1, 4, 1000, 0.1, seed=5, diagonal=True)
    assert a.dtype == torch.uint8 and tuple(a.shape) == (1, 4, 8, 8)
    assert torch.equal(a, b)
    assert torch.all(a[:, :, range(8), range(8)] == 1)
    assert not torch.equal(a, draw_block_mask(1, 4, 1000, 0.1, seed=6, diagonal=True))


def test_window_flops_brute_force():
    w = Workload("t", 1, 2, 2, 300, 64, False, True, 1.0, 0, (37, 5))
    i = np.arange(300)[:, None]
    j = np.arange(300)[None, :]
    pairs = int(((j >= i - 37) & (j <= i + 5)).sum())
    assert w.fwd_flops() == 4.0 * 2 * pairs * 64


def test_blocksparse_workload_flops():
    w = WORKLOADS["blocksparse_8k_causal"]
    m = w.block_mask()
    assert tuple(m.shape) == (2, 16, 64, 64)
    assert w.fwd_flops() == 4.0 * blocksparse_pairs(m, w.N, True) * w.d
    dense = WORKLOADS["long_8k_causal"].fwd_flops()
    assert 0.2 * dense < w.fwd_flops() < 0.35 * dense
