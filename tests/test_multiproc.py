"""Host-side multi-process logic of multi-GPU runs, on CPU with the gloo backend:
batch sharding and (batch row, K/V head) group sharding (disjoint, complete, balanced,
GQA groups whole), per-rank attention over a rank's segments reassembled into the whole
problem, and the max-over-ranks timing reduction."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_83_b200.shard import (Segment, max_over_ranks, rank_seed, segment_slices,
                                          shard_batch, shard_groups)


def test_shard_batch_covers_each_row_once():
    for world in (1, 2, 3, 4, 8):
        for gb in range(world, 3 * world + 5):
            ranges = [shard_batch(gb, world, r) for r in range(world)]
            rows = [i for a, b in ranges for i in range(a, b)]
            assert rows == list(range(gb))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1


def test_shard_batch_rejects_bad_arguments():
    with pytest.raises(ValueError):
        shard_batch(1, 2, 0)
    with pytest.raises(ValueError):
        shard_batch(4, 2, 2)


@pytest.mark.parametrize("B,Hkv", [(1, 1), (2, 16), (4, 8), (3, 5), (1, 7), (8, 16)])
def test_shard_groups_cover_each_group_once(B, Hkv):
    for world in range(1, min(B * Hkv, 12) + 1):
        owned = []
        sizes = []
        for r in range(world):
            segs = shard_groups(B, Hkv, world, r)
            assert 1 <= len(segs) <= 3
            mine = [gp for s in segs for gp in s.groups()]
            for s in segs:  # each segment is one contiguous [B, H, N, d] slice
                assert s.b_hi == s.b_lo + 1 or (s.kv_lo, s.kv_hi) == (0, Hkv)
                assert 0 <= s.kv_lo < s.kv_hi <= Hkv and 0 <= s.b_lo < s.b_hi <= B
            owned += mine
            sizes.append(len(mine))
        assert owned == [(b, kv) for b in range(B) for kv in range(Hkv)]  # disjoint, complete, in order
        assert max(sizes) - min(sizes) <= 1


def test_long_context_workload_spreads_over_eight_ranks():
    # B = 2, Hkv = 16 (8K context): batch sharding stops at 2 ranks, group sharding gives
    # each of 8 ranks 4 whole K/V heads.
    for r in range(8):
        assert shard_groups(2, 16, 8, r) == [Segment(r // 4, r // 4 + 1, 4 * (r % 4), 4 * (r % 4) + 4)]
    with pytest.raises(ValueError):
        shard_groups(2, 16, 33, 0)


def test_segment_slices_keep_gqa_groups_whole():
    q_heads, kv_heads, b = segment_slices(Segment(1, 2, 3, 5), g=4)
    assert (q_heads.start, q_heads.stop) == (12, 20)
    assert (kv_heads.start, kv_heads.stop) == (3, 5)
    assert (b.start, b.stop) == (1, 2)
    x = torch.zeros(2, 32, 8, 4)
    assert x[b, q_heads].is_contiguous()  # a kernel can take the slice as it is


def test_rank_seeds_differ():
    assert len({rank_seed(5, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# the whole problem of the two-rank test: B = 2, Hq = 6, Hkv = 3 (g = 2), N = 24, d = 8
_SHAPE = (2, 6, 3, 24, 8)


def _problem():
    r = np.random.default_rng(606)
    B, Hq, Hkv, N, d = _SHAPE
    q = r.normal(size=(B, Hq, N, d))
    k = r.normal(size=(B, Hkv, N, d))
    v = r.normal(size=(B, Hkv, N, d))
    do = r.normal(size=(B, Hq, N, d))
    return q, k, v, do


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Each rank reports its own elapsed time; every rank must receive the slowest.
        got = max_over_ranks(10.0 + rank)
        a, b = shard_batch(8 * world, world, rank)
        # Attention over this rank's groups only (the fp64 oracle stands in for the GPU
        # kernels), written into a zeroed copy of the whole outputs; a sum over ranks then
        # reassembles the full result, since every group belongs to exactly one rank.
        import oracle
        oracle.set_threads(1)
        q, k, v, do = _problem()
        B, Hq, Hkv, N, d = _SHAPE
        g = Hq // Hkv
        o = np.zeros_like(q)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        for seg in shard_groups(B, Hkv, world, rank):
            qh, kh, bs = segment_slices(seg, g)
            o[bs, qh] = oracle.attention_fwd(q[bs, qh], k[bs, kh], v[bs, kh], True, 0.4)[0]
            gq, gk, gv, _, _ = oracle.attention_bwd(q[bs, qh], k[bs, kh], v[bs, kh], do[bs, qh], True, 0.4)
            dq[bs, qh], dk[bs, kh], dv[bs, kh] = gq, gk, gv
        flat = torch.from_numpy(np.concatenate([x.ravel() for x in (o, dq, dk, dv)]))
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)
        out.put((rank, got, a, b, flat.numpy() if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_two_rank_group_shards_reassemble_the_whole_problem():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    # Both ranks must use the same port: pick it once.
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]
    assert [(r[2], r[3]) for r in res] == [(0, 8), (8, 16)]
    assert max_over_ranks(3.5) == 3.5  # no process group: identity
    import oracle
    qq, kk, vv, dd = _problem()
    o = oracle.attention_fwd(qq, kk, vv, True, 0.4)[0]
    grads = oracle.attention_bwd(qq, kk, vv, dd, True, 0.4)[:3]
    want = np.concatenate([x.ravel() for x in (o, *grads)])
    np.testing.assert_array_equal(res[0][4], want)  # each group computed once, on one rank
