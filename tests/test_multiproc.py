"""Host-side multi-process logic of multi-GPU runs, on CPU with the gloo backend:
batch sharding (disjoint, complete, balanced) and the max-over-ranks timing reduction."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_io_aware_83_b200.shard import max_over_ranks, rank_seed, shard_batch


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


def test_rank_seeds_differ():
    assert len({rank_seed(5, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Each rank reports its own elapsed time; every rank must receive the slowest.
        got = max_over_ranks(10.0 + rank)
        a, b = shard_batch(8 * world, world, rank)
        out.put((rank, got, a, b))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_shards():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    # Both ranks must use the same port: pick it once.
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]
    assert [(r[2], r[3]) for r in res] == [(0, 8), (8, 16)]
    assert max_over_ranks(3.5) == 3.5  # no process group: identity
