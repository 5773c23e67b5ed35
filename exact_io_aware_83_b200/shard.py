"""Host-side sharding for multi-GPU runs.

Attention over different (batch element, K/V-head group) pairs shares nothing, so a
multi-GPU job splits the batch across ranks and runs the unchanged single-GPU kernels on
each shard: no collective is needed on the data path.  With a fixed per-rank batch the
job scales weakly: rank r owns global batch rows [r * B_local, (r + 1) * B_local).
"""
from __future__ import annotations


def shard_batch(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """Half-open range of global batch rows owned by `rank` (contiguous, balanced)."""
    if world < 1 or not 0 <= rank < world or global_batch < world:
        raise ValueError("need global_batch >= world >= 1 and 0 <= rank < world")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's shard, so ranks draw different synthetic batches."""
    return int(seed) + 1000 * int(rank)


def max_over_ranks(value: float, group=None) -> float:
    """Largest `value` over all ranks of the default process group (identity if none)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
