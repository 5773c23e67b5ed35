"""Host-side sharding for multi-GPU runs.

Attention over different (batch element, K/V-head group) pairs shares nothing (the
FlashAttention-2 page, "Better Parallelism", parallelises over batch and heads), so a
multi-GPU job splits those pairs across ranks and runs the unchanged single-GPU kernels on
each rank's share: no collective is needed on the data path.  A K/V head and the Hq / Hkv
query heads that read it (a GQA group) always stay on one rank, so dK and dV are summed
over the group inside one kernel as in the single-GPU case.

Two splits are offered:
  shard_batch  - whole batch rows per rank (weak scaling: each rank owns its own batch);
  shard_groups - the B * Hkv (batch row, K/V head) groups in b-major order cut into
                 `world` contiguous, balanced ranges, so that one problem with few batch
                 rows (B = 2 at 8K context) still spreads over up to B * Hkv ranks.
A rank's range of groups is returned as segments, each a contiguous slice of the
[B, H, N, d] tensors: either part of one batch row's heads or whole batch rows.
"""
from __future__ import annotations

from typing import NamedTuple


def shard_batch(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """Half-open range of global batch rows owned by `rank` (contiguous, balanced)."""
    if world < 1 or not 0 <= rank < world or global_batch < world:
        raise ValueError("need global_batch >= world >= 1 and 0 <= rank < world")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class Segment(NamedTuple):
    """Batch rows [b_lo, b_hi) x K/V heads [kv_lo, kv_hi): one contiguous slice of the
    [B, H, N, d] tensors (b_hi = b_lo + 1, or the K/V-head range is every head)."""
    b_lo: int
    b_hi: int
    kv_lo: int
    kv_hi: int

    def groups(self) -> list[tuple[int, int]]:
        return [(b, kv) for b in range(self.b_lo, self.b_hi) for kv in range(self.kv_lo, self.kv_hi)]


def shard_groups(B: int, Hkv: int, world: int, rank: int) -> list[Segment]:
    """Segments of the (batch row, K/V head) groups owned by `rank`: the B * Hkv groups in
    b-major order are cut into `world` contiguous ranges whose sizes differ by at most one;
    a range is returned as at most three segments (the tail of one batch row, whole rows,
    the head of another row)."""
    total = B * Hkv
    if B < 1 or Hkv < 1 or world < 1 or not 0 <= rank < world or total < world:
        raise ValueError("need B * Hkv >= world >= 1 and 0 <= rank < world")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    segs: list[Segment] = []
    u = start
    while u < stop:
        b, kv = divmod(u, Hkv)
        if kv == 0 and stop - u >= Hkv:  # whole batch rows
            nb = (stop - u) // Hkv
            segs.append(Segment(b, b + nb, 0, Hkv))
            u += nb * Hkv
        else:
            hi = min(Hkv, kv + (stop - u))
            segs.append(Segment(b, b + 1, kv, hi))
            u += hi - kv
    return segs


def segment_slices(seg: Segment, g: int):
    """(query-head slice, K/V-head slice, batch slice) of a segment, for tensors laid out
    [B, H, N, d] (query heads kv * g .. kv * g + g - 1 read K/V head kv)."""
    return (slice(seg.kv_lo * g, seg.kv_hi * g), slice(seg.kv_lo, seg.kv_hi), slice(seg.b_lo, seg.b_hi))


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
