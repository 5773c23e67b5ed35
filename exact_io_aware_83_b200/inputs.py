"""Seeded synthetic attention inputs shared by the CUDA path's tests, the benchmark and
the oracle's callers.

This module holds none of the method's arithmetic: it only draws i.i.d. Gaussian
tensors from a CPU ``torch.Generator`` and rounds them to bf16, so the same seed gives
the same bytes on every host.  Draw order is q, k, v, then dO.

Workloads (shapes of the pages' GPT-3 2K / 8K-context training runs and of the
head-dimension-256 and grouped-query variants named on the FlashAttention-2 page):

====================  ==  ===  ===  ====  ===  ======  =========  =====================
name                  B   Hq   Hkv  N     d    causal  passes     q distribution
====================  ==  ===  ===  ====  ===  ======  =========  =====================
tiny_fwd_d64          1   1    1    128   64   no      fwd        N(0,1)
gpt_2k_causal         8   16   16   2048  128  yes     fwd+bwd    N(0,1)
long_8k_causal        2   16   16   8192  128  yes     fwd+bwd    N(0,1)
gqa_4k_causal_fwd     4   32   8    4096  128  yes     fwd        N(0,1)
d256_4k_stress        2   8    8    4096  256  no      fwd+bwd    N(0,4^2)
window_8k_1k          2   16   16   8192  128  band    fwd+bwd    N(0,1)
dropout_8k_causal     2   16   16   8192  128  yes     fwd+bwd    N(0,1)
blocksparse_8k_causal 2   16   16   8192  128  yes     fwd+bwd    N(0,1)
====================  ==  ===  ===  ====  ===  ======  =========  =====================

window_8k_1k is local attention with the band i - 1023 <= j <= i (1024 keys per row,
the row's own included); dropout_8k_causal is long_8k_causal with attention dropout
p = 0.1 (Philox4x32-10 mask, seed 8080); blocksparse_8k_causal is long_8k_causal with a
block mask enabling each 128 x 128 block with probability 1/4 and every diagonal block
(mask seed 1010), causal on top.

Packed variable-length workload: varlen_32k_ragged, 24 sequences of long-tailed length
(log-normal around 1500 tokens, clipped to [16, 8192]; 39.7k tokens in all, longest 3867), 16 heads,
d = 128, causal, forward and backward.

Decode workloads (a few new query rows against a key/value cache; K/V N(0,1)):

=================  ==  ===  ===  ==  ======  ===
name               B   Hq   Hkv  Nq  Nk      d
=================  ==  ===  ===  ==  ======  ===
decode_64k_gqa     4   32   8    1   65536   128
decode_8k_batch    64  32   8    1   8192    128
=================  ==  ===  ===  ==  ======  ===
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    backward: bool
    q_std: float
    seed: int
    window: tuple | None = None   # (left, right) key band, -1 = unlimited; None: causal flag
    dropout_p: float = 0.0        # attention dropout probability (0: none)
    dropout_seed: int = 0
    block_density: float = 0.0    # block-sparse: share of enabled 128 x 128 blocks (0: dense)
    mask_seed: int = 0

    def block_mask(self):
        """The block-sparse workload's mask (None for dense workloads)."""
        if not self.block_density:
            return None
        return draw_block_mask(self.B, self.Hq, self.N, self.block_density, self.mask_seed,
                               diagonal=True)

    @property
    def scale(self) -> float:
        # The caller passes the softmax scale as fp32; 1/sqrt(128) is not exact in fp32,
        # so every consumer uses the fp32-rounded value.
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32).item())

    def fwd_flops(self) -> float:
        """4 B Hq N^2 d, halved when causal (the metric's convention); with a key band or
        a block mask, 4 d times the number of visible (query, key) pairs."""
        if self.block_density:
            return 4.0 * blocksparse_pairs(self.block_mask(), self.N, self.causal) * self.d
        if self.window is not None:
            left, right = self.window
            pairs = 0
            for i in range(self.N):
                lo = 0 if left < 0 else max(0, i - left)
                hi = self.N - 1 if right < 0 else min(self.N - 1, i + right)
                pairs += hi - lo + 1
            return 4.0 * self.B * self.Hq * pairs * self.d
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """2.5 x the forward count."""
        return 2.5 * self.fwd_flops()

    def score_pairs(self) -> float:
        """(query, key) pairs whose score is visible, i.e. exponentials per pass (the
        forward evaluates one per pair, the backward recomputes each once)."""
        if self.block_density or self.window is not None:
            return self.fwd_flops() / (4.0 * self.d)
        per_head = self.N * (self.N + 1) / 2 if self.causal else float(self.N) * self.N
        return self.B * self.Hq * per_head


WORKLOADS = {
    w.name: w
    for w in (
        Workload("tiny_fwd_d64", 1, 1, 1, 128, 64, False, False, 1.0, 1),
        Workload("gpt_2k_causal", 8, 16, 16, 2048, 128, True, True, 1.0, 2),
        Workload("long_8k_causal", 2, 16, 16, 8192, 128, True, True, 1.0, 3),
        Workload("gqa_4k_causal_fwd", 4, 32, 8, 4096, 128, True, False, 1.0, 4),
        Workload("d256_4k_stress", 2, 8, 8, 4096, 256, False, True, 4.0, 5),
        Workload("window_8k_1k", 2, 16, 16, 8192, 128, False, True, 1.0, 6, (1023, 0)),
        Workload("dropout_8k_causal", 2, 16, 16, 8192, 128, True, True, 1.0, 9, None, 0.1, 8080),
        Workload("blocksparse_8k_causal", 2, 16, 16, 8192, 128, True, True, 1.0, 10,
                 block_density=0.25, mask_seed=1010),
    )
}


@dataclass(frozen=True)
class VarlenWorkload:
    name: str
    n_seqs: int
    mean_len: int
    H: int
    d: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32).item())

    def lens(self):
        return packed_lengths(self.n_seqs, self.mean_len, self.seed)

    def fwd_flops(self) -> float:
        """4 H d per visible (query, key) pair of every sequence."""
        pairs = sum(L * (L + 1) // 2 if self.causal else L * L for L in self.lens())
        return 4.0 * self.H * self.d * pairs

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()


VARLEN_WORKLOADS = {
    w.name: w
    for w in (VarlenWorkload("varlen_32k_ragged", 24, 1500, 16, 128, True, 31),)
}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32).item())

    def cache_bytes(self) -> int:
        """K and V of every cached row: what a decode step must read from HBM."""
        return 2 * self.B * self.Hkv * self.Nk * self.d * 2

    def io_bytes(self) -> int:
        """Algorithmic bytes of one step: read the cache and Q, write O (bf16) and LSE."""
        rows = self.B * self.Hq * self.Nq
        return self.cache_bytes() + 2 * rows * self.d * 2 + rows * 4


DECODE_WORKLOADS = {
    w.name: w
    for w in (
        DecodeWorkload("decode_64k_gqa", 4, 32, 8, 1, 65536, 128, True, 7),
        DecodeWorkload("decode_8k_batch", 64, 32, 8, 1, 8192, 128, True, 8),
    )
}


def draw(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int, q_std: float = 1.0,
         with_dout: bool = True):
    """Return bf16 CPU tensors (q, k, v[, dout]) in ``[B, H, N, d]`` layout."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q = q * q_std
    k = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32)
    out = [q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)]
    if with_dout:
        do = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
        out.append(do.to(torch.bfloat16))
    return tuple(out)


def draw_workload(w: Workload, with_dout: bool | None = None):
    """Inputs of a named workload (dO drawn when the workload has a backward pass)."""
    if with_dout is None:
        with_dout = w.backward
    return draw(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, w.q_std, with_dout)


def draw_decode(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, seed: int,
                q_std: float = 1.0):
    """Return bf16 CPU tensors (q [B, Hq, Nq, d], k_cache, v_cache [B, Hkv, Nk, d]):
    a few new query rows against a longer key/value cache, all N(0, 1) (q scaled by
    q_std)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q = q * q_std
    k = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def draw_packed(lens_q, lens_k, Hq: int, Hkv: int, d: int, seed: int, q_std: float = 1.0):
    """Packed variable-length sequences: bf16 CPU tensors q [total_q, Hq, d], k, v
    [total_k, Hkv, d], dout like q, and int32 offsets cu_q, cu_k [B + 1] (starting at 0)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    cu_q = torch.tensor([0] + list(lens_q), dtype=torch.int64).cumsum(0).to(torch.int32)
    cu_k = torch.tensor([0] + list(lens_k), dtype=torch.int64).cumsum(0).to(torch.int32)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = torch.randn((tq, Hq, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q = q * q_std
    k = torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32)
    do = torch.randn((tq, Hq, d), generator=g, dtype=torch.float32)
    bf = lambda t: t.to(torch.bfloat16)
    return bf(q), bf(k), bf(v), bf(do), cu_q, cu_k


def packed_lengths(n: int, mean: int, seed: int, lo: int = 16, hi: int = 8192):
    """n sequence lengths with a long-tailed (log-normal) mix around `mean`, clipped to
    [lo, hi]: the ragged batches that packing serves."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(n, generator=g, dtype=torch.float64) * 0.8
    lens = (torch.exp(x) * mean / math.exp(0.32)).round().clamp(lo, hi).to(torch.int64)
    return [int(v) for v in lens]


def draw_block_mask(B: int, Hq: int, N: int, density: float, seed: int, diagonal: bool = False):
    """uint8 CPU tensor [B, Hq, nb, nb], nb = ceil(N / 128): each 128 x 128 block enabled
    independently with probability `density` (the diagonal blocks always, with
    `diagonal`)."""
    nb = (N + 127) // 128
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    m = (torch.rand((B, Hq, nb, nb), generator=g, dtype=torch.float64) < density).to(torch.uint8)
    if diagonal:
        m[:, :, range(nb), range(nb)] = 1
    return m


def blocksparse_pairs(mask, N: int, causal: bool) -> int:
    """Visible (query, key) pairs of a block mask [B, Hq, nb, nb]: a counting helper for
    FLOP totals (every pair of an enabled block, j <= i only with causal)."""
    nb = mask.shape[-1]
    rows = torch.tensor([min(128, N - 128 * b) for b in range(nb)], dtype=torch.float64)
    full = rows[:, None] * rows[None, :]                  # pairs of block (qb, kb)
    if causal:
        full = torch.tril(full, -1)
        full += torch.diag(rows * (rows + 1) / 2)
    return int((mask.to(torch.float64) * full).sum().item())
