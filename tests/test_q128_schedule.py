"""Host model of the 128-query backward's protocol (fa_bwd_q128.cuh).

One CTA per 128-key block walks T steps of 128 query rows.  Tensor memory holds S^T (later
P^T) in one 128-column region and dP^T in another, into which dQ^T is accumulated once the
elementwise warps have read dP^T; the next dP^T waits until the dQ drain has read dQ^T
back.  Shared memory holds two Q stages (each with its LSE row), one dO stage with one
Delta slot, dS^T and one dQ staging tile that two fp32 reduce-adds per step read.

The model runs the loader, the MMA warp, the elementwise warps and the drain as coroutines
under random interleavings, each at its own random speed per run, beside the engines: the
tensor core (in issue order; a commit fires when the work before it is done), TMA loads
landing in any order and the bulk reduces reading the staging tile.  Every wait checks the
mbarrier phase discipline (a parity wait for phase k is only sound while k or k + 1 phases
have completed), and every buffer access checks that it reads the tile it expects and
overwrites only what every reader has finished with.  Variants that drop a wait must fail,
except those the issue order already implies, which are listed as such.
"""
import random

import pytest


class ProtocolError(AssertionError):
    pass


def simulate(T, seed=0, mma_skip_dqempty=False, mma_skip_p=False, loader_skip_qempty=False,
             loader_skip_ds=False, drain_skip_read_wait=False, ew_skip_dsempty=False,
             ew_skip_dofull=False):
    rnd = random.Random(seed)
    done, pending = {}, {}

    def count(b):
        return done.get(b, 0)

    def complete(b):
        done[b] = count(b) + 1

    def arrive(b, needed):
        pending[b] = pending.get(b, 0) + 1
        if pending[b] == needed:
            pending[b] = 0
            complete(b)

    def ready(b, k):
        """Phase k of barrier b (phases counted from 0) has completed."""
        c = count(b)
        if c not in (k, k + 1):
            raise ProtocolError(f"{b}: {c} phases completed while waiting for phase {k}")
        return c == k + 1

    def wait(b, k):
        while not ready(b, k):
            yield

    buf, readers = {}, {}

    def write(name, val):
        if readers.get(name):
            raise ProtocolError(f"{name} overwritten with {val} while {sorted(readers[name])} still read {buf.get(name)}")
        buf[name] = val

    def read_start(name, val, who):
        if buf.get(name) != val:
            raise ProtocolError(f"{who} reads {buf.get(name)} from {name}, expected {val}")
        readers.setdefault(name, set()).add(who)

    def read_end(name, who):
        readers[name].discard(who)

    tc, tma, bulk = [], [], []

    # ------------------------------------------------------------------ loader
    def loader():
        for i in range(T):
            st = i % 2
            if i >= 2 and not loader_skip_qempty:
                yield from wait(("QEmpty", st), i // 2 - 1)
            tma.append(("Q", st, i))
            write(("lse", st), i)
            arrive(("QFull", st), 2)
            yield
            if i >= 1:
                yield from wait("DOEmpty", i - 1)
            tma.append(("dO", 0, i))
            if i >= 1 and not loader_skip_ds:
                yield from wait("DS", i - 1)
            write("delta", i)
            arrive("DOFull", 2)
            yield

    # ------------------------------------------------------------------ MMA warp
    def mma():
        def issue_s(j):
            read_start(("Q", j % 2), ("Q", j), f"S({j})")
            tc.append(("S", j))
            tc.append(("commit", "S"))

        def issue_dp(j):
            read_start("dO", ("dO", j), f"dP({j})")
            tc.append(("dP", j))
            tc.append(("commit", "DP"))

        def issue_dv(j):
            read_start("Scols", ("P", j), f"dV({j})")
            read_start("dO", ("dO", j), f"dV({j})")
            tc.append(("dV", j))

        yield from wait(("QFull", 0), 0)
        yield from wait("DOFull", 0)
        issue_s(0)
        issue_dp(0)
        if not mma_skip_p:
            yield from wait("P", 0)
        issue_dv(0)
        tc.append(("commit", "DOEmpty"))
        if T > 1:
            yield from wait(("QFull", 1), 0)
            issue_s(1)
        for i in range(T):
            st = i % 2
            yield from wait("DS", i)
            read_start("dS", ("dS", i), f"dK({i})")
            read_start(("Q", st), ("Q", i), f"dK({i})")
            tc.append(("dK", i))
            tc.append(("commit", ("QEmpty", st)))
            read_start("dS", ("dS", i), f"dQ({i})")
            tc.append(("dQ", i))
            tc.append(("commit", "DQ"))
            tc.append(("commit", "DSEmpty"))
            if i + 1 < T:
                j = i + 1
                if not mma_skip_p:
                    yield from wait("P", j)
                yield from wait("DOFull", j)
                issue_dv(j)
                if not mma_skip_dqempty:
                    yield from wait("DQEmpty", i)
                issue_dp(j)
                tc.append(("commit", "DOEmpty"))
                if j + 1 < T:
                    yield from wait(("QFull", (j + 1) % 2), (j + 1) // 2)
                    issue_s(j + 1)
            yield

    # ------------------------------------------------------------------ elementwise warps
    def ew():
        for i in range(T):
            st = i % 2
            yield from wait(("QFull", st), i // 2)
            yield from wait("S", i)
            read_start("Scols", ("S", i), f"ew({i})")
            read_start(("lse", st), i, f"ew({i})")
            yield
            read_end("Scols", f"ew({i})")
            read_end(("lse", st), f"ew({i})")
            write("Scols", ("P", i))
            complete("P")
            yield
            if i >= 1 and not ew_skip_dsempty:
                yield from wait("DSEmpty", i - 1)
            if not ew_skip_dofull:
                yield from wait("DOFull", i)
            yield from wait("DP", i)
            read_start("DPcols", ("dP", i), f"ew({i})")
            read_start("delta", i, f"ew({i})")
            yield
            read_end("DPcols", f"ew({i})")
            read_end("delta", f"ew({i})")
            write("dS", ("dS", i))
            complete("DS")
            yield

    # ------------------------------------------------------------------ dQ drain
    def drain():
        for i in range(T):
            yield from wait("DQ", i)
            read_start("DPcols", ("dQ", i), f"drain({i})")
            for half in range(2):
                yield
                if half == 1:
                    read_end("DPcols", f"drain({i})")
                    complete("DQEmpty")
                if not drain_skip_read_wait:
                    while readers.get("stage"):
                        yield
                write("stage", ("dQ", i, half))
                read_start("stage", ("dQ", i, half), "reduce")
                bulk.append(("dQ", i, half))
                yield

    # ------------------------------------------------------------------ engines
    def tensor_core():
        while True:
            if not tc or rnd.random() < 0.3:
                yield
                continue
            kind, x = tc.pop(0)
            if kind == "commit":
                complete(x)
            elif kind == "S":
                write("Scols", ("S", x))
                read_end(("Q", x % 2), f"S({x})")
            elif kind == "dP":
                write("DPcols", ("dP", x))
                read_end("dO", f"dP({x})")
            elif kind == "dV":
                read_end("Scols", f"dV({x})")
                read_end("dO", f"dV({x})")
            elif kind == "dK":
                read_end("dS", f"dK({x})")
                read_end(("Q", x % 2), f"dK({x})")
            elif kind == "dQ":
                write("DPcols", ("dQ", x))
                read_end("dS", f"dQ({x})")
            yield

    def tma_engine():
        while True:
            if not tma or rnd.random() < 0.3:
                yield
                continue
            kind, st, i = tma.pop(rnd.randrange(len(tma)))
            if kind == "Q":
                write(("Q", st), ("Q", i))
                arrive(("QFull", st), 2)
            else:
                write("dO", ("dO", i))
                arrive("DOFull", 2)
            yield

    def bulk_engine():
        while True:
            if not bulk or rnd.random() < 0.3:
                yield
                continue
            bulk.pop(0)
            read_end("stage", "reduce")
            yield

    roles = [loader(), mma(), ew(), drain()]
    engines = [tensor_core(), tma_engine(), bulk_engine()]
    # Each role and engine runs at its own speed in this run (some far slower than the
    # rest), so that orders a fair interleaving would hardly reach are exercised too.
    speed = {id(g): rnd.choice((0.02, 0.2, 1.0)) for g in roles + engines}
    live = list(roles)
    for _ in range(2000000):
        if not live:
            break
        pool = live + engines
        g = rnd.choices(pool, weights=[speed[id(x)] for x in pool])[0]
        try:
            next(g)
        except StopIteration:
            live.remove(g)
    else:
        raise ProtocolError("no progress: a wait never completes")
    for _ in range(50000):
        for g in engines:
            next(g)
    if count("DQEmpty") != T or count("DS") != T or count("P") != T:
        raise ProtocolError("not every step was formed and drained")
    if tc or tma or bulk:
        raise ProtocolError("work left in an engine")


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 12])
def test_q128_protocol_is_race_free(T):
    for seed in range(60):
        simulate(T, seed=seed)


@pytest.mark.parametrize("variant", [
    dict(mma_skip_dqempty=True),      # dP^T(i + 1) written over dQ^T(i) before the drain read it
    dict(mma_skip_p=True),            # dV issued before the warps wrote P^T
    dict(loader_skip_qempty=True),    # Q(i + 2) loaded over Q(i) before dK(i) read it
    dict(loader_skip_ds=True),        # Delta(i + 1) written before dS^T(i) was formed from Delta(i)
    dict(drain_skip_read_wait=True),  # staging tile rewritten before the reduce read it
])
def test_q128_protocol_model_catches_a_dropped_wait(variant):
    with pytest.raises(ProtocolError):
        for seed in range(300):
            simulate(7, seed=seed, **variant)


@pytest.mark.parametrize("variant", [
    dict(ew_skip_dsempty=True),
    dict(ew_skip_dofull=True),
])
def test_q128_protocol_waits_implied_by_the_issue_order(variant):
    """The elementwise warps write dS^T(i) only after dP^T(i), which the MMA warp issues
    after the drain has read dQ^T(i - 1), so dK(i - 1) and dQ^T(i - 1), the readers of
    dS^T(i - 1), are complete; and dP^T(i) itself waited for dO(i)'s barrier, whose phase
    includes the Delta(i) arrival.  The kernel keeps both waits all the same."""
    for seed in range(100):
        simulate(7, seed=seed, **variant)
