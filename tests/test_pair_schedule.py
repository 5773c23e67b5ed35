"""Host model of the d = 256 pair backward's protocol (fa_bwd_pair.cuh): two CTAs of a
cluster exchanging P^T and dS^T tiles every 64-row step.

Rank 0 forms S^T and P^T and sends P^T; it consumes dS^T for dK[:, :128] and dQ^T.  Rank 1
forms dP^T and dS^T from the received P^T, keeps dS^T as its own dK operand and sends it.
The model runs, as coroutines under random interleavings, each rank's loader, MMA warp,
elementwise warps and (rank 0) dQ drain, plus the asynchronous engines: one tensor core
per rank (in issue order, commits fire when the work before them is done), TMA loads
landing in any order, and bulk copies between the CTAs landing in any order.  Every wait
checks the mbarrier phase discipline (a parity wait for phase k is only sound while k or
k + 1 phases have completed), and every buffer access checks that it reads the tile it
expects and overwrites only what every reader has finished with: the Q / dO ring stages,
the S^T and dP^T tensor-memory buffers, rank 0's dQ^T buffers, the receive buffers (X) and
the send buffers (Y, which a copy reads and rank 1's dK also reads).  Variants that drop a
wait or move a release earlier must fail.
"""
import random

import pytest


class ProtocolError(AssertionError):
    pass


def simulate(T, seed=0, r0_skip_xfree=False, r1_skip_dsempty=False, r1_skip_xfree=False,
             r0_release_x_after_dk=False, r1_skip_ds=False, r0_skip_sfree=False, r0_skip_dqempty=False):
    rnd = random.Random(seed)
    done = {}

    def count(b):
        return done.get(b, 0)

    def complete(b):
        done[b] = count(b) + 1

    def ready(b, k):
        """Phase k of barrier b (phases counted from 0) has completed."""
        c = count(b)
        if c not in (k, k + 1):
            raise ProtocolError(f"{b}: {c} phases completed while waiting for phase {k}")
        return c == k + 1

    pending = {}

    def arrive(b, needed):
        pending[b] = pending.get(b, 0) + 1
        if pending[b] == needed:
            pending[b] = 0
            complete(b)

    # buffers: current tile and the set of readers that have not finished with it
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

    tc = {0: [], 1: []}      # per-rank tensor-core queues
    tma = []                 # (rank, stage, step)
    copies = []              # (src_rank, xb, step)

    def wait(b, k):
        while not ready(b, k):
            yield

    # ------------------------------------------------------------------ rank 0
    def loader0():
        for i in range(T):
            st = i % 2
            if i >= 2:
                yield from wait(("R0", "RingEmpty", st), i // 2 - 1)
            tma.append((0, st, i))
            yield

    def mma0():
        def issue_s(i):
            read_start(("R0", "stage", i % 2), ("Q", i), f"S^T({i})")
            tc[0].append(("S", i))
            tc[0].append(("commit", ("R0", "Score", i % 2)))

        for s in range(min(2, T)):
            yield from wait(("R0", "RingFull", s), 0)
            issue_s(s)
        for i in range(T):
            xb = st = i % 2
            yield from wait(("R0", "XFull", xb), i // 2)
            read_start(("R0", "X", xb), ("dS", i), f"dK0({i})")
            read_start(("R0", "X", xb), ("dS", i), f"dQ({i})")
            read_start(("R0", "stage", st), ("Q", i), f"dK0({i})")
            tc[0].append(("dK0", i))
            if r0_release_x_after_dk:
                tc[0].append(("commit", ("R1", "XFree", xb)))
            tc[0].append(("commit", ("R0", "RingEmpty", st)))
            if i >= 2 and not r0_skip_dqempty:
                yield from wait(("R0", "DQEmpty", xb), i // 2 - 1)
            tc[0].append(("dQ", i))
            tc[0].append(("commit", ("R0", "DQFull", xb)))
            if not r0_release_x_after_dk:
                tc[0].append(("commit", ("R1", "XFree", xb)))   # multicast onto rank 1
            if i + 2 < T:
                if not r0_skip_sfree:
                    yield from wait(("R0", "SFree", xb), i // 2)
                yield from wait(("R0", "RingFull", st), (i + 2) // 2)
                issue_s(i + 2)
            yield

    def ew0():
        for i in range(T):
            xb = st = i % 2
            yield from wait(("R0", "RingFull", st), i // 2)
            yield from wait(("R0", "Score", xb), i // 2)
            read_start(("R0", "S", xb), ("S", i), f"ew0({i})")
            yield
            read_end(("R0", "S", xb), f"ew0({i})")
            complete(("R0", "SFree", xb))
            if i >= 2 and not r0_skip_xfree:
                yield from wait(("R0", "XFree", xb), i // 2 - 1)
            write(("R0", "Y", xb), ("P", i))
            yield
            read_start(("R0", "Y", xb), ("P", i), f"copy({i})")
            copies.append((0, xb, i))
            yield

    def drain0():
        for i in range(T):
            xb = i % 2
            yield from wait(("R0", "DQFull", xb), i // 2)
            read_start(("R0", "DQ", xb), ("dQ", i), f"drain({i})")
            yield
            read_end(("R0", "DQ", xb), f"drain({i})")
            complete(("R0", "DQEmpty", xb))

    # ------------------------------------------------------------------ rank 1
    def loader1():
        for i in range(T):
            st = i % 2
            if i >= 2:
                yield from wait(("R1", "RingEmpty", st), i // 2 - 1)
            tma.append((1, st, i))
            yield

    def mma1():
        def issue_dp(i):
            read_start(("R1", "stage", i % 2), ("dO", i), f"dP^T({i})")
            tc[1].append(("dP", i))
            tc[1].append(("commit", ("R1", "Score", i % 2)))

        if T > 0:
            yield from wait(("R1", "RingFull", 0), 0)
            issue_dp(0)
        for i in range(T):
            xb = st = i % 2
            yield from wait(("R1", "XFull", xb), i // 2)
            read_start(("R1", "X", xb), ("P", i), f"dV({i})")
            read_start(("R1", "stage", st), ("dO", i), f"dV({i})")
            tc[1].append(("dV", i))
            tc[1].append(("arrive", ("R0", "XFree", xb)))      # multicast onto rank 0
            if not r1_skip_ds:
                yield from wait(("R1", "DS", xb), i // 2)
            read_start(("R1", "Y", xb), ("dS", i), f"dK1({i})")
            read_start(("R1", "stage", st), ("dO", i), f"dK1({i})")
            tc[1].append(("dK1", i))
            tc[1].append(("commit", ("R1", "DSEmpty", xb)))
            tc[1].append(("commit", ("R1", "RingEmpty", st)))
            if i + 1 < T:
                yield from wait(("R1", "RingFull", (i + 1) % 2), (i + 1) // 2)
                issue_dp(i + 1)
            yield

    def ew1():
        for i in range(T):
            xb = st = i % 2
            yield from wait(("R1", "RingFull", st), i // 2)
            yield from wait(("R1", "Score", xb), i // 2)
            read_start(("R1", "DP", xb), ("dP", i), f"ew1({i})")
            yield from wait(("R1", "XFull", xb), i // 2)
            read_start(("R1", "X", xb), ("P", i), f"ew1({i})")
            yield
            read_end(("R1", "X", xb), f"ew1({i})")
            arrive(("R0", "XFree", xb), 2)      # remote arrival: the warps read P^T(i)
            if i >= 2 and not r1_skip_dsempty:
                yield from wait(("R1", "DSEmpty", xb), i // 2 - 1)
            if i >= 2 and not r1_skip_xfree:
                yield from wait(("R1", "XFree", xb), i // 2 - 1)
            read_end(("R1", "DP", xb), f"ew1({i})")
            write(("R1", "Y", xb), ("dS", i))
            complete(("R1", "DS", xb))
            yield
            read_start(("R1", "Y", xb), ("dS", i), f"copy({i})")
            copies.append((1, xb, i))
            yield

    # ------------------------------------------------------------------ engines
    def tensor_core(rank):
        q = tc[rank]
        while True:
            if not q or rnd.random() < 0.3:
                yield
                continue
            kind, x = q.pop(0)
            if kind == "commit":
                complete(x)
            elif kind == "arrive":
                arrive(x, 2)
            elif kind == "S":
                write(("R0", "S", x % 2), ("S", x))
                read_end(("R0", "stage", x % 2), f"S^T({x})")
            elif kind == "dP":
                write(("R1", "DP", x % 2), ("dP", x))
                read_end(("R1", "stage", x % 2), f"dP^T({x})")
            elif kind == "dK0":
                read_end(("R0", "X", x % 2), f"dK0({x})")
                read_end(("R0", "stage", x % 2), f"dK0({x})")
            elif kind == "dQ":
                write(("R0", "DQ", x % 2), ("dQ", x))
                read_end(("R0", "X", x % 2), f"dQ({x})")
            elif kind == "dV":
                read_end(("R1", "X", x % 2), f"dV({x})")
                read_end(("R1", "stage", x % 2), f"dV({x})")
            elif kind == "dK1":
                read_end(("R1", "Y", x % 2), f"dK1({x})")
                read_end(("R1", "stage", x % 2), f"dK1({x})")
            yield

    def tma_engine():
        while True:
            if not tma or rnd.random() < 0.3:
                yield
                continue
            rank, st, i = tma.pop(rnd.randrange(len(tma)))
            write((f"R{rank}", "stage", st), ("Q" if rank == 0 else "dO", i))
            complete((f"R{rank}", "RingFull", st))
            yield

    def copy_engine():
        while True:
            if not copies or rnd.random() < 0.3:
                yield
                continue
            src, xb, i = copies.pop(rnd.randrange(len(copies)))
            val = ("P", i) if src == 0 else ("dS", i)
            write((f"R{1 - src}", "X", xb), val)
            read_end((f"R{src}", "Y", xb), f"copy({i})")
            complete((f"R{1 - src}", "XFull", xb))
            yield

    roles = [loader0(), mma0(), ew0(), drain0(), loader1(), mma1(), ew1()]
    engines = [tensor_core(0), tensor_core(1), tma_engine(), copy_engine()]
    # Each role and engine runs at its own speed in this run (some of them far slower than
    # the rest), so that orders a fair interleaving would hardly reach are exercised too.
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
    if count(("R0", "DQEmpty", 0)) + count(("R0", "DQEmpty", 1)) != T:
        raise ProtocolError("not every dQ^T was drained")
    if count(("R0", "XFree", 0)) + count(("R0", "XFree", 1)) != T:
        raise ProtocolError("not every P^T tile was released")
    if count(("R1", "XFree", 0)) + count(("R1", "XFree", 1)) != T:
        raise ProtocolError("not every dS^T tile was released")


@pytest.mark.parametrize("T", [1, 2, 3, 5, 8, 13])
def test_pair_protocol_is_race_free(T):
    for seed in range(60):
        simulate(T, seed=seed)


@pytest.mark.parametrize("variant", [
    dict(r0_skip_xfree=True),          # P^T sent into a receive buffer still in use
    dict(r1_skip_ds=True),             # dK1 issued before the warps wrote dS^T
    dict(r0_skip_dqempty=True),        # dQ^T(i) issued before the drain read dQ^T(i - 2)
])
def test_pair_protocol_model_catches_a_dropped_wait(variant):
    with pytest.raises(ProtocolError):
        for seed in range(300):
            simulate(7, seed=seed, **variant)


@pytest.mark.parametrize("variant", [
    dict(r1_skip_dsempty=True),
    dict(r0_skip_sfree=True),
    dict(r1_skip_xfree=True),
    dict(r0_release_x_after_dk=True),
])
def test_pair_protocol_waits_implied_by_the_issue_order(variant):
    """Rank 0 issues S^T(i + 2) after dQ^T(i), and dQ^T(i) waits for dS^T(i), which needs the
    P^T(i) formed from S^T(i).  That loop through both CTAs (the one that bounds the step on
    B200) already orders four of the kernel's waits and releases, which the kernel keeps
    all the same: rank 1's "dS^T read by dK1" (dK1(i - 2) precedes dP^T(i - 1) on its tensor
    core), rank 0's "S^T read", rank 1's wait for rank 0 to release its receive buffer
    (P^T(i) exists only after S^T(i), after dQ^T(i - 2) consumed that buffer), and rank 0's
    release of it before dQ^T rather than after."""
    for seed in range(100):
        simulate(7, seed=seed, **variant)
