"""Host model of the block-sparse forward's pipeline schedule (fa_fwd.cuh, kAttnSparse).

The block-sparse forward shares its two TMEM score buffers between its two query tiles:
score tiles are numbered in block-list order (tile 0 before tile 1 within a step) and use
buffer n & 1; the MMA warp issues score tile n + 2 right after P V of score tile n.  Its
mbarriers are "S ready" per (buffer, tile), "P written" per buffer, "P V done" per tile
and "O done" per tile, plus the TMA ring's full / empty barriers.

This model runs the TMA warp, the MMA warp, both softmax warpgroups and the asynchronous
engines (tensor core in issue order, TMA copies in any order) as coroutines under random
interleavings, following the kernel's schedule step by step.  Every wait checks the
mbarrier phase discipline the hardware relies on: a parity wait for phase k is only
correct while the barrier has completed k or k + 1 phases (two behind or ahead and the
parity test passes or blocks wrongly).  It also checks that no score buffer is
overwritten before its P has been consumed, that O is rescaled only after the tile's
previous P V completed, and that each MMA reads the K or V block it expects.

A variant with one "S ready" barrier per buffer (shared by both tiles' softmax
warpgroups) must fail the check: a tile whose first block sits in a buffer's second
occupancy would wait on a phase whose parity already reads as complete.
"""
import random

import pytest

T0, T1 = 1 << 14, 1 << 15   # membership bits of a block-list entry


class PhaseError(AssertionError):
    pass


def simulate(entries, slots=4, seed=0, rescale_p=0.3, s_barrier_per_tile=True):
    rnd = random.Random(seed)
    nu = len(entries)
    nblk = [sum(1 for e in entries if e & (T0 << t)) for t in range(2)]
    total = sum(nblk)
    done = {}                    # barrier -> completed phases
    ring = {}                    # slot -> (step, kind) landed
    tma_flight = []              # (slot, (step, kind))
    engine = []                  # tensor-core queue, in issue order
    buf = {}                     # buffer -> (score tile n, "S" | "P")
    pv_done = set()              # (tile, own block index) and ("n", n)

    def count(b):
        return done.get(b, 0)

    def complete(b):
        done[b] = count(b) + 1

    def ready(b, k):
        c = count(b)
        if c not in (k, k + 1):
            raise PhaseError(f"{b}: {c} phases completed while waiting for phase {k}")
        return c == k + 1

    def s_bar(b, t):
        return ("S", b, t) if s_barrier_per_tile else ("S", b)

    def first_pos():
        return 0, (0 if entries[0] & T0 else 1)

    def advance(j, t):
        if t == 0 and entries[j] & T1:
            return j, 1
        j += 1
        return j, (0 if j < nu and entries[j] & T0 else 1)

    def last_of_step(j, t):
        return t == 1 or not entries[j] & T1

    kslot = lambda j: (2 * j) % slots
    vslot = lambda j: (2 * j + 1) % slots

    def producer():
        for j in range(nu):
            for kind in (0, 1):
                seq = 2 * j + kind
                while seq >= slots and not ready(("E", seq % slots), seq // slots - 1):
                    yield
                tma_flight.append((seq % slots, (j, kind)))
                yield

    def mma():
        if total == 0:
            return
        q = {"j": 0, "t": 0, "n": 0, "k_ready": -1}
        q["j"], q["t"] = first_pos()

        def issue_next_qk():
            j, t = q["j"], q["t"]
            if j != q["k_ready"]:
                while not ready(("F", kslot(j)), (2 * j) // slots):
                    yield
                assert ring[kslot(j)] == (j, 0), "Q K^T reads the wrong K block"
                q["k_ready"] = j
            n = q["n"]
            engine.append(("qk", n & 1, n))
            engine.append(("commit", s_bar(n & 1, t)))
            if last_of_step(j, t):
                engine.append(("commit", ("E", kslot(j))))
            q["n"] += 1
            q["j"], q["t"] = advance(j, t)

        yield from issue_next_qk()
        if total > 1:
            yield from issue_next_qk()
        cnt = [0, 0]
        j, t = first_pos()
        v_ready = -1
        for n in range(total):
            if j != v_ready:
                while not ready(("F", vslot(j)), (2 * j + 1) // slots):
                    yield
                assert ring[vslot(j)] == (j, 1), "P V reads the wrong V block"
                v_ready = j
            while not ready(("P", n & 1), n >> 1):
                yield
            engine.append(("pv", n & 1, n, t, cnt[t]))
            cnt[t] += 1
            engine.append(("commit", ("PV", t)))
            if cnt[t] == nblk[t]:
                engine.append(("commit", ("O", t)))
            if last_of_step(j, t):
                engine.append(("commit", ("E", vslot(j))))
            if n + 2 < total:
                yield from issue_next_qk()
            j, t = advance(j, t)
            yield

    def softmax(t):
        cur, nbase, prev, uses = -1, 0, 0, [0, 0]
        for k in range(nblk[t]):
            while True:
                nbase += prev
                cur += 1
                prev = bin(entries[cur] >> 14).count("1")
                if cur >= nu - 1 or entries[cur] & (T0 << t):
                    break
            n = nbase + (1 if t == 1 and entries[cur] & T0 else 0)
            b = n & 1
            phase = uses[b] if s_barrier_per_tile else n >> 1
            while not ready(s_bar(b, t), phase):
                yield
            uses[b] += 1
            assert buf.get(b) == (n, "S"), f"softmax of score tile {n} reads {buf.get(b)}"
            yield
            assert buf.get(b) == (n, "S"), "score tile overwritten while being read"
            if k > 0 and rnd.random() < rescale_p:
                while not ready(("PV", t), k - 1):
                    yield
                assert (t, k - 1) in pv_done, "O rescaled before the previous P V finished"
            buf[b] = (n, "P")
            complete(("P", b))
            yield
        if nblk[t]:
            while not ready(("O", t), 0):
                yield
            assert (t, nblk[t] - 1) in pv_done

    def async_engines():
        while True:
            if tma_flight and rnd.random() < 0.5:
                slot, item = tma_flight.pop(rnd.randrange(len(tma_flight)))
                ring[slot] = item
                complete(("F", slot))
            if engine and rnd.random() < 0.5:
                op = engine.pop(0)
                if op[0] == "qk":
                    _, b, n = op
                    if n >= 2:
                        assert buf.get(b) == (n - 2, "P") and ("n", n - 2) in pv_done, \
                            "Q K^T overwrote a buffer whose P was not consumed"
                    buf[b] = (n, "S")
                elif op[0] == "pv":
                    _, b, n, t, k = op
                    assert buf.get(b) == (n, "P"), "P V read a buffer without its P"
                    pv_done.update({(t, k), ("n", n)})
                else:
                    complete(op[1])
            yield

    roles = [producer(), mma(), softmax(0), softmax(1)]
    live = [True] * 4
    eng = async_engines()
    for _ in range(500000):
        if not any(live):
            return
        i = rnd.randrange(5)
        if i == 4:
            next(eng)
            continue
        if live[i]:
            try:
                next(roles[i])
            except StopIteration:
                live[i] = False
    raise AssertionError("no progress: the schedule deadlocks")


def random_lists(count, seed):
    rnd = random.Random(seed)
    for _ in range(count):
        nu = rnd.randint(1, 10)
        yield [j | (T0 if m & 1 else 0) | (T1 if m & 2 else 0)
               for j, m in enumerate(rnd.choice((1, 2, 3)) for _ in range(nu))]


@pytest.mark.parametrize("slots", [4, 6])   # the K/V ring at d = 128 and d = 64
def test_sparse_schedule_keeps_phase_discipline(slots):
    for i, entries in enumerate(random_lists(300, slots)):
        simulate(entries, slots=slots, seed=i, rescale_p=1.0 if i % 2 else 0.3)


def test_sparse_schedule_edge_lists():
    cases = [
        [0 | T1],                         # one block, tile 1 only
        [0 | T0 | T1],                    # one shared block
        [j | T0 for j in range(8)],       # tile 0 alone (tile 1 empty)
        [j | T1 for j in range(8)],       # tile 1 alone
        [j | (T0 if j % 2 else T1) for j in range(9)],   # alternating tiles
    ]
    for i, entries in enumerate(cases):
        for seed in range(20):
            simulate(entries, seed=100 * i + seed, rescale_p=1.0)


def test_shared_s_barrier_per_buffer_is_caught():
    # Tile 1's first block is the second occupant of buffer 1 (score tiles 0, 1 are tile
    # 0's): with one S barrier per buffer its softmax would wait for phase 1 while phase 0
    # may still be running, and a parity wait would pass at once.
    entries = [0 | T0, 1 | T0, 2 | T1, 3 | T1]
    caught = 0
    for seed in range(50):
        try:
            simulate(entries, seed=seed, s_barrier_per_tile=False)
        except PhaseError:
            caught += 1
    assert caught > 0
