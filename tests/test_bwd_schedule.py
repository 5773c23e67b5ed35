"""Host model of the backward main kernel's pipeline schedule (fa_bwd.cuh).

Per step i (one query block against the CTA's key block) the MMA warp issues, in order:
    dV(i) [reads P^T(i) from the S^T columns of TMEM, dO of Q/dO stage i]
    S^T(i+1) [overwrites the S^T columns; reads Q of stage i+1]
    dK(i), dQ^T(i) [read dS^T(i) from shared memory; dQ^T(i) overwrites the dQ^T columns
                    once the drain warps have read dQ^T(i-1)]
    dP^T(i+1) [overwrites the dP^T columns: the elementwise warps read dP^T(i) before they
               wrote dS^T(i), which dK(i) waited for]
and commits "dQ ready", "dS free" and "Q/dO stage free" after dQ^T(i).  The elementwise
warps read S^T(i), write P^T(i) over it, read dP^T(i) and write dS^T(i); the drain warps
read dQ^T(i).  The loader fills the Q/dO ring.  (The model also runs a reordering that
issues dP^T(i+1) before dK(i) behind a separate "dP read" barrier, with two dS^T
buffers: it is race-free too, but measured slower on B200.)

This model runs the loader, the MMA warp, the elementwise warps, the dQ drain and the
asynchronous engines (tensor core in issue order, TMA copies landing in any order) as
coroutines under random interleavings.  Every wait checks the mbarrier phase discipline
(a parity wait for phase k is only correct while the barrier has completed k or k + 1
phases), and every buffer access checks that it reads what it expects and overwrites only
what has been consumed: the S^T / P^T columns, the dP^T columns, the dS^T buffers, the
dQ^T columns and the Q/dO stages.  Variants that drop a wait (dP^T(i+1) issued early
without the "dP read" barrier, dS^T written without its "free" wait, a single "dS
written" barrier for two buffers, dQ^T(i) issued before dQ^T(i-1) was drained) must
fail.
"""
import random

import pytest


class ScheduleError(AssertionError):
    pass


def simulate(T, QS=3, NB=1, seed=0, dp_early=False, dpfree_wait=True, dsempty_wait=True,
             ds_barrier_per_buffer=True, dqempty_wait=True, dp_after_dk=False):
    rnd = random.Random(seed)
    done = {}
    state = {"S": None, "dP": None, "dQ": None, "dS": [None] * NB, "stage": [None] * QS}
    consumed = {"dP": set(), "dQ": set()}
    reads_left = {}           # (kind, step) -> pending engine reads of a dS buffer / stage
    engine, tma = [], []

    def count(b):
        return done.get(b, 0)

    def complete(b):
        done[b] = count(b) + 1

    def ready(b, k):
        c = count(b)
        if c not in (k, k + 1):
            raise ScheduleError(f"{b}: {c} phases completed while waiting for phase {k}")
        return c == k + 1

    def ds_bar(db):
        return ("DS", db) if ds_barrier_per_buffer else ("DS",)

    def loader():
        for i in range(T):
            st = i % QS
            if i >= QS:
                while not ready(("QE", st), i // QS - 1):
                    yield
                if reads_left.get(("stage", i - QS), 0):
                    raise ScheduleError(f"stage {st} reloaded while step {i - QS} still reads it")
            tma.append((st, i))
            yield

    def mma():
        while not ready(("QF", 0), 0):
            yield
        reads_left[("stage", 0)] = 4           # S, dP, dV, dK read stage 0
        engine.append(("S", 0))
        engine.append(("commit", ("S",)))
        engine.append(("dP", 0))
        engine.append(("commit", ("DP",)))
        for i in range(T):
            st, db, du = i % QS, i % NB, i // NB
            while not ready(("P",), i):
                yield
            engine.append(("dV", i))
            if i + 1 < T:
                st1 = (i + 1) % QS
                while not ready(("QF", st1), (i + 1) // QS):
                    yield
                reads_left[("stage", i + 1)] = 4
                engine.append(("S", i + 1))
                engine.append(("commit", ("S",)))
                if dp_early:
                    if dpfree_wait:
                        while not ready(("DPF",), i):
                            yield
                    engine.append(("dP", i + 1))
                    engine.append(("commit", ("DP",)))
            while not ready(ds_bar(db), du if ds_barrier_per_buffer else i):
                yield
            engine.append(("dK", i))
            if dp_after_dk and not dp_early and i + 1 < T:
                engine.append(("dP", i + 1))
                engine.append(("commit", ("DP",)))
            if i > 0 and dqempty_wait:
                while not ready(("DQE",), i - 1):
                    yield
            engine.append(("dQ", i))
            engine.append(("commit", ("DQ",)))
            engine.append(("commit", ("DSE", db)))
            engine.append(("commit", ("QE", st)))
            if not dp_early and not dp_after_dk and i + 1 < T:
                engine.append(("dP", i + 1))
                engine.append(("commit", ("DP",)))
            yield

    def elementwise():
        for i in range(T):
            st, db, du = i % QS, i % NB, i // NB
            while not ready(("QF", st), i // QS):
                yield
            while not ready(("S",), i):
                yield
            if state["S"] != ("S", i):
                raise ScheduleError(f"step {i} reads {state['S']} as S^T")
            yield
            state["S"] = ("P", i)
            complete(("P",))
            yield
            while not ready(("DP",), i):
                yield
            if state["dP"] != ("dP", i):
                raise ScheduleError(f"step {i} reads {state['dP']} as dP^T")
            consumed["dP"].add(i)
            complete(("DPF",))
            yield
            if dsempty_wait and du >= 1:
                while not ready(("DSE", db), du - 1):
                    yield
            if reads_left.get(("ds", i - NB), 0):
                raise ScheduleError(f"dS^T buffer {db} overwritten while step {i - NB} still reads it")
            state["dS"][db] = i
            reads_left[("ds", i)] = 2           # dK and dQ^T read it
            complete(ds_bar(db))
            yield

    def drain():
        for i in range(T):
            while not ready(("DQ",), i):
                yield
            if state["dQ"] != ("dQ", i):
                raise ScheduleError(f"drain reads {state['dQ']} as dQ^T({i})")
            consumed["dQ"].add(i)
            yield
            complete(("DQE",))

    def tensor_core():
        while True:
            if not engine or rnd.random() < 0.3:
                yield
                continue
            op = engine.pop(0)
            kind, x = op
            if kind == "commit":
                complete(x)
            elif kind == "S":
                if x > 0 and state["S"] != ("P", x - 1):
                    raise ScheduleError(f"S^T({x}) overwrites {state['S']} before P^T({x - 1}) was consumed")
                if state["stage"][x % QS] != x:
                    raise ScheduleError(f"S^T({x}) reads stage holding step {state['stage'][x % QS]}")
                state["S"] = ("S", x)
                reads_left[("stage", x)] -= 1
            elif kind == "dP":
                if x > 0 and (x - 1) not in consumed["dP"]:
                    raise ScheduleError(f"dP^T({x}) overwrites dP^T({x - 1}) before it was read")
                if state["stage"][x % QS] != x:
                    raise ScheduleError(f"dP^T({x}) reads stage holding step {state['stage'][x % QS]}")
                state["dP"] = ("dP", x)
                reads_left[("stage", x)] -= 1
            elif kind == "dV":
                if state["S"] != ("P", x):
                    raise ScheduleError(f"dV({x}) reads {state['S']} as P^T")
                reads_left[("stage", x)] -= 1
            elif kind in ("dK", "dQ"):
                if state["dS"][x % NB] != x:
                    raise ScheduleError(f"{kind}({x}) reads dS^T of step {state['dS'][x % NB]}")
                reads_left[("ds", x)] -= 1
                if kind == "dK":
                    reads_left[("stage", x)] -= 1
                else:
                    if x > 0 and (x - 1) not in consumed["dQ"]:
                        raise ScheduleError(f"dQ^T({x}) overwrites dQ^T({x - 1}) before it was drained")
                    state["dQ"] = ("dQ", x)
            yield

    def tma_engine():
        while True:
            if not tma or rnd.random() < 0.3:
                yield
                continue
            st, i = tma.pop(rnd.randrange(len(tma)))
            state["stage"][st] = i
            complete(("QF", st))
            yield

    roles = [loader(), mma(), elementwise(), drain()]
    engines = [tensor_core(), tma_engine()]
    live = list(roles)
    for _ in range(200000):
        if not live:
            break
        g = rnd.choice(live + engines)
        try:
            next(g)
        except StopIteration:
            live.remove(g)
    else:
        raise ScheduleError("no progress: a wait never completes")
    # drain the engines so every commit lands
    for _ in range(10000):
        for g in engines:
            next(g)
    if len(consumed["dQ"]) != T:
        raise ScheduleError("not every dQ^T was drained")


@pytest.mark.parametrize("T", [1, 2, 3, 5, 9, 16])
def test_backward_schedule_is_race_free(T):
    for seed in range(80):
        simulate(T, seed=seed)


@pytest.mark.parametrize("T", [1, 2, 5, 16])
def test_dp_between_dk_and_dq_is_race_free(T):
    for seed in range(80):
        simulate(T, seed=seed, dp_after_dk=True)


@pytest.mark.parametrize("T", [2, 7])
def test_early_dp_reordering_is_race_free_too(T):
    for seed in range(60):
        simulate(T, NB=2, seed=seed, dp_early=True)


def test_schedule_model_catches_an_early_dp_without_its_barrier():
    with pytest.raises(ScheduleError):
        for seed in range(200):
            simulate(6, seed=seed, dp_early=True, dpfree_wait=False)


def test_schedule_model_catches_a_missing_dq_drained_wait():
    with pytest.raises(ScheduleError):
        for seed in range(200):
            simulate(6, seed=seed, dqempty_wait=False)


def test_schedule_model_catches_a_missing_ds_free_wait_in_the_reordering():
    # In the kernel's order dP^T(i+1) follows dQ^T(i), which already orders the next dS^T
    # write after the reads of this one; with dP^T issued early the wait is what does it.
    simulate(6, seed=1, dsempty_wait=False)
    with pytest.raises(ScheduleError):
        for seed in range(200):
            simulate(6, NB=1, seed=seed, dp_early=True, dsempty_wait=False)


def test_schedule_model_catches_one_ds_barrier_for_two_buffers():
    with pytest.raises(ScheduleError):
        for seed in range(400):
            simulate(8, NB=2, seed=seed, dp_early=True, ds_barrier_per_buffer=False)
