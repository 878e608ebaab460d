"""A random-schedule model of the hand-offs inside chunk_fwd_tc_kernel (csrc/chunk_tc.cuh, the
phase-2 state chain), run on the CPU.

The four roles of one CTA are transcribed as sequential programs: the producer (TMA loads, the
Gram, the next [K; Q] S^T product, the state update), the prep warps (the state's split, [X; P]
from the Gram, the T tiles of a short chunk), the chain's lower half (R, W = T R, D1 += [X; P] W)
and its upper half (the W split, the output rows).  Their mbarrier waits, arrivals and commits are
executed in random interleavings, with two freedoms the hardware has:
  - TMA copies complete in any order;
  - a tcgen05.commit tracks only the issuing thread's MMAs, so MMA groups of different threads
    complete in any order (one thread's groups complete in issue order).
Checked in every schedule:
  - every parity wait is exact: when it is evaluated, the barrier has completed the expected phase
    or is in it, and the barrier never completes the next phase while a waiter of the current one
    has not passed (a parity wait cannot tell those cases apart);
  - every arrival lands in the phase it is meant for;
  - every shared-memory tile and tensor-memory column group is read in the version the algorithm
    expects, never while an asynchronous write to it is in flight, and never written while another
    thread's MMA or a copy still reads or writes it;
  - no schedule deadlocks, and every role finishes.
Planted mistakes in the protocol (a single T-tile barrier for both ring slots, a refill without
the release of the stage, a missing wait, a block that leaves without waiting for its last state
update) must each be caught.  The peer CTA's counter and the
cluster barriers are outside the model (they order the two CTAs of a head, not the roles).
"""
import pytest

from tests.protocol_model import Model, count_caught

BARRIERS = {"tma_full0": 1, "tma_full1": 1, "stage_empty0": 2, "stage_empty1": 2,
            "zt_full0": 1, "zt_full1": 1, "mma_c": 1, "mma_p": 1, "mma_crit": 1, "mma_s": 1,
            "zxp_full": 1, "d1a_done": 1, "s_ready": 1, "w_done": 1, "o_free": 1, "sync1": 2}
STAGE_PARTS = ("KQ", "KT", "V", "T")


def load(i):
    """TMA of ring stage i: every part of slot i & 1; lands on tma_full of the slot."""
    return ("tma", [("stage", i & 1, p) for p in STAGE_PARTS], i, f"tma_full{i & 1}", i >> 1)


# ------------------------------------------------------------------ the roles, as in the kernel

def producer(N, mut):
    if N == 0:
        return
    last = {}   # ring slot -> last stage loaded into it (the kernel's pend[])
    lc = []     # this thread's most recent commit (last_bar, last_par)

    def load_(i):
        last[i & 1] = i
        return load(i)

    def commit(bar, k):
        lc[:] = [(bar, k)]
        return ("commit", bar, k)

    def state_update(jj):  # S^T += K~_jj^T W_jj; K~_jj sits in stage jj + 1
        yield ("mma", [(("stage", (jj + 1) & 1, "KT"), jj + 1), ("R", ("W", jj)),
                       ("Sa", ("S", jj)), ("Sb", ("S", jj))],
               [("Sa", ("S", jj + 1)), ("Sb", ("S", jj + 1))])
        yield commit("mma_s", jj)

    yield load_(0)
    yield load_(1)
    ok = yield ("wait", "tma_full0", 0)
    j = 0
    while ok and j < N:
        i = j + 1
        if j > 0:
            ok = yield ("wait", "mma_crit", j - 1)
            if not ok:
                break
            yield from state_update(j - 1)
        ok = yield ("wait", f"tma_full{i & 1}", i >> 1)
        if not ok:
            break
        yield ("mma", [(("stage", i & 1, "KQ"), i), (("stage", i & 1, "KT"), i)],
               [("G", ("G", j))])
        yield commit("mma_p", j)
        if j > 0:
            ok = yield ("wait", "s_ready", j - 1)
            if ok and mut != "producer_skips_o_free":
                ok = yield ("wait", "o_free", j - 1)
            if not ok:
                break
            yield ("mma", [(("stage", i & 1, "KQ"), i), ("Ssa", ("Ssp", j)), ("Ssb", ("Ssp", j))],
                   [(("D1", i & 1), ("D1a", i))])
            yield commit("d1a_done", j)
        if j + 2 <= N:
            if mut != "refill_without_release":
                ok = yield ("wait", f"stage_empty{j & 1}", j >> 1)
                if not ok:
                    break
            yield load_(j + 2)
        j += 1
    if ok and (yield ("wait", "mma_crit", N - 1)):
        yield from state_update(N - 1)
    if mut == "no_final_drain":
        return
    # the drain before the block may leave: this thread's copies and MMAs
    for s, i in sorted(last.items()):
        yield ("wait", f"tma_full{s}", i >> 1, "drain")
    if lc:
        yield ("wait", lc[0][0], lc[0][1], "drain")


def prep(N, mut):
    if N == 0:
        return

    def zt(i):
        return ("zt_full0", i) if mut == "single_zt_barrier" else (f"zt_full{i & 1}", i >> 1)

    def finish_T(i):  # identity rows of a short chunk's T tiles (modelled for every chunk)
        yield ("rmw", ("stage", i & 1, "T"), i, ("Tfix", i))
        yield ("arrive",) + zt(i)
        yield ("arrive", f"stage_empty{i & 1}", i >> 1)

    if not (yield ("wait", "tma_full0", 0)):
        return
    yield from finish_T(0)
    for j in range(N):
        i = j + 1
        for job in ((0, 1) if j > 0 else (1,)):
            if job == 0:  # the split of S_j
                if not (yield ("wait", "mma_s", j - 1)):
                    return
                yield ("read", "Sa", ("S", j))
                yield ("read", "Sb", ("S", j))
                yield ("write", "Ssa", ("Ssp", j))
                yield ("write", "Ssb", ("Ssp", j))
                yield ("arrive", "s_ready", j - 1)
            else:  # [X_{j+1}; P_j] from the Gram, in place
                if not (yield ("wait", "mma_p", j)):
                    return
                yield ("rmw", "G", ("G", j), ("XP", j))
                yield ("arrive", "zxp_full", j)
        if i < N:
            if not (yield ("wait", f"tma_full{i & 1}", i >> 1)):
                return
            yield from finish_T(i)


def lower(N, mut):
    yield ("write", "Sa", ("S", 0))
    yield ("write", "Ssa", ("Ssp", 0))
    yield ("arrive", "sync1", 0)
    yield ("wait", "sync1", 0, "sync")
    ok, lc = True, []
    if N > 0:  # D1_0 = [K_0; .] S_0^T and D1_1 = [K_1; Q_0] S_0^T
        ok = (yield ("wait", "tma_full0", 0)) and (yield ("wait", "tma_full1", 0))
        if ok:
            for i in (0, 1):
                yield ("mma", [(("stage", i, "KQ"), i), ("Ssa", ("Ssp", 0)), ("Ssb", ("Ssp", 0))],
                       [(("D1", i), ("D1a", i))])
            yield ("commit", "d1a_done", 0)
            lc = [("d1a_done", 0)]
    for j in range(N):
        if not ok:
            break
        s = j & 1
        ok = (yield ("wait", "d1a_done", 0) if j == 0 else ("wait", "mma_crit", j - 1)) and \
            (yield ("wait", f"tma_full{s}", j >> 1))
        if not ok:
            break
        yield ("read", ("D1", s), ("D1a", 0) if j == 0 else ("D1", j))
        yield ("read", ("stage", s, "V"), j)
        if j > 0 and mut != "lower_skips_mma_s":
            if not (ok := (yield ("wait", "mma_s", j - 1))):
                break
        yield ("write", "R", ("R", j))
        zt = ("zt_full0", j) if mut == "single_zt_barrier" else (f"zt_full{s}", j >> 1)
        if not (ok := (yield ("wait",) + zt)):
            break
        yield ("mma", [(("stage", s, "T"), ("Tfix", j)), ("R", ("R", j))], [("D2", ("D2", j))])
        yield ("commit", "mma_c", j)
        lc = [("mma_c", j)]
        ok = (mut == "lower_skips_w_done" or (yield ("wait", "w_done", j))) and \
            (yield ("wait", "zxp_full", j)) and (yield ("wait", "d1a_done", j))
        if not ok:
            break
        yield ("mma", [(("D1", (j + 1) & 1), ("D1a", j + 1)), ("G", ("XP", j)), ("R", ("W", j))],
               [(("D1", (j + 1) & 1), ("D1", j + 1))])
        yield ("commit", "mma_crit", j)
        lc = [("mma_crit", j)]
    if mut == "no_final_drain":
        return
    if ok and N > 0:
        ok = yield ("wait", "mma_s", N - 1)
    if ok:
        yield ("read", "Sa", ("S", N))
    elif lc:  # the lower leader's exit path: its own last commit
        yield ("wait", lc[0][0], lc[0][1], "drain")


def upper(N, mut):
    yield ("write", "Sb", ("S", 0))
    yield ("write", "Ssb", ("Ssp", 0))
    yield ("arrive", "sync1", 0)
    yield ("wait", "sync1", 0, "sync")
    ok = True
    for j in range(N):
        if not (ok := (yield ("wait", "mma_c", j))):
            break
        yield ("arrive", f"stage_empty{j & 1}", j >> 1)
        yield ("read", "D2", ("D2", j))
        yield ("write", "R", ("W", j))
        yield ("arrive", "w_done", j)
        if not (ok := (yield ("wait", "mma_crit", j))):
            break
        yield ("read", ("D1", (j + 1) & 1), ("D1", j + 1))
        yield ("arrive", "o_free", j)
    if mut == "no_final_drain":
        return
    if ok and N > 0:
        ok = yield ("wait", "mma_s", N - 1)
    if ok:
        yield ("read", "Sb", ("S", N))


ROLES = {"P": producer, "Q": prep, "L": lower, "U": upper}


def model(N, seed, mut=None):
    return Model(BARRIERS, {name: fn(N, mut) for name, fn in ROLES.items()}, seed)


@pytest.mark.parametrize("N", [0, 1, 2, 3, 4, 7])
def test_protocol_is_exact_in_every_schedule(N):
    for seed in range(300):
        model(N, seed).run()


@pytest.mark.parametrize("mut", ["single_zt_barrier", "refill_without_release",
                                 "lower_skips_mma_s", "lower_skips_w_done", "no_final_drain"])
def test_planted_mistakes_are_caught(mut):
    assert count_caught(lambda seed: model(5, seed, mut), range(200)) > 0, mut


def test_o_free_is_implied_by_the_other_waits():
    """The producer's wait on o_free (the previous chunk's output rows read) is already implied:
    the buffer it writes held D1_{j-1}, whose output rows the upper half read before it released
    W_{j-1}, which the producer's wait on mma_crit covers.  The model finds no schedule without
    it that breaks a check (the kernel keeps the wait)."""
    for seed in range(300):
        model(5, seed, "producer_skips_o_free").run()


@pytest.mark.parametrize("N", [1, 2, 4])
def test_every_role_that_gives_up_drains_its_own_work(N):
    """Any wait may run out (as the kernel's bounded waits do); each role then leaves its loop
    and waits, with a drain bound that does not run out, for its own copies and MMAs.  In every
    schedule the block then leaves with nothing in flight, so the kernel's exit paths are
    complete."""
    took = 0
    for seed in range(300):
        m = Model(BARRIERS, {name: fn(N, None) for name, fn in ROLES.items()}, seed,
                  timeouts=True)
        m.run()
        took += m.failed
    assert took > 100  # most schedules exercise the exit paths


def test_drains_under_the_same_bound_can_leave_work_in_flight():
    """The kernel bounds its drain waits by the same limit as its other waits.  A limit short
    enough to force a timeout would then also cut drains short, and a block could leave while
    its copies or MMAs are still running, which is why the GPU tests force a timeout only in the
    watchdog self-test kernel."""
    make = lambda seed: Model(BARRIERS, {name: fn(4, None) for name, fn in ROLES.items()}, seed,
                              timeouts=True, drain_timeouts=True)
    assert count_caught(make, range(300)) > 0
