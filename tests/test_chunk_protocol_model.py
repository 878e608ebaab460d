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
    last = {}
    yield load(0)
    yield load(1)
    last[0], last[1] = 0, 1
    yield ("wait", "tma_full0", 0)

    def state_update(jj):  # S^T += K~_jj^T W_jj; K~_jj sits in stage jj + 1
        yield ("mma", [(("stage", (jj + 1) & 1, "KT"), jj + 1), ("R", ("W", jj)),
                       ("Sa", ("S", jj)), ("Sb", ("S", jj))],
               [("Sa", ("S", jj + 1)), ("Sb", ("S", jj + 1))])
        yield ("commit", "mma_s", jj)

    for j in range(N):
        i = j + 1
        if j > 0:
            yield ("wait", "mma_crit", j - 1)
            yield from state_update(j - 1)
        yield ("wait", f"tma_full{i & 1}", i >> 1)
        yield ("mma", [(("stage", i & 1, "KQ"), i), (("stage", i & 1, "KT"), i)],
               [("G", ("G", j))])
        yield ("commit", "mma_p", j)
        if j > 0:
            yield ("wait", "s_ready", j - 1)
            if mut != "producer_skips_o_free":
                yield ("wait", "o_free", j - 1)
            yield ("mma", [(("stage", i & 1, "KQ"), i), ("Ssa", ("Ssp", j)), ("Ssb", ("Ssp", j))],
                   [(("D1", i & 1), ("D1a", i))])
            yield ("commit", "d1a_done", j)
        if j + 2 <= N:
            if mut != "refill_without_release":
                yield ("wait", f"stage_empty{j & 1}", j >> 1)
            yield load(j + 2)
            last[(j + 2) & 1] = j + 2
    yield ("wait", "mma_crit", N - 1)
    yield from state_update(N - 1)
    if mut == "no_final_drain":
        return
    # the drain before the block may leave: this thread's copies and MMAs
    for s in (0, 1):
        yield ("wait", f"tma_full{s}", last[s] >> 1)
    yield ("wait", "mma_s", N - 1)


def prep(N, mut):
    if N == 0:
        return

    def zt(i):
        return ("zt_full0", i) if mut == "single_zt_barrier" else (f"zt_full{i & 1}", i >> 1)

    def finish_T(i):  # identity rows of a short chunk's T tiles (modelled for every chunk)
        yield ("rmw", ("stage", i & 1, "T"), i, ("Tfix", i))
        yield ("arrive",) + zt(i)
        yield ("arrive", f"stage_empty{i & 1}", i >> 1)

    yield ("wait", "tma_full0", 0)
    yield from finish_T(0)
    for j in range(N):
        i = j + 1
        for job in ((0, 1) if j > 0 else (1,)):
            if job == 0:  # the split of S_j
                yield ("wait", "mma_s", j - 1)
                yield ("read", "Sa", ("S", j))
                yield ("read", "Sb", ("S", j))
                yield ("write", "Ssa", ("Ssp", j))
                yield ("write", "Ssb", ("Ssp", j))
                yield ("arrive", "s_ready", j - 1)
            else:  # [X_{j+1}; P_j] from the Gram, in place
                yield ("wait", "mma_p", j)
                yield ("rmw", "G", ("G", j), ("XP", j))
                yield ("arrive", "zxp_full", j)
        if i < N:
            yield ("wait", f"tma_full{i & 1}", i >> 1)
            yield from finish_T(i)


def lower(N, mut):
    yield ("write", "Sa", ("S", 0))
    yield ("write", "Ssa", ("Ssp", 0))
    yield ("arrive", "sync1", 0)
    yield ("wait", "sync1", 0)
    if N > 0:  # D1_0 = [K_0; .] S_0^T and D1_1 = [K_1; Q_0] S_0^T
        yield ("wait", "tma_full0", 0)
        yield ("wait", "tma_full1", 0)
        for i in (0, 1):
            yield ("mma", [(("stage", i, "KQ"), i), ("Ssa", ("Ssp", 0)), ("Ssb", ("Ssp", 0))],
                   [(("D1", i), ("D1a", i))])
        yield ("commit", "d1a_done", 0)
    for j in range(N):
        s = j & 1
        if j == 0:
            yield ("wait", "d1a_done", 0)
        else:
            yield ("wait", "mma_crit", j - 1)
        yield ("wait", f"tma_full{s}", j >> 1)
        yield ("read", ("D1", s), ("D1a", 0) if j == 0 else ("D1", j))
        yield ("read", ("stage", s, "V"), j)
        if j > 0 and mut != "lower_skips_mma_s":
            yield ("wait", "mma_s", j - 1)
        yield ("write", "R", ("R", j))
        if mut == "single_zt_barrier":
            yield ("wait", "zt_full0", j)
        else:
            yield ("wait", f"zt_full{s}", j >> 1)
        yield ("mma", [(("stage", s, "T"), ("Tfix", j)), ("R", ("R", j))], [("D2", ("D2", j))])
        yield ("commit", "mma_c", j)
        if mut != "lower_skips_w_done":
            yield ("wait", "w_done", j)
        yield ("wait", "zxp_full", j)
        yield ("wait", "d1a_done", j)
        yield ("mma", [(("D1", (j + 1) & 1), ("D1a", j + 1)), ("G", ("XP", j)), ("R", ("W", j))],
               [(("D1", (j + 1) & 1), ("D1", j + 1))])
        yield ("commit", "mma_crit", j)
    if mut == "no_final_drain":
        return
    if N > 0:
        yield ("wait", "mma_s", N - 1)
    yield ("read", "Sa", ("S", N))


def upper(N, mut):
    yield ("write", "Sb", ("S", 0))
    yield ("write", "Ssb", ("Ssp", 0))
    yield ("arrive", "sync1", 0)
    yield ("wait", "sync1", 0)
    for j in range(N):
        yield ("wait", "mma_c", j)
        yield ("arrive", f"stage_empty{j & 1}", j >> 1)
        yield ("read", "D2", ("D2", j))
        yield ("write", "R", ("W", j))
        yield ("arrive", "w_done", j)
        yield ("wait", "mma_crit", j)
        yield ("read", ("D1", (j + 1) & 1), ("D1", j + 1))
        yield ("arrive", "o_free", j)
    if mut == "no_final_drain":
        return
    if N > 0:
        yield ("wait", "mma_s", N - 1)
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
