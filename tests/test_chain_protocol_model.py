"""A host-side model of the phase-1 chain kernel's cross-CTA hand-off protocol (csrc/scan_tc.cuh,
precond_chain_kernel): rank 1's key ring (NS slots, one loader, NG writer groups taking every
NG-th chunk), rank 0's forwarder sending each chunk's x and d into NX receive slots of rank 1,
and the phase-parity waits the kernel uses on each slot's barrier.

A parity wait on a barrier passes when the barrier's completed phase count has the other parity
than the one waited on, so it is exact only while the waiter is at most one phase ahead of the
slot.  Random schedules (copies landing out of order, chunks of the chain and of the writer
groups taking random times) check that, with the kernel's slot counts, every wait that passes
has really seen its own chunk's phase, and that the protocol never stalls; and that with three
receive slots for four writer groups a wait would pass on a stale phase (the protocol's first
version, which timed out on the GPU)."""
import random

import pytest

from tests.protocol_model import Model, ProtocolError, count_caught

NS, NG, NX = 5, 4, 4  # key ring slots, writer groups, receive slots (ScanChainSmem)


def simulate(nchunks, seed, ns=NS, ng=NG, nx=NX, wait_release=True):
    rng = random.Random(seed)
    full = [0] * ns        # completed phases of rank 1's full[s]
    kempty = [0] * ns      # ... of kempty[s] (writer group released the slot)
    xready = [0] * nx      # ... of xready[m] (forwarder sent x, d)
    outdone = [0] * nx     # ... of outdone[m] (writer copied them out)
    slot_chunk = {}
    issued, inflight, fwd, chain = 0, [], 0, 0
    nxt = list(range(ng))
    busy = [0] * ng
    passes = lambda done, want: (done & 1) != want
    for _ in range(400000):
        if issued < nchunks:  # rank-1 loader: chunk `issued` into its slot once released
            s = issued % ns
            if issued < ns or kempty[s] > issued // ns - 1:
                inflight.append(issued)
                issued += 1
        if inflight and rng.random() < 0.5:  # a copy lands (any order)
            c = inflight.pop(rng.randrange(len(inflight)))
            assert full[c % ns] == c // ns
            full[c % ns] += 1
        if chain < nchunks and rng.random() < 0.3:
            chain += 1
        if fwd < min(chain, nchunks):  # forwarder: chunk fwd into receive slot fwd % nx
            m = fwd % nx
            if fwd < nx or outdone[m] > fwd // nx - 1:
                slot_chunk[m] = fwd
                xready[m] += 1
                fwd += 1
        for g in range(ng):
            c = nxt[g]
            if c >= nchunks:
                continue
            s, m = c % ns, c % nx
            if busy[g] == 0:
                released = (not wait_release) or c < ns or kempty[s] > c // ns - 1
                if released and passes(full[s], (c // ns) & 1) and passes(xready[m], (c // nx) & 1):
                    if full[s] != c // ns + 1:
                        return "key tile wait passed on another chunk's phase"
                    if xready[m] != c // nx + 1 or slot_chunk.get(m) != c:
                        return "x/d wait passed on another chunk's phase"
                    outdone[m] += 1
                    busy[g] = rng.randint(1, 5)
            else:
                busy[g] -= 1
                if busy[g] == 0:
                    kempty[s] += 1
                    nxt[g] = c + ng
        if all(n >= nchunks for n in nxt) and fwd == nchunks:
            return "ok"
    return "stalled"


@pytest.mark.parametrize("nchunks", [1, 5, 9, 64])
def test_kernel_slot_counts_are_exact_and_never_stall(nchunks):
    for seed in range(60):
        assert simulate(nchunks, seed) == "ok", seed


def test_three_receive_slots_for_four_groups_alias():
    results = [simulate(64, seed, nx=3) for seed in range(40)]
    assert any(r.startswith("x/d wait passed") for r in results)


def test_two_groups_with_three_slots_are_exact():
    """The earlier two-group layout (3-slot ring, 3 receive slots) is exact as well."""
    for seed in range(40):
        assert simulate(64, seed, ns=3, ng=2, nx=3) == "ok"


# ---------------------------------------------------------------------------------------------
# All roles of both CTAs, on the shared executor (tests/protocol_model.py): every buffer that
# crosses a role boundary is versioned by its chunk, so a wait that is missing or too weak shows
# up as a read of the wrong chunk's data or a write under a pending read.  Per chunk c:
#   rank 0  forwarder  TMA of k and T_d into ring slot c % 3 (chunks 0-2 up front, chunk c + 3
#                      after fwdin(c)); after fwdin(c) and outdone(c - NG) it copies x_c and the
#                      chunk-start d_c into rank 1's receive slot c % NG, then fwdout(c), xready
#           loader     full(c), fwdout(c - 2); reads e_t from the T_d tile, writes the gate
#                      vectors of slot c % 3, meets the chain at the named barrier
#           chain      the named barrier; reads the tiles, the gate vectors and d_c (slot c % 3),
#                      writes x_c (slot c % 3) and d_{c+1} (slot (c + 1) % 3), then fwdin(c)
#   rank 1  loader     kempty(c - NS); TMA of k into key slot c % NS; r of the chunk, vready
#           writer g   chunks c = g mod NG: kempty(c - NS), full, vready, xready; copies x_c and
#                      d_c out of the receive slot, outdone; reads the key tile and r; kempty
# The named barrier (bar.sync of the loader warp and the 256 chain threads) is modelled as a
# two-party barrier with one phase per chunk.

def chain_roles(N, ns=NS, ng=NG, nx=NX, mut=None):
    def r0_forwarder():
        last = []

        def issue(c):
            last.append(c)
            return ("tma", [("r0ring", c % 3, "K"), ("r0ring", c % 3, "TD")], c,
                    f"r0full{c % 3}", c // 3)

        for c in range(min(3, N)):
            yield issue(c)
        for c in range(N):
            k, m = c % 3, c % nx
            if not (yield ("wait", f"fwdin{k}", c // 3)):
                break
            if c + 3 < N:
                yield issue(c + 3)
            if c >= nx and not (yield ("wait", f"outdone{m}", c // nx - 1)):
                break
            yield ("read", ("sX", k), c)
            yield ("read", ("sD", k), c)
            yield ("write", ("XR", m), c)
            yield ("write", ("DR", m), c)
            yield ("arrive", f"fwdout{k}", c // 3)
            yield ("arrive", f"xready{m}", c // nx)
        for c in last[-3:]:  # the copies in flight land before the block leaves
            yield ("wait", f"r0full{c % 3}", c // 3, "drain")

    def r0_loader():
        for c in range(N):
            s = c % 3
            got = yield ("wait", f"r0full{s}", c // 3)
            if got and c >= 2 and mut != "loader_skips_fwdout":
                got = yield ("wait", f"fwdout{(c - 2) % 3}", (c - 2) // 3)
            if not got:  # the failure flag, then the barrier: the chain leaves at this chunk
                yield ("write", "fail", c if mut == "fixed_exit_paths" else 1)
                yield ("arrive", "bar1", c)
                yield ("wait", "bar1", c, "sync")
                return
            yield ("read", ("r0ring", s, "TD"), c)  # e_t rides in the T_d tile
            yield ("write", ("vecs", s), c)
            yield ("arrive", "bar1", c)
            yield ("wait", "bar1", c, "sync")

    def r0_chain():
        for c in range(N):
            s = c % 3
            yield ("arrive", "bar1", c)
            yield ("wait", "bar1", c, "sync")
            flag = yield ("peek", "fail")
            if (flag <= c) if mut == "fixed_exit_paths" else flag:
                return
            yield ("read", ("r0ring", s, "K"), c)
            yield ("read", ("r0ring", s, "TD"), c)
            yield ("read", ("vecs", s), c)
            yield ("read", ("sD", s), c)
            yield ("write", ("sX", s), c)
            yield ("write", ("sD", (c + 1) % 3), c + 1)
            yield ("arrive", f"fwdin{s}", c // 3)
        yield ("read", ("sD", N % 3), N)  # d_T

    def r1_loader():
        issued = []
        for c in range(N):
            s = c % ns
            if c >= ns and not (yield ("wait", f"kempty{s}", c // ns - 1)):
                for cc in issued[-ns:]:  # its own wait ran out: the loads in flight land
                    yield ("wait", f"r1full{cc % ns}", cc // ns, "drain")
                return
            yield ("tma", [("r1ring", s)], c, f"r1full{s}", c // ns)
            issued.append(c)
            yield ("write", ("rv", s), c)
            yield ("arrive", f"vready{s}", c // ns)
            if mut == "fixed_exit_paths" and c == N - 1:
                for cc in issued[-ns:]:
                    yield ("wait", f"r1full{cc % ns}", cc // ns, "drain")

    def r1_writer(g):
        for c in range(g, N, ng):
            s, m = c % ns, c % nx
            got = True
            if c >= ns and mut != "writer_skips_kempty":
                got = yield ("wait", f"kempty{s}", c // ns - 1)
            got = got and (yield ("wait", f"r1full{s}", c // ns))
            got = got and (yield ("wait", f"vready{s}", c // ns))
            got = got and (yield ("wait", f"xready{m}", c // nx))
            if not got:
                return
            yield ("read", ("XR", m), c)
            yield ("read", ("DR", m), c)
            yield ("arrive", f"outdone{m}", c // nx)
            yield ("read", ("r1ring", s), c)
            yield ("read", ("rv", s), c)
            yield ("arrive", f"kempty{s}", c // ns)

    barriers = {"bar1": 2}
    for s in range(3):
        barriers.update({f"r0full{s}": 1, f"fwdin{s}": 1, f"fwdout{s}": 1})
    for s in range(ns):
        barriers.update({f"r1full{s}": 1, f"vready{s}": 1, f"kempty{s}": 1})
    for m in range(nx):
        barriers.update({f"xready{m}": 1, f"outdone{m}": 1})
    roles = {"r0_forwarder": r0_forwarder(), "r0_loader": r0_loader(), "r0_chain": r0_chain(),
             "r1_loader": r1_loader()}
    roles.update({f"r1_writer{g}": r1_writer(g) for g in range(ng)})
    # set before the cluster barrier that starts the roles: d_0 and the failure flag
    init = {("sD", 0): 0, "fail": N + 1 if mut == "fixed_exit_paths" else 0}
    return barriers, roles, init


def chain_model(N, seed, timeouts=False, drain_timeouts=False, **kw):
    barriers, roles, init = chain_roles(N, **kw)
    return Model(barriers, roles, seed, timeouts=timeouts, drain_timeouts=drain_timeouts,
                 init=init)


@pytest.mark.parametrize("N", [0, 1, 3, 4, 5, 6, 9, 13])
def test_all_roles_exact_in_every_schedule(N):
    for seed in range(200):
        chain_model(N, seed).run()


@pytest.mark.parametrize("kw", [dict(nx=3), dict(mut="writer_skips_kempty"),
                                dict(mut="loader_skips_fwdout")],
                         ids=["three_receive_slots", "writer_skips_kempty", "loader_skips_fwdout"])
def test_all_roles_model_catches_planted_mistakes(kw):
    assert count_caught(lambda seed: chain_model(13, seed, **kw), range(200)) > 0


# ---- exit paths when a bounded wait runs out (any wait may time out; drains do not)

@pytest.mark.parametrize("N", [1, 3, 5, 9, 13])
def test_exit_paths_with_the_two_fixes_are_complete(N):
    """With rank 1's loader waiting for its own copies on every exit, and the failure flag
    carrying the chunk at which the loader gave up (the chain leaves at that chunk's barrier),
    every schedule ends with both CTAs done and nothing in flight."""
    took = 0
    for seed in range(300):
        m = chain_model(N, seed, timeouts=True, mut="fixed_exit_paths")
        m.run()
        took += m.failed
    assert took > 200


def test_exit_paths_as_built_rely_on_the_long_bound():
    """The kernel as built has two exit-path gaps that only a wait far shorter than its 2 s
    bound can reach: rank 1's loader waits for its copies only when its own wait ran out (copies
    may still land after the writers gave up), and the chain reads a yes/no failure flag after
    the named barrier of chunk c, so a loader already failing at chunk c + 1 makes the chain leave
    a chunk early and leaves the loader at a barrier without a timeout.  Under the 2 s bound a
    key copy lands long before, and the flag is set 2 s after the chain's read."""
    kinds = set()
    for N in (3, 9):
        for seed in range(300):
            try:
                chain_model(N, seed, timeouts=True).run()
            except ProtocolError as e:
                kinds.add("in flight" if "in flight" in str(e) else
                          "barrier" if "deadlock" in str(e) and "bar1" in str(e) else str(e))
    assert kinds == {"in flight", "barrier"}, kinds
