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
