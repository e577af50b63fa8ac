"""The pipeline protocol of the tcgen05 attention kernel, checked on the host
(csrc/attn_sm100.cu describes the roles).

The producer loads the key and value tiles in the order the MMA warps
consume them: K(A,0), K(B,0), then per step j: K(A,j+1), V(A,j), K(B,j+1),
V(B,j), each present while that block still has tiles.  The kernel derives
every tile's ring slot from closed forms (slot_k, slot_v); this file
restates them and checks them against a simulation of the producer.

The roles wait on one another as follows (the model below follows them):
- QK(x,j), the n-th S = Q K^T product in the order A(0), B(0), A(1), ...,
  tests its key slot, then waits until the reader of product n - 1 has its
  scores in registers (the one S buffer is shared by both blocks);
- the softmax of x reads S(x,j) after QK(x,j) and after storing P(x,j-1);
- it stores P(x,j) after reading S(x,j) and after O += P V of (x,j-1) has
  completed (P of a block has one buffer in tensor memory);
- PV(x,j) waits for P(x,j), then tests its value slot; the PV warp walks
  (j, x) in the same order as the QK warp.

The QK warp consumes the key tiles and the PV warp the value tiles, so a
stage's previous occupant (slot e - S) can belong to the other warp.  An
mbarrier parity test is exact only while the barrier is at most one phase
behind the tested phase.  The kernel gives each stage two full barriers,
one for its even and one for its odd uses, so that the test for slot e only
needs slot e - 2S to have landed.  The model shows that:
- slot e - 2S has always landed when a consumer tests slot e, so the
  alternating barriers make every test exact;
- slot e - S has not always landed, so one barrier per stage would not be;
- the waits cannot deadlock (the producer included, which reuses a stage
  only after the MMA that read its previous tile has completed);
- the per-block barriers (S full, P stored, O += P V done) are never tested
  while two of their phases are pending, so their parity tests are exact.
"""
import graphlib

import pytest

STAGES = 5


def producer_order(nA, nB):
    out = []
    if nA > 0:
        out.append(("K", 0, 0))
    if nB > 0:
        out.append(("K", 1, 0))
    for j in range(max(nA, nB)):
        if j + 1 < nA:
            out.append(("K", 0, j + 1))
        if j < nA:
            out.append(("V", 0, j))
        if j + 1 < nB:
            out.append(("K", 1, j + 1))
        if j < nB:
            out.append(("V", 1, j))
    return out


def loads_before(j, nA, nB):
    c = (nA > 0) + (nB > 0)
    for n in (nA, nB):
        c += max(0, min(j, n - 1)) + min(j, n)
    return c


def slot_k(x, j, nA, nB):
    if j == 0:
        return 0 if x == 0 else (1 if nA > 0 else 0)
    g = j - 1
    b = loads_before(g, nA, nB)
    return b if x == 0 else b + (g + 1 < nA) + (g < nA)


def slot_v(x, j, nA, nB):
    b = loads_before(j, nA, nB)
    return b + (j + 1 < nA) if x == 0 else b + (j + 1 < nA) + (j < nA) + (j + 1 < nB)


@pytest.mark.parametrize("nA", range(0, 17))
def test_closed_form_slots_match_the_producer(nA):
    for nB in range(0, 17):
        slot = {t: e for e, t in enumerate(producer_order(nA, nB))}
        for x, n in ((0, nA), (1, nB)):
            for j in range(n):
                assert slot[("K", x, j)] == slot_k(x, j, nA, nB)
                assert slot[("V", x, j)] == slot_v(x, j, nA, nB)


def _sequence(nA, nB):
    n = (nA, nB)
    return [(x, j) for j in range(max(nA, nB)) for x in range(2) if j < n[x]]


def happens_before(nA, nB):
    """For every event, the set (bitmask) of ring slots whose landing
    happens before it, and the set of other events known to precede it.
    Events of position i in the (j, x) order depend only on events of
    positions <= i, so one pass in that order computes the closure."""
    slot = {t: e for e, t in enumerate(producer_order(nA, nB))}
    seq = _sequence(nA, nB)
    L, P = {}, {}   # landed slots (bitmask), preceding events (frozenset)

    def dep(ev, *preds, slots=()):
        m, p = 0, set()
        for q in preds:
            if q is None:
                continue
            m |= L[q]
            p |= P[q] | {q}
        for s in slots:
            m |= 1 << s
        L[ev], P[ev] = m, frozenset(p)

    for i, (x, j) in enumerate(seq):
        prev = seq[i - 1] if i else None
        dep(("QKtest", x, j), ("QKissue",) + prev if prev else None)
        dep(("QKissue", x, j), ("QKtest", x, j), ("SREAD",) + prev if prev else None,
            slots=(slot[("K", x, j)],))
        dep(("SREAD", x, j), ("QKissue", x, j), ("PSTORE", x, j - 1) if j else None)
        dep(("PSTORE", x, j), ("SREAD", x, j), ("PVissue", x, j - 1) if j else None)
        dep(("PVtest", x, j), ("PVissue",) + prev if prev else None, ("PSTORE", x, j))
        dep(("PVissue", x, j), ("PVtest", x, j), slots=(slot[("V", x, j)],))
    return slot, seq, L, P


def ring_tests(nA, nB):
    slot, seq, L, _ = happens_before(nA, nB)
    for x, j in seq:
        yield slot[("K", x, j)], L[("QKtest", x, j)]
        yield slot[("V", x, j)], L[("PVtest", x, j)]


def _landed(mask, e):
    return (mask >> e) & 1 == 1


@pytest.mark.parametrize("nA", list(range(0, 14)) + [57, 110, 139])
def test_alternating_full_barriers_make_every_ring_wait_exact(nA):
    for nB in list(range(0, 14)) + [57, 106, 110, 139, 152]:
        for e, landed in ring_tests(nA, nB):
            if e - 2 * STAGES >= 0:
                assert _landed(landed, e - 2 * STAGES), (nA, nB, e)


def test_one_full_barrier_per_stage_would_not_be_exact():
    unsafe = [(nA, nB) for nA in range(0, 9) for nB in range(0, 9)
              if any(e - STAGES >= 0 and not _landed(landed, e - STAGES)
                     for e, landed in ring_tests(nA, nB))]
    assert unsafe


@pytest.mark.parametrize("nA", range(0, 17))
def test_the_waits_cannot_deadlock(nA):
    for nB in range(0, 17):
        order = producer_order(nA, nB)
        slot = {t: e for e, t in enumerate(order)}
        seq = _sequence(nA, nB)
        consumer = {}
        for x, j in seq:
            consumer[slot[("K", x, j)]] = ("QKissue", x, j)
            consumer[slot[("V", x, j)]] = ("PVissue", x, j)
        g = {}

        def add(a, *bs):
            g.setdefault(a, set()).update(b for b in bs if b is not None)

        for e in range(len(order)):
            add(("LOAD", e), ("LOAD", e - 1) if e else None,
                consumer[e - STAGES] if e >= STAGES else None)
        for i, (x, j) in enumerate(seq):
            prev = seq[i - 1] if i else None
            add(("QKissue", x, j), ("LOAD", slot[("K", x, j)]),
                ("QKissue",) + prev if prev else None, ("SREAD",) + prev if prev else None)
            add(("SREAD", x, j), ("QKissue", x, j), ("PSTORE", x, j - 1) if j else None)
            add(("PSTORE", x, j), ("SREAD", x, j), ("PVissue", x, j - 1) if j else None)
            add(("PVissue", x, j), ("PSTORE", x, j), ("LOAD", slot[("V", x, j)]),
                ("PVissue",) + prev if prev else None)
        list(graphlib.TopologicalSorter(g).static_order())  # raises CycleError on a cycle


@pytest.mark.parametrize("nA", range(0, 13))
def test_per_block_barrier_waits_are_exact(nA):
    """S full of block x: the softmax waits for its j-th product; the
    (j+1)-th cannot complete before the softmax has read the j-th (QK(x,j+1)
    follows that read).  P stored of x: the PV warp waits for P(x,j); P(x,j+1)
    is stored only after O += P V of (x,j), which follows that wait.  O += P V
    done of x: the softmax waits for (x,j-1) before storing P(x,j); (x,j) is
    issued only after that store."""
    for nB in range(0, 13):
        _, seq, _, P = happens_before(nA, nB)
        n = (nA, nB)
        for x, j in seq:
            if j + 1 < n[x]:
                assert ("SREAD", x, j) in P[("QKissue", x, j + 1)]
                assert ("PVtest", x, j) in P[("PSTORE", x, j + 1)]
            if j >= 1:
                assert ("PSTORE", x, j) in P[("PVissue", x, j)]
                assert ("PVissue", x, j - 1) in P[("PSTORE", x, j)]
