"""The K/V ring of the tcgen05 attention kernel, checked on the host
(csrc/attn_sm100.cu describes the roles).

The producer loads, per step, the key tiles two steps ahead of the value
tiles: K(0), K(1), V(0), K(2), V(1), ..., each group holding block A's tile
then block B's while that block still has tiles.  The kernel derives every
tile's ring slot from closed forms (slot_k, slot_v); this file restates them
and checks them against a simulation of the producer.

The QK warp consumes the key tiles and the PV warp the value tiles, so a
stage's previous occupant (slot e - S) can belong to the other warp.  An
mbarrier parity test is exact only while the barrier is at most one phase
behind the tested phase.  The kernel gives each stage two full barriers,
one for its even and one for its odd uses, so that the test for slot e only
needs slot e - 2S to have landed.  The model below follows the kernel's
barrier waits (happens-before chains between the roles) and shows that:
- slot e - 2S has always landed when a consumer tests slot e, so the
  alternating barriers make every test exact;
- slot e - S has not always landed, so one barrier per stage would not be.
"""
import functools

import pytest

STAGES = 4


def producer_order(nA, nB):
    out = []
    for g in range(2 * max(nA, nB) + 1):
        is_v = g > 0 and g % 2 == 0
        j = 0 if g == 0 else (g // 2 - 1 if is_v else (g + 1) // 2)
        for x in range(2):
            if j < (nA if x == 0 else nB):
                out.append(("V" if is_v else "K", x, j))
    return out


def steps_before(m, nA, nB):
    m = max(m, 0)
    return min(m, nA) + min(m, nB)


def slot_k(x, j, nA, nB):
    return steps_before(j, nA, nB) + steps_before(j - 1, nA, nB) + (1 if x == 1 and j < nA else 0)


def slot_v(x, j, nA, nB):
    return steps_before(j + 2, nA, nB) + steps_before(j, nA, nB) + (1 if x == 1 and j < nA else 0)


@pytest.mark.parametrize("nA", range(0, 17))
def test_closed_form_slots_match_the_producer(nA):
    for nB in range(0, 17):
        slot = {t: e for e, t in enumerate(producer_order(nA, nB))}
        for x, n in ((0, nA), (1, nB)):
            for j in range(n):
                assert slot[("K", x, j)] == slot_k(x, j, nA, nB)
                assert slot[("V", x, j)] == slot_v(x, j, nA, nB)


def landed_before_tests(nA, nB):
    """For each consumer test of a ring slot, the set of slots whose landing
    happens before it.  Events and their predecessors follow the kernel:
    QK(x,j) waits K(x,j) and S_x free (the softmax read S_x(j-1)); the
    softmax reads S_x(j) after QK(x,j) and after its own previous tile; it
    stores P half h after the previous hand-off's PV half h (hand-off order
    A(0), B(0), A(1), ...); PV(x,j) waits P half 0, then V(x,j), then P half
    1.  Each MMA warp walks (j, x) in order."""
    slot = {t: e for e, t in enumerate(producer_order(nA, nB))}
    n = (nA, nB)
    seq = [(x, j) for j in range(max(nA, nB)) for x in range(2) if j < n[x]]

    def prev_handoff(x, j):
        if x == 0:
            return None if j < 1 else ((1, j - 1) if j - 1 < nB else (0, j - 1))
        if j < nA:
            return (0, j)
        return (1, j - 1) if j >= 1 else None

    @functools.lru_cache(None)
    def L(ev):
        kind, s = ev[0], set()
        if kind == "QKtest":
            i = seq.index(ev[1:])
            if i > 0:
                s |= L(("QKissue",) + seq[i - 1])
        elif kind == "QKissue":
            _, x, j = ev
            s |= L(("QKtest", x, j)) | {slot[("K", x, j)]}
            if j >= 1:
                s |= L(("SREAD", x, j - 1))
        elif kind == "SREAD":
            _, x, j = ev
            s |= L(("QKissue", x, j))
            if j >= 1:
                s |= L(("PSTORE", x, j - 1, 1))
        elif kind == "PSTORE":
            _, x, j, h = ev
            s |= L(("SREAD", x, j)) if h == 0 else L(("PSTORE", x, j, 0))
            p = prev_handoff(x, j)
            if p is not None:
                s |= L(("PVissue", p[0], p[1], h))
        elif kind == "PVtest":
            i = seq.index(ev[1:])
            if i > 0:
                s |= L(("PVissue",) + seq[i - 1] + (1,))
            s |= L(("PSTORE",) + ev[1:] + (0,))
        elif kind == "PVissue":
            _, x, j, h = ev
            s |= L(("PVtest", x, j)) | {slot[("V", x, j)]} | L(("PSTORE", x, j, h))
            if h == 1:
                s |= L(("PVissue", x, j, 0))
        return frozenset(s)

    for x, j in seq:
        yield slot[("K", x, j)], L(("QKtest", x, j))
        yield slot[("V", x, j)], L(("PVtest", x, j))


def test_alternating_full_barriers_make_every_ring_wait_exact():
    for nA in range(0, 13):
        for nB in range(0, 13):
            for e, landed in landed_before_tests(nA, nB):
                if e - 2 * STAGES >= 0:
                    assert e - 2 * STAGES in landed, (nA, nB, e)


def test_one_full_barrier_per_stage_would_not_be_exact():
    unsafe = [(nA, nB) for nA in range(0, 9) for nB in range(0, 9)
              if any(e - STAGES >= 0 and e - STAGES not in landed
                     for e, landed in landed_before_tests(nA, nB))]
    assert (2, 3) in unsafe  # PV(A, 1) tests slot 7 while K(B, 1) (slot 3) may be in flight


def hand_off_order(nA, nB):
    """The P hand-offs of one pair in the kernel's order: A(0), B(0), A(1),
    B(1), ... (a block past its last tile drops out)."""
    return [(x, j) for j in range(max(nA, nB)) for x in range(2) if j < (nA, nB)[x]]


def previous_hand_off(x, j, nA, nB):
    """The hand-off whose O += P V the softmax of block x waits for before
    storing P of its tile j, as the kernel computes it (None for the first)."""
    if x == 0:
        return None if j < 1 else ((1, j - 1) if j - 1 < nB else (0, j - 1))
    if j < nA:
        return (0, j)
    return (1, j - 1) if j >= 1 else None


@pytest.mark.parametrize("nA", range(0, 13))
def test_hand_off_waits_are_exact_within_a_pair(nA):
    """Block x tests, by parity, the phase of the previous hand-off (block
    y, its k-th) on y's barrier.  The test is exact when y's phase k - 1 is
    complete; x knows every hand-off before its own previous one complete
    (it waited for the one just before that, and the MMAs complete in
    issue order)."""
    for nB in range(0, 13):
        order = hand_off_order(nA, nB)
        pos = {h: m for m, h in enumerate(order)}
        last_own = {}
        for m, (x, j) in enumerate(order):
            prev = previous_hand_off(x, j, nA, nB)
            assert prev == (order[m - 1] if m else None)  # the chain's predecessor
            if prev is not None:
                y, k = prev
                if k >= 1:
                    known = last_own.get(x, -1) - 1
                    assert pos[(y, k - 1)] <= known, (nA, nB, x, j)
            last_own[x] = m
