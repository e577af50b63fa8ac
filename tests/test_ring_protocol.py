"""The K/V ring and the P hand-off chain of the tcgen05 attention kernel,
checked on the host (csrc/attn_sm100.cu describes the roles).

The kernel is persistent: each CTA walks a sequence of work items (pairs
of query blocks A and B).  Within an item the producer loads the key tiles
two steps ahead of the value tiles: K(0), K(1), V(0), K(2), V(1), ..., each
group holding block A's tile then block B's while that block still has
tiles; an item's slots follow the previous item's.  The kernel derives
every tile's ring slot from closed forms (slot_k, slot_v, offset by the
slots of the items before); this file restates them and checks them
against a simulation of the producer.

Each ring stage has three full barriers that take its uses in turn.  A
parity wait on slot e is exact when slot e - 3S (the barrier's previous
use) has landed.  The argument in the kernel: a consumer tests slot e only
after its own previous slot e' landed; the producer issues slots in order
and issues slot e - 2S only after slot e - 3S was consumed; so slot e - 3S
has landed whenever e - e' <= 2S.  The tests check that gap bound (at most
5) over many item sequences, and that two barriers per stage (which need
e - e' <= S) would not be enough once items follow one another.

The QK warp writes, beside each S tile, which P hand-off precedes it: the
tile it issued just before.  The PV warp consumes the hand-offs in the same
order, so each hand-off's barrier phase is its block's hand-off count; the
last test replays the records against that chain.
"""
import random

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
        assert len(slot) == 2 * (nA + nB)
        for x, n in ((0, nA), (1, nB)):
            for j in range(n):
                assert slot[("K", x, j)] == slot_k(x, j, nA, nB)
                assert slot[("V", x, j)] == slot_v(x, j, nA, nB)


def consumer_slots(items):
    """Global ring slots, in each consumer's order, for a sequence of items
    [(nA, nB), ...]: the QK warp takes the key tiles and the PV warp the
    value tiles, both walking (item, j, x) in order."""
    qk, pv, e0 = [], [], 0
    for nA, nB in items:
        for j in range(max(nA, nB)):
            for x in range(2):
                if j < (nA, nB)[x]:
                    qk.append(e0 + slot_k(x, j, nA, nB))
                    pv.append(e0 + slot_v(x, j, nA, nB))
        e0 += 2 * (nA + nB)
    return qk, pv


def max_gap(slots):
    return max((b - a for a, b in zip(slots, slots[1:])), default=0)


def random_items(rng, n):
    out = []
    for _ in range(n):
        r = rng.random()
        if r < 0.1:
            out.append((0, 0))
        elif r < 0.2:
            out.append((rng.randint(1, 9), 0))
        elif r < 0.3:
            out.append((0, rng.randint(1, 9)))
        else:
            out.append((rng.randint(1, 9), rng.randint(1, 9)))
    return out


def test_global_slots_follow_the_producer_across_items():
    rng = random.Random(7)
    for _ in range(200):
        items = random_items(rng, rng.randint(1, 6))
        order, e0 = {}, 0
        for i, (nA, nB) in enumerate(items):
            for e, t in enumerate(producer_order(nA, nB)):
                order[(i,) + t] = e0 + e
            e0 += 2 * (nA + nB)
        qk, pv = consumer_slots(items)
        want_qk = [order[(i, "K", x, j)] for i, (nA, nB) in enumerate(items)
                   for j in range(max(nA, nB)) for x in range(2) if j < (nA, nB)[x]]
        want_pv = [order[(i, "V", x, j)] for i, (nA, nB) in enumerate(items)
                   for j in range(max(nA, nB)) for x in range(2) if j < (nA, nB)[x]]
        assert qk == want_qk and pv == want_pv
        # every slot is used exactly once, by one of the two consumers
        assert sorted(qk + pv) == list(range(e0))


def test_consecutive_slots_of_a_consumer_are_at_most_5_apart():
    rng = random.Random(1)
    worst = 0
    for _ in range(3000):
        qk, pv = consumer_slots(random_items(rng, rng.randint(1, 5)))
        worst = max(worst, max_gap(qk), max_gap(pv))
    assert worst == 5
    # exhaustive over pairs of small items
    for a in range(0, 6):
        for b in range(0, 6):
            for c in range(0, 6):
                for d in range(0, 6):
                    qk, pv = consumer_slots([(a, b), (c, d)])
                    assert max_gap(qk) <= 5 and max_gap(pv) <= 5
    # the first slot each consumer tests has no earlier use of its barrier
    for a in range(0, 8):
        for b in range(0, 8):
            qk, pv = consumer_slots([(a, b)])
            if qk:
                assert qk[0] == 0 and pv[0] <= 4


def barriers_exact(items, per_stage):
    """The kernel's argument with `per_stage` barriers per stage: every test
    of slot e is exact when e - e' <= (per_stage - 1) * STAGES for the
    consumer's previous slot e', or when slot e is the barrier's first use."""
    for slots in consumer_slots(items):
        prev = None
        for e in slots:
            first_use = e < per_stage * STAGES
            if not first_use and (prev is None or e - prev > (per_stage - 1) * STAGES):
                return False
            prev = e
    return True


def test_three_full_barriers_per_stage_are_exact_and_two_are_not_across_items():
    rng = random.Random(3)
    for _ in range(2000):
        assert barriers_exact(random_items(rng, rng.randint(1, 5)), 3)
    # within one item a gap never exceeds 3, so two would do
    for a in range(0, 10):
        for b in range(0, 10):
            qk, pv = consumer_slots([(a, b)])
            assert max_gap(qk) <= 3 and max_gap(pv) <= 3
    # across items the gap reaches 5: in an item (3, 3), K_B(2) (slot 7) is
    # followed by the last value tiles V_A(1), V_B(1), V_A(2), V_B(2) and
    # then by the next item's K_A(0) (slot 12, the third use of its stage)
    assert consumer_slots([(3, 3), (1, 1)])[0][5:7] == [7, 12]
    assert not barriers_exact([(3, 3), (1, 1)], 2)
    assert barriers_exact([(3, 3), (1, 1)], 3)


def test_records_name_the_previous_hand_off_of_the_pv_chain():
    """Replay: the QK warp's record for each S tile names the previous
    hand-off (block, parity of that block's hand-off count); the PV warp
    completes hand-offs in its (item, j, x) order, and hand-off k of block
    y completes phase k of that block's barrier.  The record must name the
    hand-off that the PV warp completed just before."""
    rng = random.Random(11)
    for _ in range(500):
        items = random_items(rng, rng.randint(1, 6))
        # QK warp: records
        count = [0, 0]
        prev = None
        records = []
        for nA, nB in items:
            for j in range(max(nA, nB)):
                for x in range(2):
                    if j < (nA, nB)[x]:
                        records.append(((x, count[x]), prev, j == 0, j == (nA, nB)[x] - 1))
                        prev = (x, count[x] & 1)
                        count[x] += 1
        # PV warp: the order in which hand-offs complete
        pv_order = []
        for nA, nB in items:
            for j in range(max(nA, nB)):
                for x in range(2):
                    if j < (nA, nB)[x]:
                        pv_order.append(x)
        seen = [0, 0]
        last = None
        for (x, k), rec_prev, first, last_tile in records:
            y = pv_order.pop(0)
            assert y == x  # the same order
            assert rec_prev == last
            assert k == seen[x]
            last = (x, seen[x] & 1)
            seen[x] += 1
        # first/last flags: one of each per block per item with tiles
        n_first = sum(1 for r in records if r[2])
        n_last = sum(1 for r in records if r[3])
        want = sum((nA > 0) + (nB > 0) for nA, nB in items)
        assert n_first == want and n_last == want
