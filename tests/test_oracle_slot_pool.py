"""Pins of the slot pool's admit policy (oracle/slot_pool.py), from cases
worked by hand and from invariants that any correct run must keep."""
import numpy as np
import pytest

from oracle.slot_pool import SlotPool


def holds(p: SlotPool):
    return {e: s for e, s in enumerate(p.slot_of) if s >= 0}


def test_an_empty_pool_fills_the_lowest_slots_in_expert_order():
    p = SlotPool(10, 4)
    assert p.admit([7, 2, 5, 2]) == (3, 0)          # three distinct misses, no hits
    assert holds(p) == {2: 0, 5: 1, 7: 2}
    assert p.expert_of == [2, 5, 7, -1]


def test_hits_keep_their_slots_and_a_miss_takes_an_empty_slot_first():
    p = SlotPool(10, 4)
    p.admit([7, 2, 5])
    # 2 is a hit; 9 misses: slot 3 is empty, so it goes there although slots
    # 1 and 2 were used longer ago
    assert p.admit([2, 9]) == (1, 1)
    assert holds(p) == {2: 0, 5: 1, 7: 2, 9: 3}
    assert p.stamp == [2, 1, 1, 2]


def test_a_full_pool_evicts_the_least_recently_used_ties_to_the_lower_slot():
    p = SlotPool(10, 4)
    p.admit([7, 2, 5])
    p.admit([2, 9])
    # slots 1 (expert 5) and 2 (expert 7) were both last used in batch 1:
    # the lower slot goes
    assert p.admit([4]) == (1, 0)
    assert holds(p) == {2: 0, 4: 1, 7: 2, 9: 3}
    assert p.slot_of[5] == -1


def test_an_expert_of_the_batch_is_never_evicted():
    p = SlotPool(10, 4)
    p.admit([7, 2, 5])
    p.admit([2, 9])
    p.admit([4])
    # 7 holds the oldest slot, but it is in this batch: the miss (5) takes
    # the oldest slot among the others (slot 0, expert 2, ties with slot 3)
    assert p.admit([7, 5]) == (1, 1)
    assert holds(p) == {5: 0, 4: 1, 7: 2, 9: 3}


def test_the_batch_must_fit_and_ids_must_be_in_range():
    p = SlotPool(8, 2)
    with pytest.raises(ValueError):
        p.admit([0, 1, 2])
    with pytest.raises(ValueError):
        p.admit([8])
    with pytest.raises(ValueError):
        SlotPool(8, 0)


def test_a_pool_that_holds_every_expert_fetches_each_one_once():
    rng = np.random.default_rng(3)
    E = 12
    p = SlotPool(E, E)
    seen, fetched = set(), 0
    for _ in range(40):
        batch = rng.choice(E, size=int(rng.integers(1, 6)), replace=False)
        m, h = p.admit(batch)
        fetched += m
        seen |= set(batch.tolist())
        assert fetched == len(seen)


def test_invariants_over_a_random_skewed_sequence():
    rng = np.random.default_rng(7)
    E, n = 40, 16
    p = SlotPool(E, n)
    weights = 1.0 / np.arange(1, E + 1) ** 1.1
    weights /= weights.sum()
    for _ in range(200):
        batch = np.unique(rng.choice(E, size=int(rng.integers(1, 12)), p=weights))
        before = dict(holds(p))
        m, h = p.admit(batch)
        # hits are the batch's experts that were resident; every other one is fetched
        assert h == sum(1 for e in batch if e in before)
        assert m == len(batch) - h
        now = holds(p)
        # every expert of the batch is resident, and the resident ones kept their slots
        assert all(e in now for e in batch)
        assert all(now[e] == before[e] for e in batch if e in before)
        # slot_of and expert_of are inverse maps
        for s, e in enumerate(p.expert_of):
            if e >= 0:
                assert p.slot_of[e] == s
        assert len(now) == sum(1 for e in p.expert_of if e >= 0) <= n
        # the batch's slots carry this batch's clock
        assert all(p.stamp[now[e]] == p.clock for e in batch)
