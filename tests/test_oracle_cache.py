"""Pins of the slot-cache oracle (oracle/cache.py): hand-worked steps, the classic LRU
cache it reduces to for one whole expert per step, the closed form of a fully resident
cache, and invariants on random routing sequences."""
from collections import OrderedDict

import numpy as np
import pytest

from oracle.cache import SlotCache, fetched_planes, need_from_routing


def _flat(rounds):
    return [[(sv.expert, sv.slot, sv.lo, sv.hi) for sv in rnd] for rnd in rounds]


def test_hand_worked_bitplane_steps():
    c = SlotCache(E=4, S=2, P=8)
    # step 1: two misses into the free slots, prefixes of 3 and 2 planes
    assert _flat(c.plan([3, 0, 2, 0])) == [[(0, 0, 0, 3), (2, 1, 0, 2)]]
    # step 2: expert 0 extends from 3 to 5 planes; expert 3 evicts expert 2 (slot 1)
    assert _flat(c.plan([5, 0, 0, 1])) == [[(0, 0, 3, 5), (3, 1, 0, 1)]]
    # step 3: both slots last used at step 2, neither expert needed: the lower slot goes first
    assert _flat(c.plan([0, 4, 2, 0])) == [[(1, 0, 0, 4), (2, 1, 0, 2)]]
    # step 4: a narrower read of a resident expert fetches nothing
    assert _flat(c.plan([0, 1, 0, 0])) == [[(1, 0, 1, 1)]]


def test_rounds_when_a_step_needs_more_experts_than_slots():
    c = SlotCache(E=5, S=2, P=1)
    assert _flat(c.plan([1, 1, 1, 0, 1])) == [[(0, 0, 0, 1), (1, 1, 0, 1)], [(2, 0, 0, 1), (4, 1, 0, 1)]]


def test_victim_prefers_experts_not_needed_later_in_the_step():
    c = SlotCache(E=6, S=3, P=1)
    c.plan([0, 0, 0, 1, 1, 1])   # slots: 0 <- e3, 1 <- e4, 2 <- e5 (all last used at step 1)
    c.plan([0, 0, 0, 0, 0, 1])   # e5 refreshed (step 2)
    # step 3 serves e0 (a miss) before e3: slots 0 (e3) and 1 (e4) are equally old and
    # plain LRU would take slot 0, but e3 is needed later in the step, so e4 goes
    assert _flat(c.plan([1, 0, 0, 1, 0, 0])) == [[(0, 1, 0, 1), (3, 0, 1, 1)]]


def _textbook_lru_misses(seq, S):
    lru, misses = OrderedDict(), 0
    for e in seq:
        if e in lru:
            lru.move_to_end(e)
            continue
        misses += 1
        if len(lru) == S:
            lru.popitem(last=False)
        lru[e] = True
    return misses


@pytest.mark.parametrize("S", [1, 3, 7])
def test_one_expert_per_step_is_the_classic_lru_cache(S):
    rng = np.random.default_rng(S)
    seq = rng.integers(0, 12, size=400).tolist()
    c = SlotCache(E=12, S=S, P=1)
    misses = 0
    for e in seq:
        need = [0] * 12
        need[e] = 1
        rounds = c.plan(need)
        misses += fetched_planes(rounds)
    assert misses == _textbook_lru_misses(seq, S)


def test_fully_resident_cache_fetches_each_plane_once():
    # S = E: nothing is evicted, prefixes only grow: planes fetched = sum_e max need
    rng = np.random.default_rng(5)
    E, total, peak = 16, 0, np.zeros(16, int)
    c = SlotCache(E=E, S=E, P=8)
    for _ in range(60):
        need = (rng.integers(0, 9, size=E) * (rng.random(E) < 0.4)).tolist()
        total += fetched_planes(c.plan(need))
        peak = np.maximum(peak, need)
    assert total == int(peak.sum())


@pytest.mark.parametrize("E,S,P", [(8, 3, 8), (32, 8, 1), (64, 16, 8), (10, 10, 4)])
def test_invariants_on_random_steps(E, S, P):
    rng = np.random.default_rng(E * S + P)
    c = SlotCache(E=E, S=S, P=P)
    for _ in range(80):
        need = (rng.integers(1, P + 1, size=E) * (rng.random(E) < 0.3)).tolist()
        rounds = c.plan(need)
        served = [sv for rnd in rounds for sv in rnd]
        # every routed expert exactly once, in ascending id; nothing else
        assert [sv.expert for sv in served] == [e for e in range(E) if need[e] > 0]
        for rnd in rounds:
            assert 1 <= len(rnd) <= S
            assert len({sv.slot for sv in rnd}) == len(rnd)   # one slot per expert in a round
        for sv in served:
            assert 0 <= sv.lo <= sv.hi <= P
            assert sv.hi == need[sv.expert] or (sv.lo == sv.hi == need[sv.expert])
        # the state is one-to-one and holds every expert served in the last round
        for s, e in enumerate(c.expert_of):
            if e >= 0:
                assert c.slot_of[e] == s and 1 <= c.planes[s] <= P
        assert sum(1 for v in c.slot_of if v >= 0) == sum(1 for v in c.expert_of if v >= 0)
        for sv in rounds[-1] if rounds else []:
            assert c.slot_of[sv.expert] == sv.slot and c.planes[sv.slot] >= need[sv.expert]


def test_need_from_routing():
    offsets = np.array([0, 2, 2, 5])
    sorted_pair = np.array([4, 0, 1, 2, 5])
    bits = np.array([2, 8, 3, 4, 2, 3], np.uint8)
    assert need_from_routing(offsets, sorted_pair, bits, planes=8) == [2, 0, 8]
    assert need_from_routing(offsets, sorted_pair) == [1, 0, 1]
