"""Pins of the page-store residency model (oracle/store.py): hand-worked sequences and
invariants of the policy (bounded occupancy, selected pages resident, least recently
used eviction, protection during prefetch)."""
import math

import numpy as np

from oracle.store import PageStoreModel


def test_hand_worked_sequence():
    m = PageStoreModel(NP=6, S=3)
    assert m.fetch([0, 2]) == [(0, 0), (2, 1)]            # free slots, lowest first
    assert m.fetch([2, 5]) == [(5, 2)]                    # 2 resident (touched), 5 takes the last free slot
    # slots: 0 <- page 0 (tick 1), 1 <- page 2 (tick 2), 2 <- page 5 (tick 2)
    assert m.fetch([1, 2]) == [(1, 0)]                    # LRU unselected slot is 0 (page 0, tick 1)
    assert m.slot_of_page == [-1, 0, 1, -1, -1, 2]
    # ties of the LRU stamp go to the lower slot: slots 1 and 2 both last used at tick 3 / 2
    assert m.fetch([3]) == [(3, 2)]                       # stamps: s0=3 (page 1), s1=3 (page 2), s2=2 (page 5)
    assert m.page_of_slot == [1, 2, 3]
    assert m.fetch([4]) == [(4, 0)]                       # s0 and s1 tie at 3 -> lower slot 0
    assert m.errors == 0


def test_prefetch_order_protection_and_stop():
    m = PageStoreModel(NP=8, S=4)
    m.fetch([1, 6])                                       # slots 0, 1
    scores = [0.5, 9.0, 3.0, 3.0, -math.inf, 7.0, 8.0, 1.0]
    # protected: the current selection {1, 6}; best others: 5 (7.0), 2 and 3 tie (3.0 -> page 2 first)
    assert m.prefetch(scores, [1, 6], 3) == [(5, 2), (2, 3)]  # slots full after two: 3 cannot evict 1, 6, 5 or 2
    assert m.page_of_slot == [1, 6, 5, 2]
    # a later fetch of page 3 evicts the least recently used unselected slot: pages 1 / 6 (tick 1)
    assert m.fetch([3]) == [(3, 0)]
    # non-finite scores are never prefetched
    assert all(p != 4 for p, _ in m.prefetch(scores, [], 8))


def test_invariants_random_sequences():
    rng = np.random.default_rng(3)
    for trial in range(200):
        NP, S = int(rng.integers(2, 20)), int(rng.integers(1, 8))
        m = PageStoreModel(NP, S)
        for step in range(30):
            if rng.random() < 0.7:
                Kp = int(rng.integers(1, min(NP, S) + 1))
                sel = sorted(rng.choice(NP, Kp, replace=False).tolist())
                before = dict(enumerate(m.page_of_slot))
                copies = m.fetch(sel)
                # every selected page is resident, in a distinct slot
                assert all(m.slot_of_page[p] >= 0 for p in sel)
                # copies are exactly the selected pages that were not resident before
                assert sorted(p for p, _ in copies) == sorted(p for p in sel if p not in before.values())
            else:
                scores = rng.normal(size=NP)
                scores[rng.random(NP) < 0.2] = -np.inf
                protect = [p for p in range(NP) if m.slot_of_page[p] >= 0 and rng.random() < 0.5]
                resident_protected = [p for p in protect if m.slot_of_page[p] >= 0]
                m.prefetch(scores, protect, int(rng.integers(0, S + 2)))
                assert all(m.slot_of_page[p] >= 0 for p in resident_protected)
            # the two maps are inverse and occupancy is bounded by S
            occ = [p for p in m.page_of_slot if p >= 0]
            assert len(occ) == len(set(occ)) <= S
            for s, p in enumerate(m.page_of_slot):
                if p >= 0:
                    assert m.slot_of_page[p] == s
            assert sum(1 for s in m.slot_of_page if s >= 0) == len(occ)
