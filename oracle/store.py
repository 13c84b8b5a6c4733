"""Plain model of the tiered page store's residency policy (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` may
use this module.

Source: "WorldAttention pairs hierarchical KV caching with hybrid sparse attention
..." (news summary), HKV paragraph: KV pages are kept in a hierarchy of memories
ranked by cost, pages that are not selected are demoted to cheaper memory so that
GPU occupancy stays bounded; WorldAttention project page, Method figure
"three-tier hierarchical KV cache".  The pages fix no replacement rule; the
reading taken (least recently used, ties to the lower slot, a free slot first,
the lowest first) is written out below step by step.

State: slot_of_page[p] (-1 = only on the host tier), page_of_slot[s] (-1 = free),
stamp[s] (tick of the slot's last use), tick (one per fetch / prefetch call).
"""
from __future__ import annotations

import math


class PageStoreModel:
    def __init__(self, NP: int, S: int):
        self.NP, self.S = NP, S
        self.slot_of_page = [-1] * NP
        self.page_of_slot = [-1] * S
        self.stamp = [0] * S
        self.tick = 0
        self.errors = 0

    def _victim(self, evictable):
        """The lowest free slot; else the least recently used evictable slot (ties -> lower slot)."""
        for s in range(self.S):
            if self.page_of_slot[s] < 0:
                return s
        cands = [s for s in range(self.S) if evictable(s)]
        if not cands:
            return -1
        return min(cands, key=lambda s: (self.stamp[s], s))

    def _assign(self, p, s, copies):
        q = self.page_of_slot[s]
        if q >= 0:
            self.slot_of_page[q] = -1  # demoted: read from the host tier again
        self.page_of_slot[s] = p
        self.slot_of_page[p] = s
        self.stamp[s] = self.tick
        copies.append((p, s))

    def fetch(self, sel):
        """Make the selected pages resident.  Returns the (page, slot) copies made."""
        self.tick += 1
        copies = []
        for p in sel:
            if 0 <= p < self.NP and self.slot_of_page[p] >= 0:
                self.stamp[self.slot_of_page[p]] = self.tick
            elif not 0 <= p < self.NP:
                self.errors += 1
        for p in sel:
            if not 0 <= p < self.NP or self.slot_of_page[p] >= 0:
                continue
            s = self._victim(lambda s: self.stamp[s] < self.tick)
            if s < 0:
                self.errors += 1
                continue
            self._assign(p, s, copies)
        return copies

    def prefetch(self, scores, protect, m):
        """Make the m best-scoring unprotected pages with a finite score resident, in
        score order (ties -> lower page), never evicting a protected page or one made
        resident by this call.  Returns the copies made."""
        self.tick += 1
        protect = set(int(p) for p in protect)
        ranked = sorted((p for p in range(self.NP) if math.isfinite(scores[p]) and p not in protect),
                        key=lambda p: (-scores[p], p))
        copies = []
        for p in ranked[:m]:
            if self.slot_of_page[p] >= 0:
                self.stamp[self.slot_of_page[p]] = self.tick
                continue
            s = self._victim(lambda s: self.stamp[s] < self.tick and self.page_of_slot[s] not in protect)
            if s < 0:
                break
            self._assign(p, s, copies)
        return copies
