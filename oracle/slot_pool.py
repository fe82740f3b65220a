"""The expert slot pool's admit policy, written out on the host.

TEST INFRASTRUCTURE ONLY: the GPU tests of the cached forward compare the
library's slot pool against this model.  Nothing here is imported by the
library, and nothing of the library is imported here.

The pages name an expert "slot pool" indexed per expert (atomicmilkshake/
FreeToken fork README, "Known limits") and a "global LRU expert cache"
(FreeToken upstream README, "About"), but give no policy.  The reading
followed here:

* the experts of a batch that already hold a slot are hits; their slots are
  stamped with the batch's clock;
* every other expert of the batch (a miss), taken in increasing expert
  order, gets the next slot in the order "empty slots first, then the least
  recently used (smallest stamp), ties to the lower slot index", among the
  slots that no expert of this batch holds;
* the evicted expert, if any, no longer holds a slot; the new one is stamped;
* a batch must fit: the pool has at least as many slots as the batch has
  distinct experts.
"""
from __future__ import annotations


class SlotPool:
    """Which expert each of n slots holds, for a bank of E experts."""

    def __init__(self, E: int, n: int):
        if E < 1 or n < 1:
            raise ValueError("E and n must be positive")
        self.E, self.n = E, n
        self.slot_of = [-1] * E      # expert -> slot, -1 when not resident
        self.expert_of = [-1] * n    # slot -> expert, -1 when empty
        self.stamp = [0] * n         # clock of the slot's last use
        self.clock = 0

    def admit(self, experts) -> tuple[int, int]:
        """Admits one batch's experts; returns (misses, hits)."""
        active = sorted(set(int(e) for e in experts))
        if any(e < 0 or e >= self.E for e in active):
            raise ValueError("expert id out of range")
        if len(active) > self.n:
            raise ValueError("the batch does not fit in the pool")
        self.clock += 1
        hits = 0
        for s, e in enumerate(self.expert_of):
            if e >= 0 and e in active:
                self.stamp[s] = self.clock
                hits += 1
        # candidate slots: those no expert of this batch holds, empty first
        # (key 0), then by last use (stamp + 1), ties to the lower slot
        candidates = sorted((0 if e < 0 else self.stamp[s] + 1, s)
                            for s, e in enumerate(self.expert_of) if not (e >= 0 and e in active))
        misses = [e for e in active if self.slot_of[e] < 0]
        for r, e in enumerate(misses):
            s = candidates[r][1]
            old = self.expert_of[s]
            if old >= 0:
                self.slot_of[old] = -1
            self.expert_of[s] = e
            self.slot_of[e] = s
            self.stamp[s] = self.clock
        return len(misses), hits
