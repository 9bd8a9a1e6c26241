"""Expert cache oracle (LRU over HBM expert slots) -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU leg of ``bench.py``
may import this module.  Pure Python, one batch at a time.

What it follows: [EP-DS3] "MoE 推理架构深度实战：从 Expert Parallelism 到
DeepSeek-V3 的工程落地", section 3.2 (expert cache and preloading): inactive
experts live in host memory, the experts a batch needs are loaded into HBM, and
when HBM is full the least recently used resident expert is evicted first.

Readings (the sketch on the page leaves these open):
  * "Recently used" is counted in batches: every expert a batch routes at least
    one kept row to is stamped with that batch's number, hit or miss.  The
    page's access counter is never advanced in its sketch; a last-use stamp is
    the plain LRU reading.
  * An expert that the batch needs and that is already resident stays (it is
    counted once, not once as resident and once as a target).
  * Misses are filled in ascending expert order; each takes the resident slot
    with the oldest stamp among the slots this batch does not use, ties going to
    the lower slot index.  Empty slots carry stamp -1, so they fill first,
    lowest index first.
  * A batch that needs more distinct experts than there are slots is an error.

Pins (tests/test_cache_oracle.py): with one expert per batch the cache reduces
to textbook LRU (compared against an OrderedDict LRU), a hand-worked sequence,
and the LRU property of every eviction checked by brute force.
"""
from __future__ import annotations

from typing import Iterable, List, Tuple


class ExpertCacheOracle:
    def __init__(self, E: int, S: int):
        if not (1 <= S <= E):
            raise ValueError("need 1 <= slots <= experts")
        self.E, self.S = E, S
        self.slot_of = [-1] * E       # expert -> slot, -1 = in host memory only
        self.expert_in = [-1] * S     # slot -> expert, -1 = empty
        self.stamp = [-1] * S         # slot -> number of the batch that last used it
        self.step = 0
        self.hits = 0
        self.misses = 0

    def batch(self, needed: Iterable[int]) -> List[Tuple[int, int]]:
        """Make every expert in `needed` resident; return the loads [(expert, slot)] in order."""
        need = sorted(set(int(e) for e in needed))
        if len(need) > self.S:
            raise ValueError("batch needs more experts than the cache has slots")
        self.step += 1
        now = self.step
        missing = []
        for e in need:
            v = self.slot_of[e]
            if v >= 0:
                self.stamp[v] = now
                self.hits += 1
            else:
                missing.append(e)
        loads = []
        for e in missing:
            best = -1
            for v in range(self.S):          # oldest stamp among slots this batch does not use
                if self.stamp[v] < now and (best < 0 or self.stamp[v] < self.stamp[best]):
                    best = v
            old = self.expert_in[best]
            if old >= 0:
                self.slot_of[old] = -1
            self.expert_in[best] = e
            self.slot_of[e] = best
            self.stamp[best] = now
            self.misses += 1
            loads.append((e, best))
        return loads
