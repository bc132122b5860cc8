"""Plain model of the expert slot pool's policy.

TEST INFRASTRUCTURE ONLY (imported by the test suite): the CUDA library's
pool is checked against it decision by decision.

What it follows: "Red Metal dev8 -- resident routed top-k layer", steps
1-3 (a hard-bounded LRU makes every selected expert resident; the selected
experts are protected from eviction while the remaining misses are filled;
every selected slot is pinned for the work that uses it) and "Red Lite dev9
-- native runtime foundation", section "Native selftest" (hard capacity,
LRU hit/miss/eviction, protection of the current top-k during
acquire_many, in-flight slot protection).  Readings where the pages are
silent: a free slot is taken before anything is evicted, the lowest free
slot first; hits are refreshed in selection order before the misses, which
are refreshed in selection order as they are filled; a repeated id is one
expert; a selection that cannot be placed because every candidate slot is
in flight changes nothing and is reported as 'again'."""

from __future__ import annotations

OK, EINVAL, ENOMEM, EAGAIN = 0, -1, -3, -5


class LruModel:
    def __init__(self, n_experts: int, capacity: int):
        self.n_experts = n_experts
        self.capacity = capacity
        self.slot_expert = [-1] * capacity  # expert held by each slot
        self.expert_slot = {}  # expert -> slot
        self.last_use = [0] * capacity  # recency clock of each slot
        self.pins = [0] * capacity  # in-flight selections holding each slot
        self.tick = 0
        self.inflight = {}  # token -> slots
        self.next_token = 1

    def _touch(self, slot):
        self.tick += 1
        self.last_use[slot] = self.tick

    def plan(self, ids):
        """Returns (rc, slots, evicted, miss, token) like the library's plan."""
        if any(not 0 <= e < self.n_experts for e in ids):
            return EINVAL, None, None, None, 0
        if len(set(ids)) > self.capacity:
            return ENOMEM, None, None, None, 0
        hits = [e in self.expert_slot for e in ids]
        protected = {self.expert_slot[e] for e in ids if e in self.expert_slot}
        # choose a slot for every distinct missing expert, in selection order
        chosen, victims = set(), {}
        for e, hit in zip(ids, hits):
            if hit or e in victims:
                continue
            free = [s for s in range(self.capacity) if self.slot_expert[s] < 0 and s not in chosen]
            if free:
                s = min(free)
            else:
                cands = [s for s in range(self.capacity)
                         if s not in protected and s not in chosen and self.pins[s] == 0]
                if not cands:
                    return EAGAIN, None, None, None, 0
                s = min(cands, key=lambda c: self.last_use[c])
            chosen.add(s)
            victims[e] = s
        # commit
        slots, evicted, miss = [None] * len(ids), [-1] * len(ids), [False] * len(ids)
        for i, (e, hit) in enumerate(zip(ids, hits)):
            if hit:
                slots[i] = self.expert_slot[e]
                self._touch(slots[i])
        for i, (e, hit) in enumerate(zip(ids, hits)):
            if hit:
                continue
            if e in self.expert_slot:  # repeated id, filled by its first occurrence
                slots[i] = self.expert_slot[e]
                continue
            s = victims[e]
            old = self.slot_expert[s]
            if old >= 0:
                del self.expert_slot[old]
            evicted[i] = old
            self.slot_expert[s] = e
            self.expert_slot[e] = s
            self._touch(s)
            slots[i] = s
            miss[i] = True
        token = self.next_token
        self.next_token += 1
        held = sorted(set(slots))
        for s in held:
            self.pins[s] += 1
        self.inflight[token] = held
        return OK, slots, evicted, miss, token

    def complete(self, token):
        if token not in self.inflight:
            return EINVAL
        for s in self.inflight.pop(token):
            self.pins[s] -= 1
        return OK
