"""Global LRU expert cache across MoE layers, with live resize.

Test infrastructure only (see the package header).

Pages: during decoding one global LRU cache spans all MoE layers instead of
pinning experts in VRAM at start-up (jansverre.net page, section "Hvorfor er
båndbredden viktigere enn antall kjerner?"); the shared LRU exploits the
overlap of expert paths between adjacent tokens (aipolix.com page, paragraph on
semantic-aware caching); the GPU expert cache can be resized without
restarting the engine or reloading the host-resident pool (aipolix.com page,
paragraph on elastic memory management).

Readings (the pages give no finer rule):
* key = (layer, expert); capacity C = floor(budget / blob stride) slots;
* per layer step, S = the distinct selected experts of the batch in ascending
  id; each is looked up in that order: a hit moves the key to most-recent; a
  miss, when the cache is full, first evicts the least-recent key that is not
  in S, then inserts the key as most-recent into the victim's slot, or else
  into the lowest free slot; |S| > C is an error;
* shrink to C': evict from the least-recent end until at most C' keys remain,
  then move every survivor whose slot is >= C', in ascending slot order, to the
  lowest free slot below C'; recency order is unchanged; grow only raises C.

Events are tuples (kind, layer, expert, slot, from_slot) with kind one of
HIT, MISS, EVICT, MOVE; from_slot is the old slot for MOVE and -1 otherwise.
"""
from __future__ import annotations

HIT, MISS, EVICT, MOVE = 0, 1, 2, 3


class NoSpace(Exception):
    pass


class LRUCache:
    def __init__(self, capacity: int):
        self.capacity = int(capacity)
        self.order: list[tuple[int, int]] = []      # least recent first
        self.slot: dict[tuple[int, int], int] = {}

    def _free_slots(self) -> list[int]:
        used = set(self.slot.values())
        return [s for s in range(self.capacity) if s not in used]

    def step(self, layer: int, experts) -> list[tuple]:
        S = sorted(set(int(e) for e in experts))
        if len(S) > self.capacity:
            raise NoSpace(f"{len(S)} experts > capacity {self.capacity}")
        in_S = {(layer, e) for e in S}
        ev = []
        for e in S:
            key = (layer, e)
            if key in self.slot:
                self.order.remove(key)
                self.order.append(key)
                ev.append((HIT, layer, e, self.slot[key], -1))
                continue
            if len(self.order) == self.capacity:
                victim = next(k for k in self.order if k not in in_S)
                self.order.remove(victim)
                s = self.slot.pop(victim)
                ev.append((EVICT, victim[0], victim[1], s, -1))
            else:
                s = min(self._free_slots())
            self.slot[key] = s
            self.order.append(key)
            ev.append((MISS, layer, e, s, -1))
        return ev

    def resize(self, capacity: int) -> list[tuple]:
        capacity = int(capacity)
        if capacity < 0:
            raise NoSpace("negative capacity")
        ev = []
        while len(self.order) > capacity:
            victim = self.order.pop(0)
            s = self.slot.pop(victim)
            ev.append((EVICT, victim[0], victim[1], s, -1))
        old_cap = self.capacity
        self.capacity = capacity
        if capacity < old_cap:
            movers = sorted((s, k) for k, s in self.slot.items() if s >= capacity)
            for s, k in movers:
                dst = min(self._free_slots())
                self.slot[k] = dst
                ev.append((MOVE, k[0], k[1], dst, s))
        return ev

    def lookup(self, layer: int, expert: int) -> int:
        """Slot of a key (touching it) or -1."""
        key = (layer, int(expert))
        if key not in self.slot:
            return -1
        self.order.remove(key)
        self.order.append(key)
        return self.slot[key]
