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

HIT, MISS, EVICT, MOVE, PREFETCH = 0, 1, 2, 3, 4


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


class PrefetchingLRUCache(LRUCache):
    """The global LRU with decode-time next-layer prefetch.

    Pages: the engine preloads the experts the coming tokens are likely to
    use, judged from their activation patterns (world.tibi.club, "Cum
    reușește FreeToken să ruleze 753B pe un singur GPU?", predictive
    scheduling; low-reliability page), and the shared LRU exploits the
    overlap of adjacent tokens' expert paths (aipolix.com, paragraph on
    semantic-aware caching).  The pages give no rule; the reading used here:

    * every step adds 1 to the count of each expert of its set S at its layer;
    * after the step at layer l, the next layer n = (l + 1) mod n_layers gets
      up to ``per_layer`` prefetches: its experts selected at least once,
      ranked by count (descending, ties to the lower id), resident ones
      skipped; each is inserted like a miss (evicting, when full, the least
      recent key that is neither in the step's S at layer l nor of layer n,
      else the lowest free slot) and recorded as PREFETCH;
    * a later HIT on a prefetched key counts as a prefetch hit (once).
    """

    def __init__(self, capacity: int, n_layers: int, n_experts: int, per_layer: int):
        super().__init__(capacity)
        self.n_layers, self.n_experts, self.per_layer = n_layers, n_experts, per_layer
        self.count = [[0] * n_experts for _ in range(n_layers)]
        self.unused = set()
        self.prefetches = 0
        self.prefetch_hits = 0

    def step(self, layer, experts) -> list[tuple]:
        ev = super().step(layer, experts)
        S = sorted(set(int(e) for e in experts))
        for kind, l, e, _, _ in ev:
            if kind == HIT and (l, e) in self.unused:
                self.unused.discard((l, e))
                self.prefetch_hits += 1
            if kind == EVICT:
                self.unused.discard((l, e))
        for e in S:
            self.count[layer][e] += 1
        if self.per_layer <= 0:
            return ev
        n = (layer + 1) % self.n_layers
        keep = {(layer, e) for e in S}
        ranked = sorted((e for e in range(self.n_experts) if self.count[n][e] > 0),
                        key=lambda e: (-self.count[n][e], e))
        done = 0
        for e in ranked:
            if done >= self.per_layer:
                break
            key = (n, e)
            if key in self.slot:
                continue
            if len(self.order) == self.capacity:
                cands = [k for k in self.order if k not in keep and k[0] != n]
                if not cands:
                    break
                victim = cands[0]
                self.order.remove(victim)
                s = self.slot.pop(victim)
                self.unused.discard(victim)
                ev.append((EVICT, victim[0], victim[1], s, -1))
            else:
                s = min(self._free_slots())
            self.slot[key] = s
            self.order.append(key)
            self.unused.add(key)
            self.prefetches += 1
            ev.append((PREFETCH, n, e, s, -1))
            done += 1
        return ev

    def resize(self, capacity: int) -> list[tuple]:
        ev = super().resize(capacity)
        for kind, l, e, _, _ in ev:
            if kind == EVICT:
                self.unused.discard((l, e))
        return ev
