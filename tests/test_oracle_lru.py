"""Pins of the LRU oracle against an independent timestamp simulation."""
import numpy as np
import pytest

from oracle import lru


class StampCache:
    """Same policy written differently: each key carries the time of its last
    use; the victim is the key with the smallest stamp outside the step's set;
    slots are the lowest free ones."""

    def __init__(self, cap):
        self.cap = cap
        self.stamp = {}
        self.slot = {}
        self.clock = 0

    def step(self, layer, experts):
        S = sorted(set(experts))
        if len(S) > self.cap:
            raise lru.NoSpace()
        ev = []
        for e in S:
            self.clock += 1
            key = (layer, e)
            if key in self.slot:
                self.stamp[key] = self.clock
                ev.append((lru.HIT, layer, e, self.slot[key], -1))
                continue
            if len(self.slot) >= self.cap:
                cands = [k for k in self.slot if not (k[0] == layer and k[1] in S)]
                v = min(cands, key=lambda k: self.stamp[k])
                s = self.slot.pop(v)
                del self.stamp[v]
                ev.append((lru.EVICT, v[0], v[1], s, -1))
            else:
                s = min(set(range(self.cap)) - set(self.slot.values()))
            self.slot[key] = s
            self.stamp[key] = self.clock
            ev.append((lru.MISS, layer, e, s, -1))
        return ev

    def resize(self, cap):
        ev = []
        while len(self.slot) > cap:
            v = min(self.slot, key=lambda k: self.stamp[k])
            ev.append((lru.EVICT, v[0], v[1], self.slot.pop(v), -1))
            del self.stamp[v]
        shrink = cap < self.cap
        self.cap = cap
        if shrink:
            for k in sorted(self.slot, key=lambda k: self.slot[k]):
                if self.slot[k] >= cap:
                    dst = min(set(range(cap)) - set(self.slot.values()))
                    ev.append((lru.MOVE, k[0], k[1], dst, self.slot[k]))
                    self.slot[k] = dst
        return ev


@pytest.mark.parametrize("seed", range(6))
def test_lru_matches_stamp_simulation(seed):
    rng = np.random.default_rng(seed)
    L, E, k = 4, 12, 3
    cap = int(rng.integers(k * 2, 20))
    a, b = lru.LRUCache(cap), StampCache(cap)
    for step in range(300):
        if step % 50 == 49:
            c = int(rng.integers(k + 1, 25))
            assert a.resize(c) == b.resize(c)
            continue
        layer = step % L
        ex = [int(e) for e in rng.choice(E, int(rng.integers(1, 2 * k)), replace=True)]
        if len(set(ex)) > a.capacity:
            with pytest.raises(lru.NoSpace):
                a.step(layer, ex)
            continue
        assert a.step(layer, ex) == b.step(layer, ex)


def test_lru_hand_trace():
    c = lru.LRUCache(3)
    H, M, X, V = lru.HIT, lru.MISS, lru.EVICT, lru.MOVE
    assert c.step(0, [5, 2]) == [(M, 0, 2, 0, -1), (M, 0, 5, 1, -1)]
    assert c.step(1, [2]) == [(M, 1, 2, 2, -1)]
    # full; (0,2) is least recent but (0,5) is also old: S = {5, 9} keeps (0,5)
    assert c.step(0, [9, 5]) == [(H, 0, 5, 1, -1), (X, 0, 2, 0, -1), (M, 0, 9, 0, -1)]
    # shrink to 1: evict (1,2) then (0,5); (0,9) stays in slot 0
    assert c.resize(1) == [(X, 1, 2, 2, -1), (X, 0, 5, 1, -1)]
    assert c.resize(3) == []
    assert c.step(2, [0, 1]) == [(M, 2, 0, 1, -1), (M, 2, 1, 2, -1)]
    # shrink to 2 keeps the two most recent, moves slot 2 down to slot 0
    assert c.resize(2) == [(X, 0, 9, 0, -1), (V, 2, 1, 0, 2)]
    with pytest.raises(lru.NoSpace):
        c.step(3, [1, 2, 3])


def test_lru_all_hits_when_everything_fits():
    rng = np.random.default_rng(9)
    c = lru.LRUCache(64)
    seen = set()
    for step in range(400):
        layer = step % 4
        ex = rng.choice(16, 4, replace=False)
        for kind, l, e, s, _ in c.step(layer, ex):
            if (l, e) in seen:
                assert kind == lru.HIT
            else:
                assert kind == lru.MISS
            seen.add((l, e))


def test_lookup_touches_a_hit_and_leaves_a_miss_alone():
    """A lookup hit makes the key most recent, which changes the next victim;
    a lookup miss returns -1 and changes nothing."""
    c = lru.LRUCache(2)
    c.step(0, [1])
    c.step(0, [2])                                   # recency: (0,1) then (0,2)
    assert c.lookup(0, 1) == 0                       # (0,1) becomes most recent
    assert c.lookup(0, 7) == -1
    ev = c.step(0, [3])
    assert ev == [(lru.EVICT, 0, 2, 1, -1), (lru.MISS, 0, 3, 1, -1)]
    d = lru.LRUCache(2)
    d.step(0, [1])
    d.step(0, [2])
    assert d.step(0, [3]) == [(lru.EVICT, 0, 1, 0, -1), (lru.MISS, 0, 3, 0, -1)]   # without the lookup


def test_prefetch_hand_sequence():
    """Capacity 6, 3 layers, 8 experts, one prefetch per step, worked by hand
    from the stated rule (counts of each layer's selections; after a step at
    layer l, the most-counted non-resident expert of layer l+1 is inserted,
    evicting the least recent key outside the step's set and outside layer
    l+1)."""
    H_, M_, E_, P_ = lru.HIT, lru.MISS, lru.EVICT, lru.PREFETCH
    c = lru.PrefetchingLRUCache(6, 3, 8, 1)
    assert c.step(0, [1, 2]) == [(M_, 0, 1, 0, -1), (M_, 0, 2, 1, -1)]      # layer 1 has no counts yet
    assert c.step(1, [3]) == [(M_, 1, 3, 2, -1)]
    assert c.step(2, [1]) == [(M_, 2, 1, 3, -1)]                             # layer 0's counted experts resident
    assert c.step(0, [1, 5]) == [(H_, 0, 1, 0, -1), (M_, 0, 5, 4, -1)]
    assert c.step(1, [3, 4]) == [(H_, 1, 3, 2, -1), (M_, 1, 4, 5, -1)]      # now full
    # (2,6) evicts the least recent (0,2); then layer 0's counts 1:2, 2:1, 5:1
    # pick (0,2), evicting the least recent key outside {(2,1),(2,6)} and layer 0: (1,3)
    assert c.step(2, [1, 6]) == [(H_, 2, 1, 3, -1), (E_, 0, 2, 1, -1), (M_, 2, 6, 1, -1),
                                 (E_, 1, 3, 2, -1), (P_, 0, 2, 2, -1)]
    # (0,2) is a prefetch hit; layer 1's counts 3:2, 4:1 pick (1,3), evicting (0,1)
    assert c.step(0, [2, 5]) == [(H_, 0, 2, 2, -1), (H_, 0, 5, 4, -1), (E_, 0, 1, 0, -1), (P_, 1, 3, 0, -1)]
    assert c.prefetches == 2 and c.prefetch_hits == 1
    # (1,3) is the second prefetch hit; layer 2's counted experts 1, 6 are resident
    assert c.step(1, [3]) == [(H_, 1, 3, 0, -1)]
    assert c.prefetch_hits == 2


def test_prefetch_off_is_the_plain_lru_and_counts_are_consistent():
    import numpy as np
    rng = np.random.default_rng(11)
    a, b = lru.LRUCache(10), lru.PrefetchingLRUCache(10, 4, 16, 0)
    p = lru.PrefetchingLRUCache(10, 4, 16, 2)
    for step in range(300):
        if step == 120:
            assert a.resize(5) == b.resize(5)
            p.resize(5)
        if step == 200:
            assert a.resize(10) == b.resize(10)
            p.resize(10)
        layer = step % 4
        e = rng.choice(16, 2, replace=False)
        assert a.step(layer, e) == b.step(layer, e)
        ev = p.step(layer, e)
        # a prefetch never evicts the step's own keys nor keys of the layer it fills
        pf = [x for x in ev if x[0] == lru.PREFETCH]
        for x in ev:
            if x[0] == lru.EVICT and pf:
                assert (x[1], x[2]) not in {(layer, int(v)) for v in e}
        assert len(p.slot) <= p.capacity
    assert b.prefetches == 0 and 0 < p.prefetch_hits <= p.prefetches
