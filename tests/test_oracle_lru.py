"""Pins of the oracle's global LRU expert-slot pool.

The reference is a textbook move-to-front list LRU over (layer, expert) keys, fed
the same per-step order (unique experts ascending; hits touched first, then the
misses).  It knows nothing of slots or clocks; slot reuse is checked against it.
"""
from collections import OrderedDict

import numpy as np
import pytest


class ListLRU:
    def __init__(self, capacity):
        self.cap = capacity
        self.order = OrderedDict()       # least recent first

    def step(self, keys):
        hits = [q for q in keys if q in self.order]
        misses = [q for q in keys if q not in self.order]
        for q in hits:
            self.order.move_to_end(q)
        pinned = set(keys)
        victims = []
        for q in misses:
            if len(self.order) >= self.cap:
                victim = next(v for v in self.order if v not in pinned)
                del self.order[victim]
                victims.append(victim)
            else:
                victims.append(-1)
            self.order[q] = True
        return hits, misses, victims


def _trace(rng, steps, L, E, T, k, skew):
    p = 1.0 / np.arange(1, E + 1) ** skew
    p /= p.sum()
    for s in range(steps):
        layer = s % L
        idx = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
        yield layer, idx


@pytest.mark.parametrize("S,L,E,T,k,skew", [(6, 1, 16, 2, 2, 0.0), (20, 3, 32, 4, 3, 1.0),
                                             (64, 4, 64, 8, 8, 0.7), (9, 2, 8, 1, 8, 0.0)])
def test_lru_matches_list_lru(orc, S, L, E, T, k, skew):
    rng = np.random.default_rng(S * 7 + E)
    pool = orc.LRU(S, L, E)
    ref = ListLRU(S)
    slot_of_key = {}
    for layer, idx in _trace(rng, 200, L, E, T, k, skew):
        r = pool.step(layer, idx)
        uniq = sorted(set(idx.ravel().tolist()))
        assert r["uniq"].tolist() == uniq
        keys = [layer * E + e for e in uniq]
        hits, misses, victims = ref.step(keys)
        assert [layer * E + e for e, h in zip(r["uniq"], r["hit"]) if h] == hits
        assert [layer * E + e for e in r["miss_expert"]] == misses
        assert r["evicted"].tolist() == victims
        # a victim's slot is reused by the miss that evicted it; a fresh slot is the lowest free
        st = pool.state()
        for e, s, v in zip(r["miss_expert"], r["miss_slot"], r["evicted"]):
            if v >= 0:
                assert slot_of_key.pop(v) == s
            slot_of_key[layer * E + e] = s
        for q, s in slot_of_key.items():
            assert st["slot_key"][s] == q and st["key_slot"][q] == s
        # every chosen expert maps to the slot now holding it
        for t in range(idx.shape[0]):
            for j in range(idx.shape[1]):
                assert st["slot_key"][r["slot_of"][t, j]] == layer * E + idx[t, j]
        occupied = st["slot_key"][st["slot_key"] >= 0]
        assert len(set(occupied.tolist())) == len(occupied) <= S
        assert len(r["uniq"]) == int(r["hit"].sum()) + len(r["miss_expert"])


def test_lru_free_slots_fill_in_index_order_and_clocks(orc):
    pool = orc.LRU(4, 1, 8)
    r = pool.step(0, np.array([[5, 2]], np.int32))
    assert r["miss_slot"].tolist() == [0, 1] and r["miss_expert"].tolist() == [2, 5]
    r = pool.step(0, np.array([[5, 7]], np.int32))       # hit 5 (clock 3), miss 7 -> slot 2 (clock 4)
    st = pool.state()
    assert st["slot_clock"].tolist() == [1, 3, 4, 0] and st["clock"] == 4
    r = pool.step(0, np.array([[1, 3]], np.int32))       # 1 -> free slot 3, 3 evicts expert 2 (clock 1)
    assert r["miss_slot"].tolist() == [3, 0] and r["evicted"].tolist() == [-1, 2]


def test_lru_pinned_entries_never_evicted(orc):
    pool = orc.LRU(3, 1, 8)
    pool.step(0, np.array([[0, 1, 2]], np.int32))
    r = pool.step(0, np.array([[0, 3, 4]], np.int32))    # 0 hit and pinned; 3, 4 evict 1, 2
    assert r["evicted"].tolist() == [1, 2]


def test_lru_rejects_pool_smaller_than_step(orc):
    pool = orc.LRU(2, 1, 8)
    with pytest.raises(ValueError):
        pool.step(0, np.array([[0, 1, 2]], np.int32))


def _list_resize(ref, n_new):
    """Textbook resize of a list LRU: keep the n_new most recently used keys."""
    while len(ref.order) > n_new:
        ref.order.popitem(last=False)
    ref.cap = n_new


@pytest.mark.parametrize("sizes", [(12, 5, 9, 3, 16), (20, 20, 7, 30), (8, 1, 8)])
def test_lru_resize_matches_list_lru(orc, sizes):
    """Resizing keeps the most recently used entries and the LRU order: the slot pool
    then behaves step for step like a list LRU truncated to its n most recent keys."""
    L, E, T, k = 2, 24, 1, 1 if min(sizes) < 3 else 3
    rng = np.random.default_rng(sum(sizes))
    pool = orc.LRU(sizes[0], L, E)
    ref = ListLRU(sizes[0])
    trace = list(_trace(rng, 60 * len(sizes), L, E, T, k, 0.6))
    for phase, n in enumerate(sizes):
        if phase:
            before = list(ref.order)
            ev = pool.resize(n)
            _list_resize(ref, n)
            assert ev == len(before) - len(ref.order)
            st = pool.state()
            resident = sorted(q for q in st["slot_key"].tolist() if q >= 0)
            assert resident == sorted(ref.order) and len(st["slot_key"]) == n
            # the clocks keep the list order of the survivors
            by_clock = [st["slot_key"][s] for s in np.argsort(st["slot_clock"]) if st["slot_key"][s] >= 0]
            assert by_clock == list(ref.order)
            for s, q in enumerate(st["slot_key"].tolist()):
                if q >= 0:
                    assert st["key_slot"][q] == s
        for layer, idx in trace[phase * 60:(phase + 1) * 60]:
            r = pool.step(layer, idx)
            keys = [layer * E + e for e in r["uniq"].tolist()]
            hits, misses, victims = ref.step(keys)
            assert [layer * E + e for e, h in zip(r["uniq"], r["hit"]) if h] == hits
            assert r["evicted"].tolist() == victims


def test_lru_resize_moves_survivors_to_lowest_free_slots(orc):
    pool = orc.LRU(6, 1, 8)
    for e in range(6):                                   # expert e in slot e, clock e + 1
        pool.step(0, np.array([[e]], np.int32))
    pool.step(0, np.array([[1]], np.int32))              # expert 1 -> clock 7 (most recent)
    assert pool.resize(3) == 3                           # evicts clocks 1, 3, 4: experts 0, 2, 3
    st = pool.state()
    # survivors 1 (slot 1), 4 (slot 4 -> 0), 5 (slot 5 -> 2)
    assert st["slot_key"].tolist() == [4, 1, 5]
    assert st["slot_clock"].tolist() == [5, 7, 6] and st["clock"] == 7
    assert pool.resize(5) == 0
    assert pool.state()["slot_key"].tolist() == [4, 1, 5, -1, -1]
    r = pool.step(0, np.array([[6]], np.int32))          # a fresh slot, the lowest free one
    assert r["miss_slot"].tolist() == [3] and r["evicted"].tolist() == [-1]
    with pytest.raises(ValueError):
        pool.resize(0)
