"""The expert-cache directory (host only, no GPU): which selected experts hit,
and which slot each miss takes.

Checked against a hand-worked sequence, against a plain model of the rule
(never-used slots lowest first, then the least recently used entry over all
layers, the touched entries becoming the most recent in call order), and
against a property every least-recently-used cache has whatever its
implementation: with more slots, a sequence never hits less (inclusion).
"""
import ctypes
from collections import OrderedDict

import numpy as np
import pytest

import bit_quantized_expert_router_b200 as F


class ModelLRU:
    """The rule, written out plainly: an ordered dict from (layer, expert) to
    slot, oldest first."""

    def __init__(self, n):
        self.n, self.od, self.free = n, OrderedDict(), list(range(n))
        self.hits = self.misses = self.evictions = 0

    def lookup(self, layer, idx):
        slots, miss = [], []
        for e in idx:
            key = (layer, int(e))
            if key in self.od:
                self.od.move_to_end(key)
                slots.append(self.od[key])
                miss.append(0)
                self.hits += 1
                continue
            if self.free:
                s = self.free.pop(0)
            else:
                _, s = self.od.popitem(last=False)
                self.evictions += 1
            self.od[key] = s
            slots.append(s)
            miss.append(1)
            self.misses += 1
        return slots, miss


def test_hand_worked_sequence():
    c = F.ExpertCache(3)
    # two free slots taken lowest first
    assert [a.tolist() for a in c.lookup(0, [5, 7])] == [[0, 1], [1, 1]]
    # 7 hits in slot 1; 9 takes the last free slot
    assert [a.tolist() for a in c.lookup(0, [7, 9])] == [[1, 2], [0, 1]]
    # another layer's expert 5 is a different entry: it evicts the least
    # recently used entry (layer 0, expert 5) in slot 0, then expert 1 evicts
    # (layer 0, expert 7) in slot 1
    assert [a.tolist() for a in c.lookup(1, [5, 1])] == [[0, 1], [1, 1]]
    # (layer 0, expert 9) survived
    assert [a.tolist() for a in c.lookup(0, [9])] == [[2], [0]]
    assert c.stats() == {"hits": 2, "misses": 5, "evictions": 2}


@pytest.mark.parametrize("n_slots,K,layers,experts", [(4, 4, 1, 16), (10, 4, 3, 32), (64, 8, 6, 128), (5, 1, 2, 9)])
def test_matches_the_rule_on_random_routing(n_slots, K, layers, experts):
    rng = np.random.default_rng(n_slots * 1000 + K)
    pop = 1.0 / np.arange(1, experts + 1) ** 1.1  # skewed expert popularity
    pop /= pop.sum()
    c, m = F.ExpertCache(n_slots), ModelLRU(n_slots)
    for step in range(400):
        layer = step % layers
        idx = rng.choice(experts, size=K, replace=False, p=pop)
        got_s, got_m = c.lookup(layer, idx)
        want_s, want_m = m.lookup(layer, idx)
        assert got_s.tolist() == want_s and got_m.tolist() == want_m, step
    assert c.stats() == {"hits": m.hits, "misses": m.misses, "evictions": m.evictions}
    # every slot in use holds exactly one entry
    assert len(set(m.od.values())) == len(m.od) <= n_slots


def test_matches_the_rule_at_scale():
    """Many slots, layers and evictions: the directory's fixed-size index
    (probe runs, entries removed from the middle of a run) keeps agreeing
    with the plain model."""
    n_slots, K, layers, experts = 1000, 4, 40, 512
    rng = np.random.default_rng(77)
    pop = 1.0 / np.arange(1, experts + 1) ** 0.9
    pop /= pop.sum()
    c, m = F.ExpertCache(n_slots), ModelLRU(n_slots)
    for step in range(6000):
        layer = step % layers
        idx = rng.choice(experts, size=K, replace=False, p=pop)
        got_s, got_m = c.lookup(layer, idx)
        want_s, want_m = m.lookup(layer, idx)
        assert got_s.tolist() == want_s and got_m.tolist() == want_m, step
    assert m.evictions > 10000
    assert c.stats() == {"hits": m.hits, "misses": m.misses, "evictions": m.evictions}


def test_inclusion_more_slots_never_hit_less():
    rng = np.random.default_rng(5)
    seq = [(s % 4, rng.choice(64, size=4, replace=False)) for s in range(600)]
    hits = []
    for n in (4, 8, 16, 32, 64, 128, 256):
        c = F.ExpertCache(n)
        for layer, idx in seq:
            c.lookup(layer, idx)
        hits.append(c.stats()["hits"])
    assert hits == sorted(hits)
    assert hits[-1] == 600 * 4 - len({(l, int(e)) for l, idx in seq for e in idx})  # only cold misses left


def test_working_set_that_fits_hits_after_the_first_pass():
    c = F.ExpertCache(12)
    calls = [(l, [3 * l, 3 * l + 1, 3 * l + 2]) for l in range(4)]  # 12 entries
    for l, idx in calls:
        assert c.lookup(l, idx)[1].tolist() == [1, 1, 1]
    for _ in range(3):
        for l, idx in calls:
            assert c.lookup(l, idx)[1].tolist() == [0, 0, 0]


def test_duplicate_expert_in_one_call_and_reset():
    c = F.ExpertCache(4)
    s, m = c.lookup(0, [2, 2, 3])
    assert s.tolist() == [0, 0, 1] and m.tolist() == [1, 0, 1]
    c.reset()
    assert c.stats() == {"hits": 0, "misses": 0, "evictions": 0}
    assert c.lookup(0, [3])[0].tolist() == [0]  # all slots free again


def test_invalid_arguments():
    L = F.lib()
    h = ctypes.c_void_p()
    assert L.fmoe_cache_create(0, ctypes.byref(h)) == F.FMOE_EINVAL
    assert L.fmoe_cache_create((1 << 20) + 1, ctypes.byref(h)) == F.FMOE_EINVAL
    assert L.fmoe_cache_create(4, None) == F.FMOE_EINVAL
    assert L.fmoe_cache_lookup(None, 0, None, 1, None, None, None) == F.FMOE_EINVAL
    assert L.fmoe_cache_stats(None, None, None, None) == F.FMOE_EINVAL
    assert L.fmoe_cache_reset(None) == F.FMOE_EINVAL
    assert L.fmoe_cache_destroy(None) == F.FMOE_OK
    c = F.ExpertCache(2)
    with pytest.raises(F.FmoeError):
        c.lookup(0, [1, 2, 3])  # K above the slot count
    with pytest.raises(F.FmoeError):
        c.lookup(0, [-1])
    with pytest.raises(F.FmoeError):
        c.lookup(-1, [0])
    assert c.stats() == {"hits": 0, "misses": 0, "evictions": 0}  # rejected calls change nothing
