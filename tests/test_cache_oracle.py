"""Pins for the expert cache oracle (LRU over HBM expert slots).

Each pin ties the oracle to something other than itself: the textbook LRU it
must reduce to, a sequence worked by hand, and the LRU property of every
eviction checked by brute force over the whole history.
"""
from collections import OrderedDict

import numpy as np
import pytest

from oracle.expert_cache import ExpertCacheOracle


def textbook_lru(seq, S):
    """Classic LRU over single references: -> list of hit flags, list of resident sets."""
    cache = OrderedDict()
    hits, sets = [], []
    for e in seq:
        if e in cache:
            cache.move_to_end(e)
            hits.append(True)
        else:
            if len(cache) == S:
                cache.popitem(last=False)
            cache[e] = None
            hits.append(False)
        sets.append(set(cache))
    return hits, sets


@pytest.mark.parametrize("E,S,seed", [(8, 3, 0), (16, 5, 1), (32, 32, 2), (40, 1, 3)])
def test_one_expert_per_batch_is_textbook_lru(E, S, seed):
    rng = np.random.default_rng(seed)
    seq = [int(v) for v in rng.zipf(1.3, size=400) % E]
    want_hits, want_sets = textbook_lru(seq, S)
    c = ExpertCacheOracle(E, S)
    for e, hit, want in zip(seq, want_hits, want_sets):
        loads = c.batch([e])
        assert (loads == []) == hit
        assert {x for x in c.expert_in if x >= 0} == want
    assert c.hits == sum(want_hits)
    assert c.misses == len(seq) - sum(want_hits)


def test_hand_worked_sequence():
    # E=6, S=3.  Stamps after each batch written out by hand:
    #  b1 {0,1}: empty slots 0,1 (stamp -1)        -> loads (0,0),(1,1); stamps [1,1,-1]
    #  b2 {2}:   empty slot 2                      -> (2,2);             stamps [1,1,2]
    #  b3 {3,0}: 0 hits slot 0 (stamp 3); 3 takes the oldest unused slot 1 (stamp 1)
    #                                              -> (3,1);             stamps [3,3,2]
    #  b4 {4,5}: unused slots by age: 2 (2), 0 (3), 1 (3) -> (4,2),(5,0); stamps [4,3,4]
    #  b5 {1,5}: 5 hits slot 0; 1 was evicted, oldest unused slot 1 (3) -> (1,1)
    c = ExpertCacheOracle(6, 3)
    assert c.batch([1, 0]) == [(0, 0), (1, 1)]
    assert c.batch([2]) == [(2, 2)]
    assert c.batch([3, 0]) == [(3, 1)]
    assert c.batch([5, 4]) == [(4, 2), (5, 0)]
    assert c.stamp == [4, 3, 4]
    assert c.batch([1, 5]) == [(1, 1)]
    assert c.expert_in == [5, 1, 4]
    assert c.slot_of == [-1, 1, -1, -1, 2, 0]
    assert (c.hits, c.misses) == (2, 7)


@pytest.mark.parametrize("E,S,seed", [(64, 24, 5), (256, 128, 6), (16, 16, 7)])
def test_every_eviction_is_least_recently_used(E, S, seed):
    rng = np.random.default_rng(seed)
    c = ExpertCacheOracle(E, S)
    last_use = {}                      # expert -> batch number it was last needed in
    for b in range(1, 120):
        n = int(rng.integers(1, S + 1))
        pop = rng.zipf(1.2, size=4 * n) % E
        need = sorted(set(int(v) for v in pop))[:n]
        before = {e: c.slot_of[e] for e in range(E) if c.slot_of[e] >= 0}
        loads = c.batch(need)
        # loads are exactly the needed experts that were not resident, in ascending order
        assert [e for e, _ in loads] == [e for e in need if e not in before]
        for e, v in loads:
            victim = next((x for x, s in before.items() if s == v), None)
            if victim is not None:
                assert victim not in need
                # no resident, unneeded expert that survives was used less recently
                survivors = [x for x in before if x not in need and c.slot_of[x] >= 0]
                assert all(last_use[victim] <= last_use[x] for x in survivors)
            else:
                assert len(before) < S
        for e in need:
            last_use[e] = b
            assert c.slot_of[e] >= 0
        resident = [e for e in range(E) if c.slot_of[e] >= 0]
        assert len(resident) <= S
        for e in resident:
            assert c.expert_in[c.slot_of[e]] == e


def test_batch_larger_than_cache_is_an_error():
    c = ExpertCacheOracle(8, 2)
    with pytest.raises(ValueError):
        c.batch([0, 1, 2])
