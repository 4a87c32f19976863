"""Pins of the oracle's expert-cache plan (per-layer LFU over the router's
top-k ids) to a sequence worked by hand and to invariants that any correct
plan satisfies.  Each test names the mistake it is there to catch."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lfu_sequence.txt")


def _ints(field):
    return [int(v) for v in field.split(",")] if field.strip() != "-" else []


def test_hand_worked_sequence():
    """catches: evicting a pinned slot, the wrong tie rule, counts that survive
    eviction, misses filled before hits are found."""
    c = oracle.LfuCache(4)
    for ln in open(GOLDEN):
        if not ln.strip() or ln.startswith("#"):
            continue
        ids, slot_of, misses, slots, counts = [f.strip() for f in ln.split("|")]
        got_slot, got_miss = c.step(_ints(ids))
        assert got_slot.tolist() == _ints(slot_of), ln
        want_miss = [tuple(int(v) for v in m.split(":")) for m in misses.split(",")] \
            if misses != "-" else []
        assert got_miss == want_miss, ln
        assert c.expert.tolist() == _ints(slots), ln
        assert c.count.tolist() == _ints(counts), ln


@pytest.mark.parametrize("nslots,k,E", [(16, 8, 128), (16, 16, 64), (8, 1, 5)])
def test_invariants_on_long_random_sequences(nslots, k, E):
    """catches: a token's expert missing after its step, duplicates in the
    cache, a miss on an expert that was cached, a hit that was not."""
    g = np.random.default_rng(nslots + k + E)
    c = oracle.LfuCache(nslots)
    hits = misses = 0
    for _ in range(400):
        # skewed draws so that hits happen
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        ids = g.choice(E, k, replace=False, p=p / p.sum()).astype(np.int32)
        before = set(c.expert.tolist())
        slot_of, miss = c.step(ids)
        for j, e in enumerate(ids):
            assert c.expert[slot_of[j]] == e
        cached = [e for e in c.expert.tolist() if e >= 0]
        assert len(cached) == len(set(cached))
        assert {m[0] for m in miss} == {int(e) for e in ids if int(e) not in before}
        hits += k - len(miss)
        misses += len(miss)
    assert hits > 0 and misses > 0


def test_rejects_repeats_and_overflow():
    c = oracle.LfuCache(4)
    with pytest.raises(ValueError):
        c.step([1, 1])
    with pytest.raises(ValueError):
        c.step([1, 2, 3, 4, 5])


def test_lfu_rejects_slot_counts_beyond_its_flags():
    """The plan keeps one pinned flag per slot for at most 256 slots; more
    slots (or none) are refused instead of overrunning the flags."""
    for n in (0, 257, 1000):
        c = oracle.LfuCache(nslots=max(n, 1))
        c.nslots = n
        c.expert = np.full(max(n, 1), -1, np.int32)
        c.count = np.zeros(max(n, 1), np.int64)
        with pytest.raises(ValueError):
            c.step([1])
