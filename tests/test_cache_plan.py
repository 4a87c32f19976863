"""The library's LFU expert-cache plan (host code, no GPU) against the
oracle's, step by step, and against the hand-worked sequence."""
import os

import numpy as np
import pytest

import oracle
from moe_expert_gemv_b200 import qmoe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lfu_sequence.txt")


@pytest.mark.parametrize("nslots,k,E,skew", [(16, 8, 128, 1.1), (16, 16, 64, 0.8),
                                             (4, 3, 12, 1.5), (8, 1, 9, 0.0)])
def test_plan_equals_oracle(nslots, k, E, skew):
    g = np.random.default_rng(nslots * 100 + k)
    lib_plan, ref = qmoe.LfuPlan(nslots), oracle.LfuCache(nslots)
    p = 1.0 / np.arange(1, E + 1) ** skew
    for t in range(1500):
        ids = g.choice(E, k, replace=False, p=p / p.sum())
        a, b = lib_plan.step(ids), ref.step(ids)
        assert a[0].tolist() == b[0].tolist() and a[1] == b[1], "step %d" % t
    e, c = lib_plan.slots()
    assert e.tolist() == ref.expert.tolist() and c.tolist() == ref.count.tolist()


def test_hand_worked_sequence():
    plan = qmoe.LfuPlan(4)
    for ln in open(GOLDEN):
        if not ln.strip() or ln.startswith("#"):
            continue
        ids, slot_of, misses, slots, counts = [f.strip() for f in ln.split("|")]
        got_slot, got_miss = plan.step([int(v) for v in ids.split(",")])
        assert got_slot.tolist() == [int(v) for v in slot_of.split(",")], ln
        want = [tuple(int(v) for v in m.split(":")) for m in misses.split(",")] \
            if misses != "-" else []
        assert got_miss == want, ln
        e, c = plan.slots()
        assert e.tolist() == [int(v) for v in slots.split(",")], ln
        assert c.tolist() == [int(v) for v in counts.split(",")], ln


def test_rejections_leave_the_cache_unchanged():
    plan = qmoe.LfuPlan(4)
    plan.step([1, 2])
    before = [a.copy() for a in plan.slots()]
    for bad in ([3, 3], [1, 2, 3, 4, 5]):
        with pytest.raises(ValueError):
            plan.step(bad)
    after = plan.slots()
    assert all(np.array_equal(x, y) for x, y in zip(before, after))
