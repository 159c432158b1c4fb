"""Pins of the warm-tier cache model (oracle/hga_warm.py) against facts fixed
outside itself: a textbook ordered-dict LRU, closed forms of LRU hit counts, and
invariants of the table.  The warm tier is the bounded VRAM cache of recently
routed spans of the HGA technical summary ("Architettura della Memoria").
"""

from collections import OrderedDict

import numpy as np
import pytest

from oracle import hga_warm as W


def _dict_lru(steps, capacity):
    """The textbook LRU (an ordered dict, least recent first) with a step's
    requests touched together: hits leave their place, the oldest entries make
    room, then the step's requests enter in ascending order."""
    d = OrderedDict()
    out = []
    for req in steps:
        hits = sum(1 for r in req if r in d)
        for r in req:
            d.pop(r, None)
        while len(d) + len(req) > capacity:
            d.popitem(last=False)
        for r in sorted(req):
            d[r] = True
        out.append((hits, set(d)))
    return out


def _run(steps, slots):
    tag, stamp = W.empty_table(slots)
    res = []
    for req in steps:
        slot_of, hits, misses = W.warm_step(tag, stamp, req)
        res.append((slot_of, hits, misses, tag.copy(), stamp.copy()))
    return res


def _random_steps(rng, n_steps, per_step, universe, drift):
    """Request sets that drift: each step keeps a share of the last one."""
    cur = sorted(rng.choice(universe, per_step, replace=False).tolist())
    steps = [cur]
    for _ in range(n_steps - 1):
        keep = [c for c in cur if rng.random() < drift]
        fresh = [x for x in rng.permutation(universe).tolist() if x not in keep]
        cur = sorted(keep + fresh[:per_step - len(keep)])
        steps.append(cur)
    return steps


@pytest.mark.parametrize("slots,per_step,universe,drift",
                         [(8, 8, 40, 0.5), (12, 8, 40, 0.7), (32, 8, 100, 0.9),
                          (16, 3, 20, 0.3), (64, 32, 200, 0.8), (33, 32, 64, 0.95)])
def test_matches_textbook_lru(slots, per_step, universe, drift):
    """Same cached set and hit count as the ordered-dict LRU after every step."""
    rng = np.random.default_rng(slots * 1000 + per_step)
    steps = _random_steps(rng, 80, per_step, universe, drift)
    ref = _dict_lru(steps, slots)
    got = _run(steps, slots)
    for (hits_r, set_r), (_, hits, _, tag, _) in zip(ref, got):
        assert hits == hits_r
        assert set(int(t) for t in tag if t >= 0) == set_r


def test_compulsory_misses_only_when_everything_fits():
    """With room for every group ever requested, the misses are the first touches."""
    rng = np.random.default_rng(5)
    steps = _random_steps(rng, 50, 6, 30, 0.4)
    got = _run(steps, 30)
    seen = set()
    for req, (_, hits, misses, _, _) in zip(steps, got):
        assert sorted(misses) == sorted(set(req) - seen)
        seen |= set(req)


def test_cycle_larger_than_the_cache_never_hits():
    """LRU on a cyclic scan of more groups than slots: every request misses."""
    steps = [[3 * i + j for j in range(3)] for i in range(5)] * 4   # 15 groups, 12 slots
    got = _run(steps, 12)
    assert all(hits == 0 for _, hits, _, _, _ in got)


def test_repeated_set_hits_in_full_after_the_first_step():
    got = _run([[1, 4, 9, 16]] * 10, 4)
    assert [h for _, h, _, _, _ in got] == [0] + [4] * 9
    # the slots never move once assigned
    assert all(r[0] == got[0][0] for r in got)


def test_exact_capacity_holds_exactly_the_last_step():
    rng = np.random.default_rng(7)
    steps = _random_steps(rng, 40, 10, 50, 0.6)
    for req, (_, _, _, tag, _) in zip(steps, _run(steps, 10)):
        assert sorted(int(t) for t in tag) == req


def test_table_invariants():
    rng = np.random.default_rng(11)
    steps = _random_steps(rng, 60, 16, 120, 0.75)
    prev_clock = 0
    for req, (slot_of, hits, misses, tag, stamp) in zip(steps, _run(steps, 40)):
        live = tag[tag >= 0]
        assert len(set(live.tolist())) == len(live)                # unique tags
        assert [int(tag[s]) for s in slot_of] == req                # every request cached
        clock = int(stamp.max())
        assert clock == prev_clock + 1                               # one tick per step
        assert all(stamp[s] == clock for s in slot_of)
        assert (stamp[tag < 0] == 0).all()
        assert hits + len(misses) == len(req)
        prev_clock = clock


def test_victims_least_recent_first_then_lower_id():
    """Hand-worked: slots filled over three steps, then two misses evict the
    two oldest groups, the lower id first among the oldest step's."""
    tag, stamp = W.empty_table(4)
    W.warm_step(tag, stamp, [10, 20])     # step 1: slots 0, 1
    W.warm_step(tag, stamp, [5])          # step 2: slot 2
    W.warm_step(tag, stamp, [20, 30])     # step 3: 20 hits, 30 -> slot 3
    slot_of, hits, misses = W.warm_step(tag, stamp, [7, 8])
    assert hits == 0 and misses == [7, 8]
    # 10 (stamp 1) goes first, then 5 (stamp 2); 20 and 30 (stamp 3) stay
    assert slot_of == [0, 2]
    assert tag.tolist() == [7, 20, 8, 30]
    assert stamp.tolist() == [4, 3, 4, 3]


def test_kept_groups_rule():
    # chunk = gid // 4; candidates are chunks 1..5 with sink 1, local 2, cur 8
    row = [-1, 3, 4, 4, 9, 8, 23, 24, 12, -1]
    ids, at = W.kept_groups(row, cur=8, sink=1, local=2, groups_per_chunk=4)
    assert ids == [4, 9, 23]
    assert at == [2, 4, 6]
    assert W.slot_map_row([5, 6, 7], at, len(row)) == [-1, -1, 5, -1, 6, -1, 7, -1, -1, -1]
