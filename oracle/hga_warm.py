"""CPU model of the warm tier: a bounded device-memory LRU of routed groups.

TEST INFRASTRUCTURE ONLY.  The test suite and the benchmark's CPU leg are the
only callers allowed; the product never imports or runs this module, and this
module imports nothing from the product.

What it restates
----------------
The technical summary of "Hierarchical Global Attention (HGA)" (gist.science,
paper 2606.30709; Italian page "Riepilogo Tecnico", section "Architettura della
Memoria", and the French page's "Architecture Memoire"): between the hot tier
(summaries and the always-visible windows, in VRAM) and the cold tier (the
whole K/V history, in host RAM or NVMe) sits a warm tier, a bounded LRU cache
in VRAM of recently routed spans.  The pages give neither its unit, nor its
size, nor how a step's several requests are ordered, nor ties.  Readings
(each one is listed in the design notes):

W1  The cached unit is one routed group (g tokens of K and V): the unit that
    level-2 routing selects and the host tier fetches.
W2  One decode step makes one batch of requests per (sequence, KV head): the
    groups the attention keeps from that unit's group_idx row (valid,
    in a candidate chunk, strictly ascending: the rule the attention applies).
    All of a step's requests are touched at once, so a request never evicts
    another request of the same step.
W3  Recency is a step clock per (sequence, KV head): one more than the largest
    stamp in its table.  A hit or an inserted group gets the clock as stamp.
W4  Victims are taken in the order (empty slots by slot index) then
    (stamp, group id) ascending: least recently used first; among groups last
    used in the same step, the lower id first.  The step's misses, ascending,
    take the victims in that order.

The state of one (sequence, KV head) is tag[M] (group id, -1 when empty) and
stamp[M] (0 when empty); slot s caches the K/V rows of group tag[s].

Pinned by tests/test_warm_pins.py: a textbook ordered-dict LRU gives the same
cached set and hit counts; closed forms (compulsory misses only when every
requested group fits; zero hits for a cycle larger than the cache; a repeated
request set hits in full after its first step); invariants (unique tags, every
request cached after its step, stamps).
"""

from __future__ import annotations

import numpy as np


def kept_groups(group_idx_row, cur: int, sink: int, local: int, groups_per_chunk: int):
    """Groups kept from one group_idx row, with their input positions (W2).

    An entry is kept when it is >= 0, names a group of a candidate chunk
    (sink <= chunk < cur - local) and exceeds every entry kept before it."""
    ids, at = [], []
    for j, gid in enumerate(int(x) for x in group_idx_row):
        if gid < 0:
            continue
        c = gid // groups_per_chunk
        if not (sink <= c < cur - local):
            continue
        if ids and gid <= ids[-1]:
            continue
        ids.append(gid)
        at.append(j)
    return ids, at


def empty_table(slots: int):
    """A cleared table: every slot empty."""
    return np.full(slots, -1, dtype=np.int64), np.zeros(slots, dtype=np.int64)


def warm_step(tag: np.ndarray, stamp: np.ndarray, requests):
    """One step of the cache of one (sequence, KV head), in place.

    requests: the step's kept group ids, ascending and distinct (W2); there
    must be no more of them than slots.  Returns (slot_of, hits, misses):
    slot_of[i] is the slot that holds requests[i] after the step; misses are
    the requests that were not cached (their rows are fetched from the host)."""
    M = len(tag)
    requests = [int(r) for r in requests]
    assert len(requests) <= M
    assert all(a < b for a, b in zip(requests, requests[1:]))
    clock = int(stamp.max()) + 1 if M else 1                       # W3
    where = {int(t): s for s, t in enumerate(tag) if t >= 0}
    slot_of = [where.get(r, -1) for r in requests]
    hit_slots = {s for s in slot_of if s >= 0}
    for s in hit_slots:
        stamp[s] = clock

    def order(s):                                                   # W4
        return (0, s, 0) if tag[s] < 0 else (1, int(stamp[s]), int(tag[s]))

    victims = sorted((s for s in range(M) if s not in hit_slots), key=order)
    misses = [i for i, s in enumerate(slot_of) if s < 0]
    for v, i in zip(victims, misses):
        tag[v] = requests[i]
        stamp[v] = clock
        slot_of[i] = v
    return slot_of, len(requests) - len(misses), [requests[i] for i in misses]


def slot_map_row(slot_of, at, kg: int):
    """The slot of every entry of a group_idx row: slot_of at the kept entries'
    input positions, -1 elsewhere."""
    row = [-1] * kg
    for s, j in zip(slot_of, at):
        row[j] = s
    return row
