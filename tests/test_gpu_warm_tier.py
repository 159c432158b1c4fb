"""Warm tier: a bounded VRAM LRU of routed groups in front of the host tier
(HGA technical summary, "Architettura della Memoria").

The table the kernel keeps (tags, stamps, slot map, hit and miss counts) must
equal the oracle's cache model bit for bit on the same requests, step after
step; the attention read through the cache must give the device-resident
path's bits (and the oracle's output within the bf16 tolerance).
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import TOL, layer_of, oracle_head, to_device  # noqa: E402
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402
from oracle import hga_oracle as O  # noqa: E402
from oracle import hga_warm as W  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def _wl(**kw):
    base = dict(batch=2, context=4096, heads_q=8, heads_kv=2)
    base.update(kw)
    return S.workload("host_tier_decode_128k", **base)


class Warm:
    """One layer's buffers: the device cache (reference path), the pinned host
    cache, the warm table and working buffers, and the oracle's cache model."""

    def __init__(self, wl, x, slots):
        self.wl, self.x, self.M = wl, x, slots
        n, bh = wl.context, wl.batch * wl.heads_kv
        self.n, self.bh = n, bh
        self.dev_layer = layer_of(wl)
        self.host_layer = layer_of(wl)
        self.host_layer.kv_loc = B.HGA_KV_HOST_PINNED
        self.k = to_device(x["k"], wl.dtype)
        self.v = to_device(x["v"], wl.dtype)
        self.k_host = self.k.cpu().pin_memory()
        self.v_host = self.v.cpu().pin_memory()
        rows = B.hga_warm_rows(self.host_layer, slots)
        assert rows == (wl.sink + wl.local + 1) * wl.chunk + slots * wl.group
        self.k_work = torch.full((bh, rows, wl.head_dim), float("nan"), dtype=torch.bfloat16,
                                 device="cuda")
        self.v_work = torch.full_like(self.k_work, float("nan"))
        self.tags = torch.full((bh, slots), 12345, dtype=torch.int32, device="cuda")
        self.stamps = torch.full((bh, slots), 777, dtype=torch.int32, device="cuda")
        B.hga_warm_reset(self.host_layer, slots, self.tags, self.stamps)
        self.slot_map = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device="cuda")
        self.counters = torch.zeros(2, dtype=torch.int64, device="cuda")
        self.cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device="cuda")
        self.gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device="cuda")
        self.ci = torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device="cuda")
        self.gi = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device="cuda")
        # the oracle's cache model, per (sequence, KV head)
        self.model = [W.empty_table(slots) for _ in range(bh)]
        self.hits = self.misses = 0

    def model_step(self, gi: np.ndarray, pos: np.ndarray) -> np.ndarray:
        """The oracle's table update for one step's group_idx rows; returns its slot map."""
        wl = self.wl
        smap = np.full((self.bh, wl.topk_groups), -1, dtype=np.int64)
        for u in range(self.bh):
            cur = int(pos[u // wl.heads_kv]) // wl.chunk
            ids, at = W.kept_groups(gi[u], cur, wl.sink, wl.local, wl.chunk // wl.group)
            tag, stamp = self.model[u]
            slot_of, hits, misses = W.warm_step(tag, stamp, ids)
            smap[u] = W.slot_map_row(slot_of, at, wl.topk_groups)
            self.hits += hits
            self.misses += len(misses)
        return smap

    def attend(self, q, pos_t, warm: bool):
        wl = self.wl
        out = torch.empty(wl.batch, wl.heads_q, 1, wl.head_dim, device="cuda")
        lse = torch.empty(wl.batch, wl.heads_q, 1, device="cuda")
        if warm:
            B.hga_attend_warm(self.host_layer, q, pos_t, self.k_work, self.v_work, self.n, self.gi,
                              self.slot_map, self.M, out, lse)
        else:
            B.hga_attend(self.dev_layer, q, 1, pos_t, self.k, self.v, self.n, self.gi, out, lse)
        return out, lse

    def gather(self, pos_t, refresh):
        B.hga_gather_warm(self.host_layer, self.k_host, self.v_host, self.n, pos_t, self.gi, self.M,
                          self.tags, self.stamps, self.slot_map, self.k_work, self.v_work,
                          refresh_window=refresh, counters=self.counters)

    def check_table(self, smap_model):
        assert np.array_equal(self.slot_map.cpu().numpy(), smap_model)
        tags, stamps = self.tags.cpu().numpy(), self.stamps.cpu().numpy()
        for u in range(self.bh):
            assert np.array_equal(tags[u], self.model[u][0]), f"tags of unit {u}"
            assert np.array_equal(stamps[u], self.model[u][1]), f"stamps of unit {u}"
        assert self.counters.cpu().tolist() == [self.hits, self.misses]


def _plant(rng, row, wl, cur):
    """Entries the attention drops: a -1, a window-chunk group, a duplicate,
    a descending entry."""
    row = row.copy()
    gpc = wl.chunk // wl.group
    row[3] = -1
    row[5] = (cur - 1) * gpc           # a local chunk: not a candidate
    row[8] = row[7]                     # duplicate
    row[12], row[13] = row[13], row[12]  # descending pair: the later one is dropped
    return row


@pytest.mark.parametrize("slots,keep", [(32, 0.9), (48, 0.8), (128, 0.95), (2048, 0.5)])
def test_warm_table_matches_the_oracle_model(slots, keep):
    """64 steps of synthetic selections (some with entries the attention drops):
    table, slot map and counts equal the cache model; outputs equal the
    device-resident path bit for bit."""
    wl = _wl()
    x = S.make_inputs(wl, 51)
    w = Warm(wl, x, slots)
    pos = np.array([4095, 3001], dtype=np.int64)
    pos_t = torch.as_tensor(pos, device="cuda")
    q = to_device(x["q"], wl.dtype)
    req = S.group_requests(wl, 52 + slots, 64, pos, keep)
    rng = np.random.default_rng(slots)
    assert B.hga_device_status() == 0
    for t in range(64):
        gi = req[t].reshape(w.bh, wl.topk_groups)
        planted = t % 8 == 5
        if planted:
            gi = np.stack([_plant(rng, gi[u], wl, int(pos[u // wl.heads_kv]) // wl.chunk)
                           for u in range(w.bh)])
        w.gi.copy_(torch.as_tensor(gi, dtype=torch.int32))
        w.gather(pos_t, refresh=(t == 0))
        out_w, lse_w = w.attend(q, pos_t, warm=True)
        out_d, lse_d = w.attend(q, pos_t, warm=False)
        torch.cuda.synchronize()
        assert B.hga_device_status() == (6 if planted else 0)   # dropped entries are flagged
        w.check_table(w.model_step(gi, pos))
        assert torch.equal(out_w.view(torch.int32), out_d.view(torch.int32)), f"out at step {t}"
        assert torch.equal(lse_w.view(torch.int32), lse_d.view(torch.int32)), f"lse at step {t}"
        if t in (0, 63):   # the oracle's attention over the same selection
            out = out_w.cpu().numpy()
            for b, h in ((0, 0), (1, 1)):
                prm, qo, k, v, pl, summ = oracle_head(wl, dict(x, pos=pos), b, h)
                ora = O.hga_layer(qo, k, v, pl, prm, summaries=summ,
                                  group_idx_override=[[list(gi[b * wl.heads_kv + h])]])
                g = wl.gqa
                assert np.max(np.abs(out[b, h * g:(h + 1) * g] - ora["out"])) <= TOL[wl.dtype]
    assert w.hits > 0 and w.misses > 0


def test_warm_decode_loop_equals_device_and_cold_paths():
    """64 decode steps with drifting queries and advancing positions (across
    chunk boundaries), routed on the GPU: the warm path (window rows copied one
    per step after the first) gives the device-resident path's and the cold
    host path's bits at every step; the table stays a valid cache of the kept
    groups; consecutive steps hit."""
    wl = _wl()
    x = S.make_inputs(wl, 53)
    slots = 96
    w = Warm(wl, x, slots)
    qs = S.drifting_queries(wl, 54, 64, 0.95)
    cold_rows = B.hga_hot_rows(w.host_layer)
    k_cold = torch.full((w.bh, cold_rows, wl.head_dim), float("nan"), dtype=torch.bfloat16,
                        device="cuda")
    v_cold = torch.full_like(k_cold, float("nan"))
    start = 4000
    B.hga_build_summaries(w.dev_layer, w.k, w.n, 0, start, w.cs, w.gs)
    hits = []
    for t, p in enumerate(range(start, start + 64)):
        pos = np.array([p, p - 3], dtype=np.int64)
        pos_t = torch.as_tensor(pos, device="cuda")
        q = to_device(qs[t], wl.dtype)
        B.hga_build_summaries(w.dev_layer, w.k, w.n, p, p + 1, w.cs, w.gs)
        B.hga_route(w.dev_layer, q, 1, pos_t, w.cs, w.gs, w.n, w.ci, w.gi)
        before = w.counters.cpu().tolist()
        w.gather(pos_t, refresh=1 if t == 0 else 2)   # then the newest window row only
        out_w, lse_w = w.attend(q, pos_t, warm=True)
        out_d, lse_d = w.attend(q, pos_t, warm=False)
        B.hga_gather_host(w.host_layer, w.k_host, w.v_host, w.n, pos_t, w.gi, k_cold, v_cold,
                          refresh_window=(t == 0))
        out_c = torch.empty_like(out_d)
        lse_c = torch.empty_like(lse_d)
        B.hga_attend(w.host_layer, q, 1, pos_t, k_cold, v_cold, w.n, w.gi, out_c, lse_c)
        torch.cuda.synchronize()
        assert B.hga_device_status() == 0
        for a, b_ in ((out_w, out_d), (lse_w, lse_d), (out_w, out_c), (lse_w, lse_c)):
            assert torch.equal(a.view(torch.int32), b_.view(torch.int32)), f"step at {p}"
        # the table holds every kept group at the slot the map names, stamped now
        gi = w.gi.cpu().numpy()
        smap, tags, stamps = (w.slot_map.cpu().numpy(), w.tags.cpu().numpy(),
                              w.stamps.cpu().numpy())
        for u in range(w.bh):
            live = tags[u][tags[u] >= 0]
            assert len(np.unique(live)) == len(live)
            assert stamps[u].max() == t + 1
            kept = gi[u] >= 0      # the GPU routing's rows are all valid
            assert (smap[u][~kept] == -1).all()
            assert np.array_equal(tags[u][smap[u][kept]], gi[u][kept])
            assert (stamps[u][smap[u][kept]] == t + 1).all()
        after = w.counters.cpu().tolist()
        assert after[0] + after[1] - before[0] - before[1] == int((gi >= 0).sum())
        hits.append(after[0] - before[0])
    total = int(w.counters.cpu()[0] + w.counters.cpu()[1])
    assert hits[0] == 0
    assert sum(hits) > 0.5 * total, f"hit rate {sum(hits) / total:.2f} with drifting queries"


def test_warm_reset_of_one_sequence():
    """Resetting one sequence empties its tables only; the cache refills and
    still follows the model (which resets the same tables)."""
    wl = _wl()
    x = S.make_inputs(wl, 55)
    w = Warm(wl, x, 40)
    pos = np.array([4095, 4095], dtype=np.int64)
    pos_t = torch.as_tensor(pos, device="cuda")
    req = S.group_requests(wl, 56, 20, pos, 0.85)
    for t in range(20):
        gi = req[t].reshape(w.bh, wl.topk_groups)
        if t == 10:
            before = w.tags.cpu().numpy()
            B.hga_warm_reset(w.host_layer, w.M, w.tags, w.stamps, seq=1)
            tags = w.tags.cpu().numpy()
            assert np.array_equal(tags[:wl.heads_kv], before[:wl.heads_kv])
            assert (tags[wl.heads_kv:] == -1).all()
            assert (w.stamps.cpu().numpy()[wl.heads_kv:] == 0).all()
            for u in range(wl.heads_kv, 2 * wl.heads_kv):
                w.model[u] = W.empty_table(w.M)
        w.gi.copy_(torch.as_tensor(gi, dtype=torch.int32))
        w.gather(pos_t, refresh=(t == 0))
        torch.cuda.synchronize()
        w.check_table(w.model_step(gi, pos))


def test_warm_attend_flags_a_slot_outside_the_table():
    """A slot map that disagrees with group_idx is flagged; the read stays in the buffer."""
    wl = _wl()
    x = S.make_inputs(wl, 57)
    w = Warm(wl, x, 32)
    pos = np.array([4095, 4095], dtype=np.int64)
    pos_t = torch.as_tensor(pos, device="cuda")
    q = to_device(x["q"], wl.dtype)
    w.gi.copy_(torch.as_tensor(S.group_requests(wl, 58, 1, pos, 1.0)[0].reshape(w.bh, -1)))
    w.gather(pos_t, refresh=True)
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    w.slot_map[1, 4] = w.M          # one past the table
    out, _ = w.attend(q, pos_t, warm=True)
    torch.cuda.synchronize()
    assert B.hga_device_status() == 6
    assert torch.isfinite(out).all()
    assert B.hga_device_status() == 0


def test_cold_tier_decode_loop_equals_device_path(tmp_path):
    """The history in a file (the cold tier): each step plans on the GPU, stages the
    misses and window rows from the file on the host, fills the warm buffers and
    attends; 48 routed steps with drifting queries across chunk boundaries give the
    device-resident path's bits, and only the misses are read."""
    wl = _wl()
    x = S.make_inputs(wl, 59)
    slots = 64
    w = Warm(wl, x, slots)
    lay = w.host_layer
    qs = S.drifting_queries(wl, 60, 48, 0.95)
    plan = torch.empty(w.bh, wl.topk_groups, 2, dtype=torch.int32, device="cuda")
    n_plan = torch.empty(w.bh, dtype=torch.int32, device="cuda")
    plan_h = torch.empty(plan.shape, dtype=torch.int32).pin_memory()
    n_plan_h = torch.empty(n_plan.shape, dtype=torch.int32).pin_memory()
    staging = torch.zeros(B.hga_cold_stage_bytes(lay), dtype=torch.uint8).pin_memory()
    start = 4000
    B.hga_build_summaries(w.dev_layer, w.k, w.n, 0, start, w.cs, w.gs)
    read_groups = 0
    with B.ColdStore(tmp_path / "kv.bin", lay, w.n, create=True) as store:
        store.write(w.k_host, w.v_host, 0, start)          # the prompt's history
        for t, p in enumerate(range(start, start + 48)):
            store.write(w.k_host, w.v_host, p, p + 1)       # the step's new row
            pos = np.array([p, p - 3], dtype=np.int64)
            pos_t = torch.as_tensor(pos, device="cuda")
            q = to_device(qs[t], wl.dtype)
            mode = 1 if t == 0 else 2
            B.hga_build_summaries(w.dev_layer, w.k, w.n, p, p + 1, w.cs, w.gs)
            B.hga_route(w.dev_layer, q, 1, pos_t, w.cs, w.gs, w.n, w.ci, w.gi)
            B.hga_warm_plan(lay, w.n, pos_t, w.gi, slots, w.tags, w.stamps, w.slot_map, plan,
                            n_plan, counters=w.counters)
            plan_h.copy_(plan)
            n_plan_h.copy_(n_plan)
            torch.cuda.synchronize()
            store.stage(lay, pos, plan_h.numpy(), n_plan_h.numpy(), mode, staging, threads=4)
            B.hga_warm_fill(lay, w.n, pos_t, staging, plan, n_plan, slots, mode, w.k_work,
                            w.v_work)
            out_w, lse_w = w.attend(q, pos_t, warm=True)
            out_d, lse_d = w.attend(q, pos_t, warm=False)
            torch.cuda.synchronize()
            assert B.hga_device_status() == 0
            assert torch.equal(out_w.view(torch.int32), out_d.view(torch.int32)), f"step at {p}"
            assert torch.equal(lse_w.view(torch.int32), lse_d.view(torch.int32))
            read_groups += int(n_plan_h.sum())
    hits, misses = w.counters.cpu().tolist()
    assert misses == read_groups and hits > misses
