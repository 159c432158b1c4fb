"""Ragged serving batches over a paged K/V pool (block tables).

The paged decode step must give the dense decode step's bits (routing, scores,
outputs and the appended summary rows) on a cache holding the same rows, for
any page size and any scattering of the pages, with every sequence at its own
position; the paged summary build must give the dense build's rows; and the
output must match the oracle.  A block-table entry that is not a page of the
pool is flagged and read as zeros, never outside the pool.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import compare_head, layer_of, to_device  # noqa: E402
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def paginate(k, v, pos, page, seed, spare=7):
    """Scatter each sequence's rows [0, pos[b]] into a shuffled pool of pages.

    Returns (k_pool, v_pool [n_pages, Hkv, page, D], block_table [B, max_pages]
    with -1 past each sequence's last page, n_pages)."""
    b_, hkv, n, d = k.shape
    max_pages = n // page
    need = [int(p) // page + 1 for p in pos]
    n_pages = sum(need) + spare
    order = np.random.default_rng(seed).permutation(n_pages)
    bt = np.full((b_, max_pages), -1, dtype=np.int32)
    kp = torch.zeros(n_pages, hkv, page, d, dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    at = 0
    for b in range(b_):
        for j in range(need[b]):
            pg = int(order[at])
            at += 1
            bt[b, j] = pg
            kp[pg] = k[b, :, j * page:(j + 1) * page]
            vp[pg] = v[b, :, j * page:(j + 1) * page]
    return kp, vp, torch.as_tensor(bt, device=k.device), n_pages


class Batch:
    """A ragged batch: the dense cache and its paged copy, with summary tables,
    routing and output buffers for each."""

    def __init__(self, wl, x, pos, page, seed):
        self.wl, self.x, self.page = wl, x, page
        self.pos = np.asarray(pos, dtype=np.int64)
        self.pos_t = torch.as_tensor(self.pos, device="cuda")
        self.layer = layer_of(wl, B.HGA_F32)
        self.q = to_device(x["q"], wl.dtype)
        self.k = to_device(x["k"], wl.dtype)
        self.v = to_device(x["v"], wl.dtype)
        self.kp, self.vp, self.bt, self.n_pages = paginate(self.k, self.v, self.pos, page, seed)
        self.kv = B.kv_pages(self.bt, self.n_pages, page, wl.context // page)
        self.bufs = {name: self.new_bufs() for name in ("dense", "paged")}

    def new_bufs(self):
        wl = self.wl
        bh, n = wl.batch * wl.heads_kv, wl.context
        return dict(cs=torch.full((bh, n // wl.chunk, wl.head_dim), float("nan"), device="cuda"),
                    gs=torch.full((bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim),
                                  float("nan"), device="cuda"),
                    ci=torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device="cuda"),
                    gi=torch.empty(bh, wl.topk_groups, dtype=torch.int32, device="cuda"),
                    csc=torch.empty(bh, wl.topk_chunks, device="cuda"),
                    gsc=torch.empty(bh, wl.topk_groups, device="cuda"),
                    out=torch.empty(wl.batch, wl.heads_q, 1, wl.head_dim, device="cuda"),
                    lse=torch.empty(wl.batch, wl.heads_q, 1, device="cuda"))

    def summaries(self):
        """Every row closed before each sequence's token (the step appends the rest)."""
        d, p = self.bufs["dense"], self.bufs["paged"]
        for b in range(self.wl.batch):   # dense: the batch builder, one sequence at a time
            lay = layer_of(self.wl.with_(batch=1), B.HGA_F32)
            sl = slice(b * self.wl.heads_kv, (b + 1) * self.wl.heads_kv)
            B.hga_build_summaries(lay, self.k[b:b + 1], self.wl.context, 0, int(self.pos[b]),
                                  d["cs"][sl], d["gs"][sl])
        B.hga_build_summaries_paged(self.layer, self.kp, self.kv, self.pos_t, p["cs"], p["gs"])

    def step(self, which, append=True):
        bf = self.bufs[which]
        if which == "dense":
            B.hga_decode_step(self.layer, self.q, self.pos_t, bf["cs"], bf["gs"], self.wl.context,
                              self.k, self.v, bf["ci"], bf["gi"], bf["out"], bf["lse"],
                              chunk_score=bf["csc"], group_score=bf["gsc"], append=append)
        else:
            B.hga_decode_step_paged(self.layer, self.q, self.pos_t, bf["cs"], bf["gs"], self.kp,
                                    self.vp, self.kv, bf["ci"], bf["gi"], bf["out"], bf["lse"],
                                    chunk_score=bf["csc"], group_score=bf["gsc"], append=append)


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int32), b.contiguous().view(torch.int32))


def _closed_rows_equal(batch, upto):
    """Summary rows of every group / chunk that ends at or before upto[b], bitwise."""
    wl = batch.wl
    d, p = batch.bufs["dense"], batch.bufs["paged"]
    for b in range(wl.batch):
        sl = slice(b * wl.heads_kv, (b + 1) * wl.heads_kv)
        n_groups = (int(upto[b]) + 1) // wl.group
        n_chunks = (int(upto[b]) + 1) // wl.chunk
        gd = d["gs"][sl].reshape(wl.heads_kv, -1, wl.head_dim)[:, :n_groups]
        gp = p["gs"][sl].reshape(wl.heads_kv, -1, wl.head_dim)[:, :n_groups]
        assert _same_bits(gd, gp), f"group rows of sequence {b}"
        assert _same_bits(d["cs"][sl, :n_chunks], p["cs"][sl, :n_chunks]), f"chunk rows of {b}"


RAGGED = [8191, 5000, 40 * 64 + 17, 1023, 7777, 4095, 64 * 3 - 1, 2 * 64 * 16 - 1]


@pytest.mark.parametrize("page,many", [(16, 0), (64, 0), (256, 0), (32, 20), (64, 16)])
def test_paged_step_is_bitwise_the_dense_step(page, many):
    """many = 20: 20 sequences x 8 KV heads, more items than SMs (two CTAs per SM);
    many = 16: 128 items, one CTA each; else 8 sequences (each item on a cluster of
    CTAs)."""
    if many:
        pos = np.random.default_rng(4).integers(100, 4096, many)
        wl = S.workload("llama3_8b_decode_32k", batch=many, context=4096)
    else:
        pos = RAGGED
        wl = S.workload("llama3_8b_decode_32k", batch=len(RAGGED), context=8192)
    x = S.make_inputs(wl, 71)
    bt = Batch(wl, x, pos, page, seed=page)
    bt.summaries()
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    _closed_rows_equal(bt, bt.pos - 1)
    bt.step("dense")
    bt.step("paged")
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    d, p = bt.bufs["dense"], bt.bufs["paged"]
    for name in ("ci", "gi"):
        assert torch.equal(d[name], p[name]), name
    for name in ("csc", "gsc", "out", "lse"):
        assert _same_bits(d[name], p[name]), name
    _closed_rows_equal(bt, bt.pos)   # the appended rows too


def test_paged_step_matches_the_oracle():
    wl = S.workload("llama3_8b_decode_32k", batch=len(RAGGED), context=8192)
    x = S.make_inputs(wl, 72)
    bt = Batch(wl, x, RAGGED, 64, seed=3)
    bt.summaries()
    bt.step("paged")
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    p = bt.bufs["paged"]
    res = dict(chunk_idx=p["ci"].cpu().numpy().reshape(wl.batch, wl.heads_kv, 1, -1),
               group_idx=p["gi"].cpu().numpy().reshape(wl.batch, wl.heads_kv, 1, -1),
               out=p["out"].cpu().numpy(), lse=p["lse"].cpu().numpy())
    xp = dict(x, pos=bt.pos)
    for b in range(wl.batch):
        compare_head(wl, xp, res, b, (3 * b) % wl.heads_kv)


def test_paged_small_batch_long_block_table():
    """One sequence at 80K tokens in 16-token pages: 5120 block-table entries staged
    in shared memory beside a cluster's partial buffers.  The step takes a cluster
    size whose whole shared memory (dynamic and static) a block may have, and
    matches the dense step: the same routing and scores, bit for bit, and the
    output up to the merge order of a different cluster size."""
    wl = S.workload("llama3_8b_decode_32k", batch=1, context=81920)
    x = S.make_inputs(wl, 75)
    bt = Batch(wl, x, [81919], 16, seed=11)
    bt.summaries()
    bt.step("dense")
    bt.step("paged")
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    d, p = bt.bufs["dense"], bt.bufs["paged"]
    for name in ("ci", "gi"):
        assert torch.equal(d[name], p[name]), name
    for name in ("csc", "gsc"):
        assert _same_bits(d[name], p[name]), name
    # another cluster size deals the units to other warps, whose P is rounded to bf16
    # against another running maximum: differences of a few 1e-5 in the output
    torch.testing.assert_close(p["out"], d["out"], atol=1e-3, rtol=0)
    torch.testing.assert_close(p["lse"], d["lse"], atol=1e-4, rtol=0)
    res = dict(chunk_idx=p["ci"].cpu().numpy().reshape(wl.batch, wl.heads_kv, 1, -1),
               group_idx=p["gi"].cpu().numpy().reshape(wl.batch, wl.heads_kv, 1, -1),
               out=p["out"].cpu().numpy(), lse=p["lse"].cpu().numpy())
    compare_head(wl, dict(x, pos=bt.pos), res, 0, 5)


def test_paged_decode_loop_keeps_matching_the_dense_loop():
    """Consecutive steps with appends across group and chunk boundaries: the
    paged tables and outputs stay bitwise equal to the dense ones."""
    wl = S.workload("llama3_8b_decode_32k", batch=3, context=4096)
    x = S.make_inputs(wl, 73)
    start = np.array([4000, 2030, 1000], dtype=np.int64)
    bt = Batch(wl, x, start + 40, 32, seed=9)   # pages up to the last step's position
    bt.pos = start.copy()
    bt.pos_t = torch.as_tensor(bt.pos, device="cuda")
    bt.summaries()
    for t in range(40):
        bt.pos_t.copy_(torch.as_tensor(start + t))
        bt.pos = start + t
        bt.step("dense")
        bt.step("paged")
        torch.cuda.synchronize()
        assert B.hga_device_status() == 0
        d, p = bt.bufs["dense"], bt.bufs["paged"]
        assert torch.equal(d["gi"], p["gi"]) and _same_bits(d["out"], p["out"]), f"step {t}"
    _closed_rows_equal(bt, bt.pos)


def test_bad_block_table_entry_is_flagged_and_read_as_zeros():
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=4096)
    x = S.make_inputs(wl, 74)
    pos = [4095, 3000]
    bt = Batch(wl, x, pos, 64, seed=5)
    bt.summaries()
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    good = bt.bt.clone()
    for b, j, bad in ((1, 3000 // 64, bt.n_pages + 5),   # sequence 1's current chunk (a tile read)
                      (0, 4095 // 64, -7),               # the page sequence 0's append reads
                      (0, 0, -1)):                       # sequence 0's sink page
        bt.bt.copy_(good)
        bt.bt[b, j] = bad
        bt.step("paged")
        torch.cuda.synchronize()
        assert B.hga_device_status() == 6, (b, j, bad)
        assert torch.isfinite(bt.bufs["paged"]["out"]).all()
    bt.bt.copy_(good)
    bt.bt[0, 0] = bt.n_pages
    B.hga_build_summaries_paged(bt.layer, bt.kp, bt.kv, bt.pos_t, bt.bufs["paged"]["cs"],
                                bt.bufs["paged"]["gs"])
    torch.cuda.synchronize()
    assert B.hga_device_status() == 6
    bt.bt.copy_(good)
    bt.step("paged")
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
