"""Pins of the float64 oracle against facts fixed outside itself.

Each test checks the oracle against a library routine, a closed form, brute
force or an invariant of the method (HGA technical summary, "Metodologia ->
Meccanismo Core", items 1-4), never against a retyped copy of its own formula.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import hga_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _params(**kw):
    base = dict(head_dim=16, heads_q=4, heads_kv=2, chunk=16, group=4, sink=1, local=2,
                topk_chunks=3, topk_groups=5, n_high_pairs=4, rope_theta=100.0)
    base.update(kw)
    return O.HGAParams(**base)


# ------------------------------------------------------------------------ RoPE

@pytest.mark.parametrize("d,theta", [(64, 1e4), (128, 5e5), (16, 100.0)])
def test_rope_frequencies_match_transformers(d, theta):
    """omega_i equals the inverse frequencies of the Llama rotary embedding (R1)."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    cfg = LlamaConfig(hidden_size=2 * d, num_attention_heads=2, head_dim=d, rope_theta=theta)
    ref = LlamaRotaryEmbedding(cfg).inv_freq.double().numpy()
    np.testing.assert_allclose(O.rope_inv_freq(d, theta), ref, rtol=1e-6)


@pytest.mark.parametrize("d", [16, 64, 128])
def test_rope_rotation_matches_transformers_rotate_half(d):
    """The pair layout and rotation sense equal transformers' apply_rotary_pos_emb (R1)."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, d))
    pos = np.array([0, 1, 2, 5, 31.5, 100, 1023.0])
    freqs = pos[:, None] * O.rope_inv_freq(d, 1e4)[None, :]
    emb = np.concatenate([freqs, freqs], axis=-1)
    cos = torch.from_numpy(np.cos(emb))[None]
    sin = torch.from_numpy(np.sin(emb))[None]
    xt = torch.from_numpy(x)[None, None]
    ref, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
    np.testing.assert_allclose(O.rope_apply(x, pos, 1e4), ref[0, 0].numpy(), atol=1e-12)


def test_rope_inverse_and_composition():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 32))
    p = rng.uniform(-500, 500, 5)
    np.testing.assert_allclose(O.rope_apply(O.rope_apply(x, p, 1e4), -p, 1e4), x, atol=1e-10)
    q = O.rope_apply(x, p, 1e4)
    np.testing.assert_allclose(O.rope_apply(q, p, 1e4), O.rope_apply(x, 2 * p, 1e4), atol=1e-9)


# ------------------------------------------------------------------- summaries

def _dirichlet(length, omega):
    """Mean of the rotations by angles (m - (L-1)/2) * omega, m = 0..L-1 (a pure scaling)."""
    return math.sin(length * omega / 2) / (length * math.sin(omega / 2))


@pytest.mark.parametrize("n_high", [0, 3, 8])
@pytest.mark.parametrize("length,t0", [(16, 0), (16, 48), (4, 12), (64, 4096)])
def test_summary_closed_form_of_a_constant_raw_key(n_high, length, t0):
    """Keys k_t = R(t) k0 (one raw key at every position) have a closed-form summary.

    High pairs: mean over t of R(t omega) k0 = R(r omega) * D_L(omega) k0, with
    D_L the Dirichlet factor sin(L omega/2) / (L sin(omega/2)) and r the span
    centre.  Low pairs: every raw key is k0, so the summary is R(r omega) k0.
    A wrong centre, a swapped split or a missing normalisation fails this.
    """
    d, theta = 16, 50.0
    rng = np.random.default_rng(3)
    k0 = rng.standard_normal(d)
    pos = t0 + np.arange(length)
    k_rot = O.rope_apply(np.repeat(k0[None], length, 0), pos, theta)
    got = O.span_summary(k_rot, t0, n_high, theta)
    omega = O.rope_inv_freq(d, theta)
    scale = np.array([_dirichlet(length, w) if i < n_high else 1.0 for i, w in enumerate(omega)])
    r = t0 + (length - 1) / 2
    want = O.rope_apply((k0 * np.concatenate([scale, scale]))[None], [r], theta)[0]
    np.testing.assert_allclose(got, want, atol=1e-11)


def test_summary_all_high_pairs_is_mean_of_rotated_keys():
    """With every pair high-frequency, a summary is the plain mean of the stored keys."""
    rng = np.random.default_rng(4)
    k_rot = rng.standard_normal((64, 32))
    np.testing.assert_allclose(O.span_summary(k_rot, 640, 16, 1e4), k_rot.mean(0), atol=1e-13)


def test_summary_no_high_pairs_is_rotated_mean_of_raw_keys():
    """With no high pairs, a summary is the mean raw (pre-RoPE) key rotated at the centre.

    The keys are rotated with transformers' RoPE, so this also ties the
    un-rotation inside the oracle to the library's rotation.
    """
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    d, theta, t0, length = 32, 1e4, 192, 64
    rng = np.random.default_rng(5)
    raw = rng.standard_normal((length, d))

    def lib_rotate(x, pos):
        f = np.asarray(pos, dtype=np.float64)[:, None] * O.rope_inv_freq(d, theta)[None]
        e = np.concatenate([f, f], -1)
        xt = torch.from_numpy(x)[None, None]
        out, _ = apply_rotary_pos_emb(xt, xt, torch.from_numpy(np.cos(e))[None],
                                      torch.from_numpy(np.sin(e))[None])
        return out[0, 0].numpy()

    k_rot = lib_rotate(raw, t0 + np.arange(length))
    want = lib_rotate(raw.mean(0)[None], [t0 + 31.5])[0]
    np.testing.assert_allclose(O.span_summary(k_rot, t0, 0, theta), want, atol=1e-12)


def test_summary_score_is_shift_invariant():
    """Scores depend only on relative rotation: moving the query and the span by delta keeps them."""
    d, theta = 32, 1e4
    rng = np.random.default_rng(6)
    raw_k = rng.standard_normal((16, d))
    raw_q = rng.standard_normal(d)
    t0, p = 64, 300

    def score(shift):
        k_rot = O.rope_apply(raw_k, t0 + shift + np.arange(16), theta)
        s = O.span_summary(k_rot, t0 + shift, 5, theta)
        return float(O.rope_apply(raw_q[None], [p + shift], theta)[0] @ s)

    base = score(0)
    for delta in (1, 37, 1000, 65536):
        assert score(delta) == pytest.approx(base, rel=1e-9, abs=1e-9)


@pytest.mark.parametrize("n_high", [0, 2, 5, 8])
@pytest.mark.parametrize("chunk,group", [(16, 4), (32, 8)])
def test_build_summaries_table_rows_sit_at_their_span_centres(n_high, chunk, group):
    """Every row of the chunk and group tables against the closed form of a constant raw key.

    Chunk c holds the keys k_t = R(t) a_c: one raw key a_c (different for every
    chunk) rotated to each token's own position.  Then the row of chunk c is
    R(r) (D_C(omega) a_c) on high pairs and R(r) a_c on low pairs with
    r = c*C + (C-1)/2, and the row of group w of chunk c is the same with
    r = c*C + w*g + (g-1)/2 and the Dirichlet factor D_g.  A row computed at
    another position (the chunk start, the group's chunk start, a shifted
    centre), from another chunk's tokens, or missing its normalisation fails.
    """
    d, theta, nc = 16, 50.0, 6
    prm = _params(chunk=chunk, group=group, n_high_pairs=n_high, rope_theta=theta)
    rng = np.random.default_rng(31 + n_high)
    a = rng.standard_normal((nc, d))
    pos = np.arange(nc * chunk)
    k_rot = O.rope_apply(np.repeat(a, chunk, axis=0), pos, theta)
    cs, gs = O.build_summaries(k_rot, prm)
    omega = O.rope_inv_freq(d, theta)

    def closed_form(raw, length, centre):
        f = np.array([_dirichlet(length, w) if i < n_high else 1.0 for i, w in enumerate(omega)])
        return O.rope_apply((raw * np.concatenate([f, f]))[None], [centre], theta)[0]

    ng = chunk // group
    assert cs.shape == (nc, d) and gs.shape == (nc, ng, d)
    for c in range(nc):
        np.testing.assert_allclose(cs[c], closed_form(a[c], chunk, c * chunk + (chunk - 1) / 2),
                                   atol=1e-11)
        for w in range(ng):
            centre = c * chunk + w * group + (group - 1) / 2
            np.testing.assert_allclose(gs[c, w], closed_form(a[c], group, centre), atol=1e-11)


def test_span_summary_start_position_cancels():
    """The summary of given keys does not depend on the start position passed with them.

    Un-rotating token m at t0 + m and re-rotating the mean at t0 + (L-1)/2 is
    one rotation by (L-1)/2 - m: the absolute start cancels, which is why a
    summary can be formed with one offset table for every span.
    """
    rng = np.random.default_rng(17)
    k_rot = rng.standard_normal((16, 32))
    base = O.span_summary(k_rot, 0, 5, 1e4)
    for t0 in (1, 48, 1000, 65536):
        np.testing.assert_allclose(O.span_summary(k_rot, t0, 5, 1e4), base, atol=1e-9)


def test_build_summaries_leaves_incomplete_rows_undefined():
    prm = _params()
    k = np.random.default_rng(7).standard_normal((64, 16))
    cs, gs = O.build_summaries(k, prm, n_valid=37)
    assert np.isfinite(cs[:2]).all() and np.isnan(cs[2:]).all()   # chunks 0-1 end at 31
    assert np.isfinite(gs[2, 0]).all() and np.isnan(gs[2, 1]).all()  # group 8 ends at 35, 9 at 39


# --------------------------------------------------------------------- routing

def _brute_top(ids, score_of, k):
    """Best k-subset by total score; ties to the lexicographically smallest sorted ids."""
    best, best_key = None, None
    for sub in itertools.combinations(sorted(ids), min(k, len(ids))):
        key = (-sum(score_of(i) for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(best) + [-1] * (k - len(best))


@pytest.mark.parametrize("seed", range(6))
def test_chunk_routing_matches_brute_force(seed):
    """Level-1 selection equals the best-total-score subset of candidate chunks.

    Scores are recomputed per query head and summed, not from the mean query,
    so the GQA aggregation is checked too (the mean ranks like the sum).
    """
    rng = np.random.default_rng(100 + seed)
    prm = _params(topk_chunks=int(rng.integers(1, 5)))
    g = prm.gqa
    n = 16 * 12
    k = rng.standard_normal((n, 16))
    cs, _ = O.build_summaries(k, prm)
    q_heads = rng.standard_normal((g, 16))
    cur = 11
    got, cand, _ = O.route_chunks(O.routing_query(q_heads), cs, cur, prm)
    assert cand == list(range(prm.sink, cur - prm.local))
    want = _brute_top(cand, lambda j: sum(float(qh @ cs[j]) for qh in q_heads), prm.topk_chunks)
    assert got == want


@pytest.mark.parametrize("seed", range(4))
def test_group_routing_matches_brute_force(seed):
    rng = np.random.default_rng(200 + seed)
    prm = _params(topk_groups=int(rng.integers(1, 7)))
    k = rng.standard_normal((16 * 12, 16))
    _, gs = O.build_summaries(k, prm)
    q_heads = rng.standard_normal((prm.gqa, 16))
    chunks = [2, 5, 7]
    got, cand, _ = O.route_groups(O.routing_query(q_heads), gs, chunks + [-1], prm)
    assert cand == [c * 4 + i for c in chunks for i in range(4)]
    want = _brute_top(cand, lambda gid: sum(float(qh @ gs[gid // 4, gid % 4]) for qh in q_heads),
                      prm.topk_groups)
    assert got == want


def test_routing_ties_go_to_lower_index_and_pad():
    assert O.top_k([4, 5, 6, 7], [1.0, 2.0, 2.0, 2.0], 2) == [5, 6]
    assert O.top_k([4, 5, 6], [3.0, 3.0, 3.0], 5) == [4, 5, 6, -1, -1]
    assert O.top_k([], [], 3) == [-1, -1, -1]
    assert O.top_k([9, 2], [0.0, -0.0], 1) == [2]  # +0 and -0 are equal scores


def test_forced_and_candidate_sets_of_the_tiny_workload():
    """Decode at 1023 with C=64, sink 1, local 2 (the tiny fp32 workload), from a text fixture."""
    with open(os.path.join(GOLDEN, "tiny_decode_sets.json")) as f:
        fx = json.load(f)
    prm = O.HGAParams(head_dim=64, heads_q=1, heads_kv=1, chunk=fx["C"], group=fx["g"],
                      sink=fx["sink"], local=fx["local"], topk_chunks=fx["kc"], topk_groups=fx["kg"])
    cur = fx["pos"] // fx["C"]
    assert cur == fx["cur"]
    assert O.forced_chunks(cur, prm) == fx["forced_chunks"]
    assert O.candidate_chunks(cur, prm) == fx["candidate_chunks"]
    groups = list(range(8, 8 + fx["kg"]))  # any kg groups of candidate chunks
    assert len(O.visible_tokens(fx["pos"], cur, groups, prm)) == fx["visible_tokens"]


@pytest.mark.parametrize("cur,sink,local", [(0, 1, 4), (2, 1, 4), (5, 3, 1), (5, 0, 0), (40, 2, 3)])
def test_forced_chunks_always_visible(cur, sink, local):
    prm = _params(sink=sink, local=local)
    forced = set(O.forced_chunks(cur, prm))
    assert cur in forced
    assert set(range(min(sink, cur + 1))) <= forced
    assert set(range(max(0, cur - local), cur + 1)) <= forced
    assert not forced & set(O.candidate_chunks(cur, prm))


# ---------------------------------------------------------- whole path vs dense

def _dense_causal(q, k, v, q_pos, mask_fn=None):
    """Dense attention through torch's SDPA in float64 (query head hq reads KV head hq // G)."""
    hq, lq, d = q.shape
    g = hq // k.shape[0]
    kk = torch.from_numpy(np.repeat(k, g, axis=0))[None]
    vv = torch.from_numpy(np.repeat(v, g, axis=0))[None]
    n = k.shape[1]
    allowed = np.arange(n)[None, :] <= np.asarray(q_pos)[:, None]
    if mask_fn is not None:
        allowed = allowed & mask_fn()
    mask = torch.from_numpy(np.broadcast_to(allowed, (hq, lq, n)).copy())[None]
    out = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[None], kk, vv,
                                                           attn_mask=mask)
    return out[0].numpy()


@pytest.mark.parametrize("n,pos", [(256, 255), (256, 200), (256, 70), (256, 5)])
def test_full_coverage_decode_equals_dense_causal(n, pos):
    """With top-k covering every candidate, the routed layer is dense causal attention."""
    prm = _params(topk_chunks=100, topk_groups=1000)
    rng = np.random.default_rng(pos)
    q = rng.standard_normal((4, 1, 16))
    k = rng.standard_normal((2, n, 16))
    v = rng.standard_normal((2, n, 16))
    res = O.hga_layer(q, k, v, pos, prm)
    np.testing.assert_allclose(res["out"], _dense_causal(q, k, v, [pos]), atol=1e-12)


def test_full_coverage_prefill_equals_dense_causal():
    prm = _params(topk_chunks=100, topk_groups=1000)
    rng = np.random.default_rng(9)
    n = 128
    q = rng.standard_normal((4, n, 16))
    k = rng.standard_normal((2, n, 16))
    v = rng.standard_normal((2, n, 16))
    res = O.hga_layer(q, k, v, n - 1, prm)
    np.testing.assert_allclose(res["out"], _dense_causal(q, k, v, np.arange(n)), atol=1e-12)


@pytest.mark.parametrize("prefill", [False, True])
def test_routed_layer_equals_masked_dense_attention(prefill):
    """Sparse routing: the output is dense attention under the mask of the routed sets.

    The mask is rebuilt here from the routed ids by chunk / group membership,
    independently of the oracle's token-list construction.
    """
    prm = _params(topk_chunks=2, topk_groups=3)
    rng = np.random.default_rng(11)
    n = 16 * 10
    lq = n if prefill else 1
    q = rng.standard_normal((4, lq, 16))
    k = rng.standard_normal((2, n, 16))
    v = rng.standard_normal((2, n, 16))
    res = O.hga_layer(q, k, v, n - 1, prm)
    q_pos = np.arange(n - lq, n)
    t = np.arange(n)
    for h in range(2):
        def mask_fn():
            m = np.zeros((lq, n), dtype=bool)
            for r, p in enumerate(q_pos):
                cur = p // prm.chunk
                blk = 0 if lq == 1 else cur
                gsel = res["group_idx"][h, blk]
                c = t // prm.chunk
                m[r] = (c < prm.sink) | (c >= cur - prm.local) | np.isin(t // prm.group, gsel[gsel >= 0])
            return m
        want = _dense_causal(q[2 * h:2 * h + 2], k[h:h + 1], v[h:h + 1], q_pos, mask_fn)
        np.testing.assert_allclose(res["out"][2 * h:2 * h + 2], want, atol=1e-12)


def test_attention_weights_sum_to_one_and_lse():
    rng = np.random.default_rng(12)
    k = rng.standard_normal((50, 8))
    v = rng.standard_normal((50, 8))
    q = rng.standard_normal(8) * 3
    toks = np.array([0, 3, 4, 17, 49])
    o, lse, w = O.attend(q, k, v, toks)
    assert w.sum() == pytest.approx(1.0, abs=1e-14)
    assert lse == pytest.approx(math.log(sum(math.exp(k[t] @ q / math.sqrt(8)) for t in toks)))
    np.testing.assert_allclose(o, w @ v[toks], atol=1e-14)


def test_routed_selection_contains_forced_and_respects_k():
    prm = _params(topk_chunks=3, topk_groups=4)
    rng = np.random.default_rng(13)
    n = 16 * 20
    q = rng.standard_normal((4, 1, 16))
    k = rng.standard_normal((2, n, 16))
    v = rng.standard_normal((2, n, 16))
    res = O.hga_layer(q, k, v, n - 1, prm)
    cur = (n - 1) // 16
    for h in range(2):
        cidx = res["chunk_idx"][h, 0]
        gidx = res["group_idx"][h, 0]
        assert list(cidx) == sorted(cidx) and len(set(cidx)) == 3
        assert all(prm.sink <= c < cur - prm.local for c in cidx)
        assert set(g // 4 for g in gidx) <= set(cidx)
        toks = O.visible_tokens(n - 1, cur, gidx, prm)
        for c in O.forced_chunks(cur, prm):
            assert set(range(c * 16, min((c + 1) * 16, n))) <= set(toks)
        assert len(toks) == (1 + 2 + 1) * 16 + 4 * 4


def test_needle_chunks_are_routed():
    """Planted needle chunks (keys at cosine 0.9 to the query) are selected (sanity, not parity)."""
    import hga_synth as S
    wl = S.workload("llama3_8b_decode_32k", batch=1, context=4096, heads_kv=2, heads_q=8)
    x = S.make_inputs(wl, seed=7)
    prm = O.HGAParams(head_dim=128, heads_q=8, heads_kv=2, n_high_pairs=32, rope_theta=5e5)
    q = S.widen(x["q"][0], wl.dtype)
    k = S.widen(x["k"][0], wl.dtype)
    v = S.widen(x["v"][0], wl.dtype)
    res = O.hga_layer(q, k, v, wl.context - 1, prm)
    for h in range(2):
        needles = S.needle_chunks(wl, 7, 0, h)
        assert len(needles) == 2
        assert set(needles) <= set(res["chunk_idx"][h, 0])
