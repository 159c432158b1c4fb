"""Float64 CPU oracle of the Hierarchical Global Attention (HGA) hot path.

TEST INFRASTRUCTURE ONLY.  The test suite, the package ``smoke()`` check and the
CPU-baseline leg of the benchmark are the only callers allowed.  The product
(the CUDA library and its Python binding) never imports or runs this module,
and this module imports nothing from the product.  Both sides only share the
seeded input generator, which holds none of the method's arithmetic.

What it restates
----------------
The technical summary of "Hierarchical Global Attention (HGA)" (gist.science,
paper 2606.30709; Italian page "Riepilogo Tecnico", section "Metodologia ->
Meccanismo Core", items 1-4, and the same list on the French page "Resume
Technique -> Mecanisme Central"):

1. Partitioning: the sequence is cut into fixed-size chunks of C tokens, and
   each chunk into groups.
2. Hierarchical routing: level 1 scores the current query against a table of
   chunk key summaries of earlier chunks; level 2 scores the groups inside the
   selected chunks.  The current chunk, a configurable number of initial sink
   chunks and the recent local chunks are always visible.
3. RoPE-aware summaries: high-frequency RoPE pairs are rotated per token and
   then averaged; low-frequency pairs are averaged as raw keys and rotated at
   the chunk's representative position.  No new layers.
4. Exact token attention: the original K/V of the selected tokens enter a
   standard softmax; no summary value reaches the output.

Routing is a heuristic, so this file takes the algorithm's steps in that order,
written plainly in float64 with no blocking, fusion or reordering.

Readings where the pages are silent (each one is listed in the design notes):

R1  RoPE pairs use the rotate-half layout: pair i is dims (i, i + D/2) and
    turns by angle t * omega_i with omega_i = theta^(-2i/D).  No RoPE scaling.
R2  "High-frequency" pairs are the first ``n_high_pairs`` pairs (largest omega).
R3  The representative position of a chunk or group spanning tokens
    t0..t0+L-1 is its centre t0 + (L-1)/2.
R4  "Average" is the arithmetic mean over all tokens of a complete chunk/group.
R5  Stored keys are post-RoPE; the raw key of token t is R(-t) k_rot[t].
R6  The routing query is the mean of the post-RoPE query vectors of the G
    query heads that share the KV head (and, for a prefill block, of the
    block's queries).  Query head hq reads KV head hq // G.
R7  Level-1 candidates are the complete chunks j with sink <= j < cur - local;
    the forced chunks {0..sink-1} U {cur-local..cur} are added outside top-k.
R8  Ties go to the lower index; selections are returned in ascending order,
    padded with -1 when fewer than k candidates exist.
R9  Level 2 is one top-kg over all groups of the selected chunks; a group is
    named by its global id chunk * (C / g) + group-in-chunk.
R10 cur = pos // C.  Tokens after the query position are never visible.  A
    prefill block is one chunk of C queries routed together.
R11 Softmax scale 1/sqrt(D), natural-log LSE, no bias.

Pinned by tests/test_oracle_pins.py (dense-attention limit, closed-form
summaries, library RoPE, brute-force routing, invariants).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class HGAParams:
    """Method parameters of one attention layer (names follow the pages' notation)."""

    head_dim: int            # D
    heads_q: int             # Hq
    heads_kv: int            # Hkv (GQA: G = Hq / Hkv query heads per KV head)
    chunk: int = 64          # C, fixed chunk size (core mechanism, item 1)
    group: int = 16          # g, tokens per group inside a chunk
    sink: int = 1            # initial "sink" chunks that are always visible
    local: int = 4           # recent local chunks that are always visible
    topk_chunks: int = 16    # kc, level-1 top-k
    topk_groups: int = 32    # kg, level-2 top-k
    n_high_pairs: int = 32   # RoPE pairs averaged after per-token rotation
    rope_theta: float = 10000.0

    @property
    def gqa(self) -> int:
        return self.heads_q // self.heads_kv

    @property
    def groups_per_chunk(self) -> int:
        return self.chunk // self.group


# ---------------------------------------------------------------- RoPE (R1, R2)

def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """omega_i = theta^(-2i/D) for the D/2 rotation pairs (R1)."""
    pairs = head_dim // 2
    return np.power(float(theta), -2.0 * np.arange(pairs, dtype=np.float64) / head_dim)


def rope_apply(x: np.ndarray, positions, theta: float) -> np.ndarray:
    """Rotate the rows x[..., T, D] to positions[T] (rotate-half pairing, R1).

    Positions may be fractional or negative; a negative position undoes the
    rotation of the matching positive one.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    p = d // 2
    ang = np.asarray(positions, dtype=np.float64).reshape(-1, 1) * rope_inv_freq(d, theta)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :p], x[..., p:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def high_freq_dims(head_dim: int, n_high_pairs: int) -> np.ndarray:
    """Boolean mask over the D dims: True where the pair is high-frequency (R2)."""
    p = head_dim // 2
    pair_is_high = np.arange(p) < n_high_pairs
    return np.concatenate([pair_is_high, pair_is_high])


# ------------------------------------------------------ summaries (item 3, R3-R5)

def span_summary(k_rot_span: np.ndarray, t0: int, n_high_pairs: int, theta: float) -> np.ndarray:
    """Mixed RoPE-aware key summary of the contiguous tokens t0 .. t0+L-1.

    High-frequency pairs: the stored keys are already rotated per token, so
    they are averaged as they are.  Low-frequency pairs: each key is brought
    back to raw key space at its own absolute position, the raw keys are
    averaged, and the mean is rotated at the span's representative position.
    """
    k_rot_span = np.asarray(k_rot_span, dtype=np.float64)
    length, d = k_rot_span.shape
    positions = t0 + np.arange(length, dtype=np.float64)
    centre = t0 + (length - 1) / 2.0                                # R3
    mean_rotated = k_rot_span.mean(axis=0)                           # high pairs
    raw = rope_apply(k_rot_span, -positions, theta)                  # R5: undo RoPE
    mean_raw = raw.mean(axis=0)                                      # R4
    low_part = rope_apply(mean_raw[None, :], [centre], theta)[0]     # rotate at centre
    return np.where(high_freq_dims(d, n_high_pairs), mean_rotated, low_part)


def build_summaries(k_rot: np.ndarray, prm: HGAParams, n_valid: int | None = None):
    """Chunk and group summary tables of one (sequence, KV head).

    k_rot: [N, D] post-RoPE keys, token t at position t.
    Returns (chunk_sum [Nc, D], group_sum [Nc, C/g, D]) with Nc = N // C.
    Rows whose tokens are not all below ``n_valid`` are NaN (not yet complete).
    """
    k_rot = np.asarray(k_rot, dtype=np.float64)
    n, d = k_rot.shape
    n_valid = n if n_valid is None else n_valid
    nc = n // prm.chunk
    ng = prm.groups_per_chunk
    chunk_sum = np.full((nc, d), np.nan)
    group_sum = np.full((nc, ng, d), np.nan)
    for c in range(nc):
        c0 = c * prm.chunk
        if c0 + prm.chunk <= n_valid:
            chunk_sum[c] = span_summary(k_rot[c0:c0 + prm.chunk], c0, prm.n_high_pairs, prm.rope_theta)
        for gi in range(ng):
            g0 = c0 + gi * prm.group
            if g0 + prm.group <= n_valid:
                group_sum[c, gi] = span_summary(k_rot[g0:g0 + prm.group], g0, prm.n_high_pairs,
                                                prm.rope_theta)
    return chunk_sum, group_sum


# ----------------------------------------------------------------- routing (item 2)

def routing_query(q_rows: np.ndarray) -> np.ndarray:
    """R6: mean of the post-RoPE query vectors q_rows[..., D] of one KV head's block."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    return q_rows.reshape(-1, q_rows.shape[-1]).mean(axis=0)


def forced_chunks(cur: int, prm: HGAParams) -> list[int]:
    """Always-visible chunks: the sink chunks, the recent local chunks and the current one."""
    sink = set(range(0, min(prm.sink, cur + 1)))
    recent = set(range(max(0, cur - prm.local), cur + 1))
    return sorted(sink | recent)


def candidate_chunks(cur: int, prm: HGAParams) -> list[int]:
    """R7: complete chunks of the intermediate context, sink <= j < cur - local."""
    return list(range(prm.sink, max(prm.sink, cur - prm.local)))


def top_k(ids, scores, k: int) -> list[int]:
    """R8: the k best ids by score, ties to the lower id, returned ascending, -1 padded."""
    order = sorted(range(len(ids)), key=lambda i: (-scores[i], ids[i]))
    chosen = sorted(ids[i] for i in order[:k])
    return chosen + [-1] * (k - len(chosen))


def route_chunks(qbar: np.ndarray, chunk_sum: np.ndarray, cur: int, prm: HGAParams):
    """Level 1: score every candidate chunk summary against the routing query.

    Returns (selected ids [kc], candidate ids, candidate scores).
    """
    cand = candidate_chunks(cur, prm)
    scores = [float(np.dot(qbar, chunk_sum[j])) for j in cand]
    return top_k(cand, scores, prm.topk_chunks), cand, scores


def route_groups(qbar: np.ndarray, group_sum: np.ndarray, chunk_idx, prm: HGAParams):
    """Level 2 (R9): one top-kg over all groups of the selected chunks.

    Returns (selected global group ids [kg], candidate ids, candidate scores).
    """
    ng = prm.groups_per_chunk
    cand, scores = [], []
    for c in chunk_idx:
        if c < 0:
            continue
        for gi in range(ng):
            cand.append(c * ng + gi)
            scores.append(float(np.dot(qbar, group_sum[c, gi])))
    return top_k(cand, scores, prm.topk_groups), cand, scores


def visible_tokens(query_pos: int, cur: int, group_idx, prm: HGAParams) -> np.ndarray:
    """Token set of one query: forced chunks (causal at query_pos) plus the routed groups."""
    toks = set()
    for c in forced_chunks(cur, prm):
        toks.update(range(c * prm.chunk, (c + 1) * prm.chunk))
    for gid in group_idx:
        if gid >= 0:
            toks.update(range(gid * prm.group, (gid + 1) * prm.group))
    return np.array(sorted(t for t in toks if t <= query_pos), dtype=np.int64)


# ------------------------------------------------------ exact attention (item 4, R11)

def attend(q_vec: np.ndarray, k: np.ndarray, v: np.ndarray, tokens: np.ndarray):
    """Standard softmax attention of one query row over the given tokens.

    Returns (output [D], natural-log LSE of the scaled scores, weights [T]).
    """
    q_vec = np.asarray(q_vec, dtype=np.float64)
    kk = np.asarray(k[tokens], dtype=np.float64)
    vv = np.asarray(v[tokens], dtype=np.float64)
    s = kk @ q_vec / math.sqrt(q_vec.shape[0])
    m = s.max()
    e = np.exp(s - m)
    z = e.sum()
    w = e / z
    return w @ vv, m + math.log(z), w


# ------------------------------------------------------------------ whole layer

def query_blocks(q_len: int, pos_last: int, chunk: int):
    """Split the queries pos_last-q_len+1 .. pos_last into routing blocks (R10).

    Decode (q_len == 1) is one block.  Otherwise the queries must start on a
    chunk boundary and fill whole chunks; each chunk of queries is one block.
    Returns a list of (first query row, number of rows, current chunk).
    """
    first_pos = pos_last - q_len + 1
    if q_len == 1:
        return [(0, 1, pos_last // chunk)]
    if q_len % chunk or first_pos % chunk or first_pos < 0:
        raise ValueError("prefill queries must cover whole, aligned chunks")
    return [(i, chunk, (first_pos + i) // chunk) for i in range(0, q_len, chunk)]


def hga_layer(q, k, v, pos_last: int, prm: HGAParams, summaries=None, group_idx_override=None):
    """Whole HGA hot path for one sequence.

    q: [Hq, Lq, D] post-RoPE queries at positions pos_last-Lq+1 .. pos_last.
    k, v: [Hkv, N, D] post-RoPE key cache and value cache (token t at position t).
    summaries: optional (chunk_sum [Hkv, Nc, D], group_sum [Hkv, Nc, Ng, D]).
    group_idx_override: optional [Hkv, nblk, kg] index sets to attend over
        instead of the routed ones (used to check attention on a given
        selection when two routings differ only by a near-tie).

    Returns a dict with out [Hq, Lq, D], lse [Hq, Lq], chunk_idx / group_idx
    [Hkv, nblk, k] and the candidate ids/scores of every routing call.
    """
    q = np.asarray(q, dtype=np.float64)
    hq, lq, d = q.shape
    hkv = k.shape[0]
    g = hq // hkv
    n = k.shape[1]
    blocks = query_blocks(lq, pos_last, prm.chunk)
    if summaries is None:
        per_head = [build_summaries(k[h], prm, n_valid=pos_last + 1) for h in range(hkv)]
        chunk_sum = np.stack([s[0] for s in per_head])
        group_sum = np.stack([s[1] for s in per_head])
    else:
        chunk_sum, group_sum = summaries
    out = np.zeros((hq, lq, d))
    lse = np.zeros((hq, lq))
    chunk_idx = np.full((hkv, len(blocks), prm.topk_chunks), -1, dtype=np.int64)
    group_idx = np.full((hkv, len(blocks), prm.topk_groups), -1, dtype=np.int64)
    chunk_cand, group_cand = {}, {}
    first_pos = pos_last - lq + 1
    for h in range(hkv):
        kh = np.asarray(k[h], dtype=np.float64)
        vh = np.asarray(v[h], dtype=np.float64)
        for bi, (r0, nr, cur) in enumerate(blocks):
            qbar = routing_query(q[h * g:(h + 1) * g, r0:r0 + nr])
            cidx, ccand, cscore = route_chunks(qbar, chunk_sum[h], cur, prm)
            gidx, gcand, gscore = route_groups(qbar, group_sum[h], cidx, prm)
            chunk_idx[h, bi], group_idx[h, bi] = cidx, gidx
            chunk_cand[(h, bi)] = (ccand, cscore)
            group_cand[(h, bi)] = (gcand, gscore)
            use_groups = gidx if group_idx_override is None else group_idx_override[h][bi]
            for r in range(r0, r0 + nr):
                toks = visible_tokens(first_pos + r, cur, use_groups, prm)
                for hh in range(h * g, (h + 1) * g):
                    out[hh, r], lse[hh, r], _ = attend(q[hh, r], kh, vh, toks)
    assert n >= pos_last + 1
    return dict(out=out, lse=lse, chunk_idx=chunk_idx, group_idx=group_idx,
                chunk_candidates=chunk_cand, group_candidates=group_cand)
