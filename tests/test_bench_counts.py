"""The roofline numerators of bench.py against the oracle's visible token sets.

bench.py counts algorithmic bytes (decode) and FLOPs (prefill) from closed forms;
here those counts are checked against the token sets the oracle builds, query by
query, for a routing that fills every level-1 and level-2 slot.
"""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import hga_synth as S  # noqa: E402
from oracle import hga_oracle as O  # noqa: E402


def params(wl):
    return O.HGAParams(head_dim=wl.head_dim, heads_q=wl.heads_q, heads_kv=wl.heads_kv,
                       chunk=wl.chunk, group=wl.group, sink=wl.sink, local=wl.local,
                       topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                       n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta)


def full_routing(prm, cur):
    """The first kc candidate chunks and the first kg of their groups."""
    ng = prm.chunk // prm.group
    chunks = list(range(prm.sink, max(prm.sink, cur - prm.local)))[:prm.topk_chunks]
    return chunks, [c * ng + i for c in chunks for i in range(ng)][:prm.topk_groups]


@pytest.mark.parametrize("name,kw", [("llama3_8b_decode_32k", {}),
                                     ("wide_head_decode_64k", dict(chunk=128, topk_chunks=32,
                                                                   topk_groups=64))])
def test_decode_bytes_cover_the_oracle_token_set(name, kw):
    wl = S.workload(name, **kw)
    prm = params(wl)
    p = wl.context - 1
    cur = p // wl.chunk
    chunks, groups = full_routing(prm, cur)
    toks = O.visible_tokens(p, cur, groups, prm)
    nb = bench.step_bytes(wl)
    assert nb["tokens"] == len(toks)
    units = wl.batch * wl.heads_kv
    e = 2 if wl.dtype == "bf16" else 4
    kv = units * len(toks) * wl.head_dim * e * 2
    assert kv <= nb["attend"] <= kv * 1.02          # K/V rows dominate, plus q, out, ids
    n_cand = cur - wl.local - wl.sink
    rows = units * n_cand * wl.head_dim * 4           # every candidate chunk summary, fp32
    assert rows <= nb["route_chunks"] <= rows * 1.02
    g_rows = units * len(chunks) * (wl.chunk // wl.group) * wl.head_dim * 4
    assert g_rows <= nb["route_groups"] <= g_rows * 1.1


def test_prefill_flops_count_the_oracle_visible_pairs():
    wl = S.workload("llama3_8b_prefill_64k", context=2048, heads_q=8, heads_kv=2)
    prm = params(wl)
    pairs = 0
    for blk in range(wl.context // wl.chunk):
        _, groups = full_routing(prm, blk)
        for i in range(wl.chunk):
            pairs += len(O.visible_tokens(blk * wl.chunk + i, blk, groups, prm))
    pairs *= wl.heads_q * wl.batch     # every query head of every sequence
    assert bench.prefill_flops(wl) == 4.0 * wl.head_dim * pairs
