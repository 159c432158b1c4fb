"""Float64 CPU oracle of the HGA attention's backward pass over fixed index sets.

TEST INFRASTRUCTURE ONLY.  The test suite and the benchmark's CPU leg are the
only callers allowed; the product never imports or runs this module, and this
module imports nothing from the product.

What it restates
----------------
The technical summary of "Hierarchical Global Attention (HGA)" (gist.science,
paper 2606.30709; Italian page "Riepilogo Tecnico", "Risultati Sperimentali"
and "Contributi Chiave") reports training and fine-tuning through the method:
the layer is trained end to end.  Its output is an exact softmax attention over
a token set that the routing selects ("Meccanismo Core", item 4); the routing
is a selection (top-k of summary scores), so no gradient flows through it or
through the summaries, and the gradients of the layer are those of softmax
attention restricted to each query's selected set.  For one query row q with
visible tokens T, s = K_T q / sqrt(D), w = softmax(s), o = w V_T, and an
upstream gradient do:

    dV_T += w (x) do
    dw    = V_T do
    ds    = w * (dw - do . o)
    dq    = K_T^T ds / sqrt(D)
    dK_T += ds (x) q / sqrt(D)

summed over the G query heads that share a KV head and over every query row.

Pinned by tests/test_backward_pins.py: torch autograd (float64) through a dense
attention under an independently rebuilt mask, central finite differences, the
dense causal limit when the routing keeps everything, and the closed form of
the sum of the value gradients.
"""

from __future__ import annotations

import math

import numpy as np

from . import hga_oracle as O


def attend_backward(q_vec, k, v, tokens, d_out):
    """Gradients of one query row's attention output o (over `tokens`) given
    the upstream gradient d_out: returns (dq [D], dk_rows [T, D], dv_rows [T, D]),
    the rows in the order of `tokens`."""
    q_vec = np.asarray(q_vec, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    kk = np.asarray(k[tokens], dtype=np.float64)
    vv = np.asarray(v[tokens], dtype=np.float64)
    scale = 1.0 / math.sqrt(q_vec.shape[0])
    o, _, w = O.attend(q_vec, k, v, tokens)
    dv = np.outer(w, d_out)
    dw = vv @ d_out
    ds = w * (dw - float(d_out @ o))
    dq = (kk.T @ ds) * scale
    dk = np.outer(ds, q_vec) * scale
    return dq, dk, dv


def hga_layer_backward(q, k, v, pos_last: int, prm: O.HGAParams, group_idx, d_out):
    """dq [Hq, Lq, D], dk and dv [Hkv, N, D] of the layer output of hga_layer over
    the index sets group_idx [Hkv, nblk, kg] (the routed groups of each query
    block), for the upstream gradient d_out [Hq, Lq, D]."""
    q = np.asarray(q, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    hq, lq, d = q.shape
    hkv, n = k.shape[0], k.shape[1]
    g = hq // hkv
    dq = np.zeros_like(q)
    dk = np.zeros((hkv, n, d))
    dv = np.zeros((hkv, n, d))
    first_pos = pos_last - lq + 1
    for h in range(hkv):
        kh = np.asarray(k[h], dtype=np.float64)
        vh = np.asarray(v[h], dtype=np.float64)
        for bi, (r0, nr, cur) in enumerate(O.query_blocks(lq, pos_last, prm.chunk)):
            groups = group_idx[h][bi]
            for r in range(r0, r0 + nr):
                toks = O.visible_tokens(first_pos + r, cur, groups, prm)
                for hh in range(h * g, (h + 1) * g):
                    gq, gk, gv = attend_backward(q[hh, r], kh, vh, toks, d_out[hh, r])
                    dq[hh, r] = gq
                    dk[h, toks] += gk
                    dv[h, toks] += gv
    return dq, dk, dv
