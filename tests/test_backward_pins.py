"""Pins of the backward-pass oracle (oracle/hga_backward.py) against facts fixed
outside itself: torch autograd in float64 through a dense attention under a mask
rebuilt here from the routed ids, central finite differences of the oracle's own
forward, the dense causal limit, and the closed form of the summed value
gradients.  HGA technical summary, "Meccanismo Core", item 4 (exact attention
over the selected tokens) and "Risultati Sperimentali" (trained end to end).
"""

import numpy as np
import pytest
import torch

from oracle import hga_backward as BW
from oracle import hga_oracle as O


def _params(**kw):
    base = dict(head_dim=16, heads_q=4, heads_kv=2, chunk=16, group=4, sink=1, local=2,
                topk_chunks=2, topk_groups=3, n_high_pairs=4, rope_theta=100.0)
    base.update(kw)
    return O.HGAParams(**base)


def _inputs(seed, lq, n, d=16, hq=4, hkv=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((hq, lq, d)), rng.standard_normal((hkv, n, d)),
            rng.standard_normal((hkv, n, d)), rng.standard_normal((hq, lq, d)))


def _mask(prm, group_idx, lq, n, h):
    """Visibility of every (query row, token) for KV head h, from chunk / group
    membership of the routed ids (not from the oracle's token lists)."""
    q_pos = np.arange(n - lq, n)
    t = np.arange(n)
    c = t // prm.chunk
    m = np.zeros((lq, n), dtype=bool)
    for r, p in enumerate(q_pos):
        cur = p // prm.chunk
        blk = 0 if lq == 1 else cur
        gsel = np.asarray(group_idx[h][blk])
        m[r] = ((c < prm.sink) | (c >= cur - prm.local) |
                np.isin(t // prm.group, gsel[gsel >= 0])) & (t <= p)
    return m


def _autograd(q, k, v, d_out, masks):
    """dq, dk, dv of sum(out * d_out) for masked dense attention, by torch autograd."""
    hq, lq, d = q.shape
    hkv = k.shape[0]
    g = hq // hkv
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    outs = []
    for hh in range(hq):
        h = hh // g
        s = qt[hh] @ kt[h].T / np.sqrt(d)
        s = s.masked_fill(~torch.from_numpy(masks[h]), float("-inf"))
        outs.append(torch.softmax(s, dim=-1) @ vt[h])
    loss = (torch.stack(outs) * torch.from_numpy(d_out)).sum()
    loss.backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("prefill", [False, True])
def test_backward_equals_autograd_of_masked_dense_attention(prefill):
    prm = _params()
    n = 16 * 10
    lq = n if prefill else 1
    q, k, v, dout = _inputs(21 + lq, lq, n)
    res = O.hga_layer(q, k, v, n - 1, prm)
    gi = res["group_idx"]
    dq, dk, dv = BW.hga_layer_backward(q, k, v, n - 1, prm, gi, dout)
    masks = [_mask(prm, gi, lq, n, h) for h in range(2)]
    rq, rk, rv = _autograd(q, k, v, dout, masks)
    np.testing.assert_allclose(dq, rq, atol=1e-11)
    np.testing.assert_allclose(dk, rk, atol=1e-11)
    np.testing.assert_allclose(dv, rv, atol=1e-11)


def test_backward_equals_dense_causal_gradients_when_routing_keeps_everything():
    prm = _params(topk_chunks=100, topk_groups=1000)
    n = 64
    q, k, v, dout = _inputs(5, n, n)
    res = O.hga_layer(q, k, v, n - 1, prm)
    dq, dk, dv = BW.hga_layer_backward(q, k, v, n - 1, prm, res["group_idx"], dout)
    qt = torch.tensor(q[None], requires_grad=True)
    kt = torch.tensor(np.repeat(k, 2, axis=0)[None], requires_grad=True)
    vt = torch.tensor(np.repeat(v, 2, axis=0)[None], requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    (out * torch.from_numpy(dout[None])).sum().backward()
    np.testing.assert_allclose(dq, qt.grad[0].numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad[0].numpy().reshape(2, 2, n, 16).sum(1), atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad[0].numpy().reshape(2, 2, n, 16).sum(1), atol=1e-11)


def test_backward_matches_finite_differences_of_the_forward():
    """Central differences of sum(out * d_out) through the oracle's forward with the
    index sets held fixed (the routing is a selection, not a function to differentiate)."""
    prm = _params(head_dim=8, n_high_pairs=2)
    n = 64
    q, k, v, dout = _inputs(8, n, n, d=8)
    gi = O.hga_layer(q, k, v, n - 1, prm)["group_idx"]
    dq, dk, dv = BW.hga_layer_backward(q, k, v, n - 1, prm, gi, dout)

    def loss(qq, kk, vv):
        out = O.hga_layer(qq, kk, vv, n - 1, prm, group_idx_override=gi)["out"]
        return float((out * dout).sum())

    rng = np.random.default_rng(3)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            lp = loss(*[xp if a is x else a for a in args])
            lm = loss(*[xm if a is x else a for a in args])
            assert abs((lp - lm) / (2 * eps) - grad[idx]) < 1e-6, (name, idx)


def test_value_gradients_sum_to_the_summed_output_gradients():
    """Every row's weights sum to one, so summing dV over all tokens gives the sum
    of d_out over the rows (and heads) of each KV head."""
    prm = _params()
    n = 16 * 8
    q, k, v, dout = _inputs(13, n, n)
    gi = O.hga_layer(q, k, v, n - 1, prm)["group_idx"]
    _, dk, dv = BW.hga_layer_backward(q, k, v, n - 1, prm, gi, dout)
    for h in range(2):
        np.testing.assert_allclose(dv[h].sum(0), dout[2 * h:2 * h + 2].sum((0, 1)), atol=1e-10)
    # and the score gradients of each row sum to zero: shifting every key of a
    # row's set by the same vector leaves its output unchanged, so for decode
    # (one row, one set) the key gradients sum to zero
    qd, kd, vd, dd = _inputs(14, 1, n)
    gd = O.hga_layer(qd, kd, vd, n - 1, prm)["group_idx"]
    _, dkd, _ = BW.hga_layer_backward(qd, kd, vd, n - 1, prm, gd, dd)
    np.testing.assert_allclose(dkd.sum(1), 0.0, atol=1e-12)
