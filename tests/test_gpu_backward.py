"""Backward pass of the prefill attention over the routed index sets.

Both sides get the same inputs, the oracle's routing included: the GPU forward
(hga_attend) and backward (hga_attend_backward) against the float64 oracle
(oracle/hga_backward.py).  Also: groups routed by more query blocks than one
work item takes (the split and fixed-order reduce), keys no query sees,
a prompt continuing a cache, the closed-form sum of the value gradients, and
bit-identical repeated runs.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import layer_of, params_of, to_device  # noqa: E402
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402
from oracle import hga_backward as BW  # noqa: E402
from oracle import hga_oracle as O  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def _wl(**kw):
    base = dict(batch=1, heads_q=8, heads_kv=2, context=2048, topk_chunks=4, topk_groups=8,
                local=2, needles=0)
    base.update(kw)
    return S.workload("llama3_8b_prefill_64k", **base)


def _oracle_routing(wl, x, b):
    """The oracle's group_idx [Hkv, nblk, kg] of sequence b (prefill of the whole context)."""
    prm = params_of(wl)
    q = S.widen(x["q"][b], wl.dtype)
    k = S.widen(x["k"][b], wl.dtype)
    v = S.widen(x["v"][b], wl.dtype)
    return O.hga_layer(q, k, v, wl.context - 1, prm)["group_idx"]


def _with_hot_group(gi, wl, hot):
    """Adds group `hot` to every block's selection where it is a candidate (a key
    group that most blocks route), keeping each row ascending and -1 padded."""
    gi = gi.copy()
    gpc = wl.chunk // wl.group
    for h in range(gi.shape[0]):
        for j in range(gi.shape[1]):
            if not (wl.sink <= hot // gpc < j - wl.local):
                continue
            row = [int(x) for x in gi[h, j] if x >= 0]
            if hot not in row:
                row = sorted(set(row[:-1] + [hot])) if len(row) == wl.topk_groups else sorted(row + [hot])
            gi[h, j] = row + [-1] * (wl.topk_groups - len(row))
    return gi


def _run(wl, x, gi, q_len=None, seed=0):
    """GPU forward (out f32, lse) and backward on group_idx gi [B, Hkv, nblk, kg]."""
    q_len = q_len or wl.context
    n = wl.context
    layer = layer_of(wl, B.HGA_F32)
    q = to_device(x["q"], wl.dtype)
    k = to_device(x["k"], wl.dtype)
    v = to_device(x["v"], wl.dtype)
    pos = torch.full((wl.batch,), n - 1, dtype=torch.int64, device="cuda")
    g = torch.as_tensor(gi, dtype=torch.int32, device="cuda").contiguous()
    out = torch.empty(wl.batch, wl.heads_q, q_len, wl.head_dim, device="cuda")
    lse = torch.empty(wl.batch, wl.heads_q, q_len, device="cuda")
    wsb = B.hga_workspace_size(layer, n, q_len)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    B.hga_attend(layer, q, q_len, pos, k, v, n, g, out, lse, ws, wsb)
    rng = np.random.default_rng(seed)
    dout_np = S.store(rng.standard_normal((wl.batch, wl.heads_q, q_len, wl.head_dim)).astype(np.float32),
                      wl.dtype)
    dout = to_device(dout_np, wl.dtype)
    dq = torch.full((wl.batch, wl.heads_q, q_len, wl.head_dim), float("nan"), device="cuda")
    dk = torch.full((wl.batch, wl.heads_kv, n, wl.head_dim), float("nan"), device="cuda")
    dv = torch.full_like(dk, float("nan"))
    bwb = B.hga_attend_backward_workspace_size(layer, n, q_len)
    bws = torch.empty(bwb, dtype=torch.uint8, device="cuda")
    B.hga_attend_backward(layer, q, q_len, pos, k, v, n, g, out, lse, dout, dq, dk, dv, bws, bwb)
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    return dict(dq=dq.cpu().numpy(), dk=dk.cpu().numpy(), dv=dv.cpu().numpy(), dout=dout_np,
                again=lambda: (B.hga_attend_backward(layer, q, q_len, pos, k, v, n, g, out, lse,
                                                     dout, dq, dk, dv, bws, bwb),
                               torch.cuda.synchronize(),
                               (dq.clone(), dk.clone(), dv.clone()))[2])


def _close(got, want, what, rel=1e-2):
    err = float(np.max(np.abs(got - want)))
    scale = float(np.max(np.abs(want)))
    assert err <= rel * scale, f"{what}: max-abs {err:.3e} vs {rel} x {scale:.3e}"


@pytest.mark.parametrize("hot", [False, True])
def test_backward_matches_the_oracle(hot):
    """2048 tokens in 32 blocks: sink groups (seen by every block) and, with hot,
    a group routed by every later block, both split over several work items."""
    wl = _wl()
    x = S.make_inputs(wl, 81)
    gi = _oracle_routing(wl, x, 0)
    if hot:
        gi = _with_hot_group(gi, wl, hot=2 * (wl.chunk // wl.group) + 1)
    r = _run(wl, x, gi[None])
    prm = params_of(wl)
    dq, dk, dv = BW.hga_layer_backward(S.widen(x["q"][0], wl.dtype), S.widen(x["k"][0], wl.dtype),
                                       S.widen(x["v"][0], wl.dtype), wl.context - 1, prm, gi,
                                       S.widen(r["dout"][0], wl.dtype))
    _close(r["dq"][0], dq, "dq")
    _close(r["dk"][0], dk, "dk")
    _close(r["dv"][0], dv, "dv")
    again = r["again"]()   # a second run: the same bits (fixed summation order)
    for t0, name in zip(again, ("dq", "dk", "dv")):
        assert np.array_equal(t0.cpu().numpy().view(np.int32), r[name].view(np.int32)), name


def test_backward_of_a_prompt_continuing_a_cache():
    """The last 8 chunks of a 1024-token cache as queries: keys before them get
    gradients only where some block sees them; the rest are exactly zero."""
    wl = _wl(context=1024)
    x = S.make_inputs(wl, 82)
    q_len = 512
    xq = dict(x, q=np.ascontiguousarray(x["q"][:, :, -q_len:]))
    prm = params_of(wl)
    q = S.widen(xq["q"][0], wl.dtype)
    k = S.widen(x["k"][0], wl.dtype)
    v = S.widen(x["v"][0], wl.dtype)
    gi = O.hga_layer(q, k, v, wl.context - 1, prm)["group_idx"]
    r = _run(wl, xq, gi[None], q_len=q_len)
    dq, dk, dv = BW.hga_layer_backward(q, k, v, wl.context - 1, prm, gi,
                                       S.widen(r["dout"][0], wl.dtype))
    _close(r["dq"][0], dq, "dq")
    _close(r["dk"][0], dk, "dk")
    _close(r["dv"][0], dv, "dv")
    unseen = np.all(dk == 0.0, axis=-1) & np.all(dv == 0.0, axis=-1)
    assert unseen.any()
    assert (r["dk"][0][unseen] == 0.0).all() and (r["dv"][0][unseen] == 0.0).all()


def test_value_gradients_sum_to_the_output_gradients_at_8k():
    """At 8192 tokens and 4 sequences: per KV head, the value gradients summed over
    all keys equal the output gradients summed over its rows and heads (every
    softmax row sums to one); no NaN anywhere."""
    wl = _wl(batch=4, context=8192, heads_q=16, heads_kv=4, topk_chunks=16, topk_groups=32,
             local=4)
    x = S.make_inputs(wl, 83)
    layer = layer_of(wl, B.HGA_F32)
    q = to_device(x["q"], wl.dtype)
    pos = torch.full((wl.batch,), wl.context - 1, dtype=torch.int64, device="cuda")
    cs = torch.empty(wl.batch * wl.heads_kv, wl.context // wl.chunk, wl.head_dim, device="cuda")
    gs = torch.empty(wl.batch * wl.heads_kv, wl.context // wl.chunk, wl.chunk // wl.group,
                     wl.head_dim, device="cuda")
    k = to_device(x["k"], wl.dtype)
    B.hga_build_summaries(layer, k, wl.context, 0, wl.context, cs, gs)
    nblk = wl.context // wl.chunk
    ci = torch.empty(wl.batch * wl.heads_kv * nblk, wl.topk_chunks, dtype=torch.int32, device="cuda")
    gi = torch.empty(wl.batch * wl.heads_kv * nblk, wl.topk_groups, dtype=torch.int32, device="cuda")
    B.hga_route(layer, q, wl.context, pos, cs, gs, wl.context, ci, gi)
    torch.cuda.synchronize()
    gi_np = gi.cpu().numpy().reshape(wl.batch, wl.heads_kv, nblk, wl.topk_groups)
    r = _run(wl, x, gi_np)
    for name in ("dq", "dk", "dv"):
        assert np.isfinite(r[name]).all(), name
    dout = S.widen(r["dout"], wl.dtype).reshape(wl.batch, wl.heads_kv, wl.gqa, wl.context, -1)
    want = dout.sum(axis=(2, 3))
    got = r["dv"].astype(np.float64).sum(axis=2)
    assert np.max(np.abs(got - want)) <= 1e-2 * np.max(np.abs(want))
