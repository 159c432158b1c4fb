"""hga_decode_step against hga_build_summaries + hga_route + hga_attend and the oracle.

Routing of at most 64 chunks and 128 groups runs the one-launch kernel (one CTA
per SM up to one item per SM, two CTAs per SM above, each working through
items); wider routing runs the append, routing and attention kernels through the
same call.  The one-launch kernel scores with the routing
kernel's arithmetic, so the routed indices and scores must be bit-identical.  Its
warps attend the units in another grouping, so the running maxima against which P
is rounded to bf16 differ and the outputs agree to that rounding (well inside the
2e-2 output tolerance).  Every case is also checked against the float64 oracle.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import (compare_head, compare_routing_all, layer_of, sample_units,  # noqa: E402
                         to_device)
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def run_both(wl, x, out_dtype=B.HGA_F32):
    """hga_route + hga_attend, and hga_decode_step, on the same device inputs."""
    layer = layer_of(wl, out_dtype)
    n = x["k"].shape[2]
    bh, nc, ng = wl.batch * wl.heads_kv, n // wl.chunk, wl.chunk // wl.group
    q, k, v = (to_device(x[t], wl.dtype) for t in ("q", "k", "v"))
    pos = torch.as_tensor(x["pos"], dtype=torch.int64, device="cuda")
    cs = torch.full((bh, nc, wl.head_dim), float("nan"), device="cuda")
    gs = torch.full((bh, nc, ng, wl.head_dim), float("nan"), device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, cs, gs)
    odt = torch.float32 if out_dtype == B.HGA_F32 else torch.bfloat16
    res = {}
    for fused in (False, True):
        ci = torch.full((bh, 1, wl.topk_chunks), -7, dtype=torch.int32, device="cuda")
        gi = torch.full((bh, 1, wl.topk_groups), -7, dtype=torch.int32, device="cuda")
        csc = torch.empty((bh, 1, wl.topk_chunks), device="cuda")
        gsc = torch.empty((bh, 1, wl.topk_groups), device="cuda")
        out = torch.full((wl.batch, wl.heads_q, 1, wl.head_dim), 7.0, dtype=odt, device="cuda")
        lse = torch.empty((wl.batch, wl.heads_q, 1), device="cuda")
        if fused:
            B.hga_decode_step(layer, q, pos, cs, gs, n, k, v, ci, gi, out, lse, csc, gsc)
        else:
            B.hga_route(layer, q, 1, pos, cs, gs, n, ci, gi, csc, gsc)
            B.hga_attend(layer, q, 1, pos, k, v, n, gi, out, lse)
        torch.cuda.synchronize()
        assert B.hga_device_status() == 0
        shape = (wl.batch, wl.heads_kv, 1, -1)
        res[fused] = dict(chunk_idx=ci.cpu().numpy().reshape(shape),
                          group_idx=gi.cpu().numpy().reshape(shape),
                          chunk_score=csc.cpu().numpy().reshape(shape),
                          group_score=gsc.cpu().numpy().reshape(shape),
                          out=out.float().cpu().numpy(), lse=lse.cpu().numpy())
    return res[False], res[True]


def check_same_routing_close_output(sep, fus, out_tol):
    assert np.array_equal(sep["chunk_idx"], fus["chunk_idx"])
    assert np.array_equal(sep["group_idx"], fus["group_idx"])
    assert np.array_equal(np.nan_to_num(sep["chunk_score"], nan=-9.0),
                          np.nan_to_num(fus["chunk_score"], nan=-9.0))
    assert np.array_equal(np.nan_to_num(sep["group_score"], nan=-9.0),
                          np.nan_to_num(fus["group_score"], nan=-9.0))
    assert np.isfinite(fus["out"]).all()
    np.testing.assert_allclose(fus["out"], sep["out"], atol=out_tol, rtol=0)
    np.testing.assert_allclose(fus["lse"], sep["lse"], atol=1e-4, rtol=0)


@pytest.mark.parametrize("name,kw,pos", [
    ("llama3_8b_decode_32k", dict(batch=3, context=8192), None),
    ("llama3_8b_decode_32k", dict(batch=5, context=2048, heads_q=8, heads_kv=2, needles=0),
     [2047, 2047 - 37, 700, 100, 5]),
    ("llama3_8b_decode_32k", dict(batch=2, context=4096, heads_q=32, heads_kv=2), None),
    ("llama3_8b_decode_32k", dict(batch=2, context=4096, heads_q=8, heads_kv=8), None),
    ("wide_head_decode_64k", dict(batch=2, context=8192, chunk=128, topk_chunks=32,
                                  topk_groups=64), None),
])
def test_decode_step_equals_route_then_attend(name, kw, pos):
    """Group sizes G = 4, 4, 16, 1 and 8; ragged positions down to no candidates; C = 128."""
    wl = S.workload(name, **kw)
    x = S.make_inputs(wl, 31)
    if pos is not None:
        x["pos"] = np.array(pos, dtype=np.int64)
    sep, fus = run_both(wl, x)
    check_same_routing_close_output(sep, fus, 1e-2)
    for b in range(wl.batch):
        for h in sorted({0, wl.heads_kv - 1}):
            compare_head(wl, x, fus, b, h)


def test_decode_step_bf16_output_and_nan_past_query():
    """bf16 output; the cache past each query holds NaN, which must not reach the output."""
    wl = S.workload("llama3_8b_decode_32k", batch=3, context=4096, heads_q=8, heads_kv=2,
                    needles=0)
    x = S.make_inputs(wl, 32)
    x["pos"] = np.array([4000, 2100, 1234], dtype=np.int64)
    nan = np.uint16(0x7FC0)
    for b in range(3):
        x["k"][b, :, x["pos"][b] + 1:] = nan
        x["v"][b, :, x["pos"][b] + 1:] = nan
    sep, fus = run_both(wl, x, out_dtype=B.HGA_BF16)
    check_same_routing_close_output(sep, fus, 1e-2)
    for b in range(3):
        compare_head(wl, x, fus, b, 1)


def test_decode_step_llama3_8b_32k_batch16_full_size():
    """The benchmark's decode workload at full size: 32768 tokens, batch 16, planted needles."""
    wl = S.workload("llama3_8b_decode_32k")
    x = S.make_inputs(wl, S.seed_for(1))
    sep, fus = run_both(wl, x, out_dtype=B.HGA_BF16)
    check_same_routing_close_output(sep, fus, 1e-2)
    compare_routing_all(wl, S.seed_for(1), fus)   # all 128 units
    for b, h in sample_units(wl, 16, seed=2):
        compare_head(wl, x, fus, b, h)
    for b in range(wl.batch):
        for h in range(wl.heads_kv):
            assert set(S.needle_chunks(wl, S.seed_for(1), b, h)) <= set(fus["chunk_idx"][b, h, 0])


@pytest.mark.parametrize("name,kw", [
    ("llama3_8b_decode_32k", dict(batch=12, context=4096, needles=0)),
    ("wide_head_decode_64k", dict(batch=10, context=8192, chunk=128, topk_chunks=8,
                                  topk_groups=16)),
])
def test_decode_step_one_cta_per_item(name, kw):
    """Batches of up to one (sequence, KV head) item per SM (one CTA per SM); ragged
    positions, down to a sequence with no candidate chunk."""
    wl = S.workload(name, **kw)
    x = S.make_inputs(wl, 33)
    rng = np.random.default_rng(5)
    pos = rng.integers(wl.chunk, wl.context, size=wl.batch)
    pos[0], pos[1], pos[2] = wl.context - 1, 5, 2 * wl.chunk + 3
    x["pos"] = pos.astype(np.int64)
    sep, fus = run_both(wl, x)
    check_same_routing_close_output(sep, fus, 1e-2)
    for b in (0, 1, 2, wl.batch - 1):
        compare_head(wl, x, fus, b, 0)


@pytest.mark.parametrize("name,kw", [
    ("wide_head_decode_64k", dict(batch=32, context=4096)),                    # 256 items: 2 CTAs/SM
    ("wide_head_decode_64k", dict(batch=12, context=8192, topk_chunks=64, topk_groups=128)),
    ("wide_head_decode_64k", dict(batch=12, context=8192, chunk=128, topk_chunks=32,
                                  topk_groups=64)),
])
def test_decode_step_one_launch_wide_shapes(name, kw):
    """More items than SMs (persistent CTAs, two per SM), and the widest routing lists
    (top-64 chunks / top-128 groups; C = 128 with top-32 / top-64)."""
    wl = S.workload(name, **kw)
    x = S.make_inputs(wl, 34)
    rng = np.random.default_rng(6)
    pos = rng.integers(wl.chunk, wl.context, size=wl.batch)
    pos[0], pos[1] = wl.context - 1, 3 * wl.chunk + 9
    x["pos"] = pos.astype(np.int64)
    assert B.hga_decode_step_launches(layer_of(wl), wl.context) == 1
    sep, fus = run_both(wl, x)
    check_same_routing_close_output(sep, fus, 1e-2)
    for b in (0, 1, wl.batch - 1):
        compare_head(wl, x, fus, b, wl.heads_kv - 1)


@pytest.mark.parametrize("batch,kg", [(2, 32), (10, 32), (2, 256)])
def test_decode_step_append_is_bitwise_the_batch_build(batch, kg):
    """With append, hga_decode_step writes the summary rows each sequence's token closes
    (a group; a group and its chunk; nothing), bit for bit as hga_build_summaries does,
    on the one-launch kernel and on the kernel sequence (top-256 groups)."""
    wl = S.workload("llama3_8b_decode_32k", batch=batch, context=4096, needles=0,
                    topk_chunks=64 if kg > 128 else 16, topk_groups=kg)
    x = S.make_inputs(wl, 35)
    n = wl.context
    pos = np.array([n - 1, 2 * 64 * 9 + 15, 1000, 64 * 20 - 1, 64 * 33 + 47, 3000, 16 * 100 - 1,
                    64 * 50 + 31, 2048 + 63, 4000][:batch], dtype=np.int64)
    x["pos"] = pos
    layer = layer_of(wl)
    assert B.hga_decode_step_launches(layer, n) == (1 if kg <= 128 else 2)
    bh, nc, ng = wl.batch * wl.heads_kv, n // wl.chunk, wl.chunk // wl.group
    q, k, v = (to_device(x[t], wl.dtype) for t in ("q", "k", "v"))
    pos_t = torch.as_tensor(pos, device="cuda")
    full_c = torch.full((bh, nc, wl.head_dim), float("nan"), device="cuda")
    full_g = torch.full((bh, nc, ng, wl.head_dim), float("nan"), device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, full_c, full_g)
    # every sequence's tables as a decode loop holds them before its token: rows closed
    # by the token itself or later are unset (NaN)
    cs, gs = full_c.clone(), full_g.clone()
    for b in range(batch):
        p = int(pos[b])
        rows = slice(b * wl.heads_kv, (b + 1) * wl.heads_kv)
        cs[rows, (p + 1) // wl.chunk - (1 if (p + 1) % wl.chunk == 0 else 0):] = float("nan")
        gs_flat = gs[rows].reshape(wl.heads_kv, nc * ng, wl.head_dim)
        gs_flat[:, (p + 1) // wl.group - (1 if (p + 1) % wl.group == 0 else 0):] = float("nan")
        gs[rows] = gs_flat.reshape(wl.heads_kv, nc, ng, wl.head_dim)
    ci = torch.empty((bh, 1, wl.topk_chunks), dtype=torch.int32, device="cuda")
    gi = torch.empty((bh, 1, wl.topk_groups), dtype=torch.int32, device="cuda")
    out = torch.empty((wl.batch, wl.heads_q, 1, wl.head_dim), device="cuda")
    B.hga_decode_step(layer, q, pos_t, cs, gs, n, k, v, ci, gi, out, append=True)
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    for b in range(batch):
        p = int(pos[b])
        rows = slice(b * wl.heads_kv, (b + 1) * wl.heads_kv)
        c_done = (p + 1) // wl.chunk        # chunk rows complete through the token
        g_done = (p + 1) // wl.group
        got_c, want_c = cs[rows, :c_done], full_c[rows, :c_done]
        assert torch.equal(got_c.view(torch.int32), want_c.view(torch.int32)), b
        got_g = gs[rows].reshape(wl.heads_kv, nc * ng, -1)[:, :g_done]
        want_g = full_g[rows].reshape(wl.heads_kv, nc * ng, -1)[:, :g_done]
        assert torch.equal(got_g.view(torch.int32), want_g.view(torch.int32)), b
        assert torch.isnan(cs[rows, c_done:]).all() and \
            torch.isnan(gs[rows].reshape(wl.heads_kv, nc * ng, -1)[:, g_done:]).all()
    # the step's routing and output are those of the separate calls on the full tables
    sep, fus = run_both(wl, x)
    assert np.array_equal(ci.cpu().numpy().reshape(sep["chunk_idx"].shape), sep["chunk_idx"])
    assert np.array_equal(gi.cpu().numpy().reshape(sep["group_idx"].shape), sep["group_idx"])
    np.testing.assert_allclose(out.cpu().numpy(), sep["out"], atol=1e-2, rtol=0)


def test_decode_step_bounded_wait_times_out_and_recovers():
    """A wait that runs out ends the kernel with HGA_ERR_TIMEOUT instead of hanging.

    The debug hook makes one warp skip a group-summary copy it then waits for
    (nothing is in flight into that stage); the wait gives up after 2 ms, the
    item's partial is dropped and every barrier is still reached.  The next call
    without the hook is correct again.
    """
    wl = S.workload("llama3_8b_decode_32k", batch=10, context=2048, needles=0)
    x = S.make_inputs(wl, 36)
    layer = layer_of(wl)
    assert B.hga_decode_step_launches(layer, wl.context) == 1
    n = wl.context
    bh, nc, ng = wl.batch * wl.heads_kv, n // wl.chunk, wl.chunk // wl.group
    q, k, v = (to_device(x[t], wl.dtype) for t in ("q", "k", "v"))
    pos = torch.as_tensor(x["pos"], device="cuda")
    cs = torch.empty((bh, nc, wl.head_dim), device="cuda")
    gs = torch.empty((bh, nc, ng, wl.head_dim), device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, cs, gs)
    ci = torch.empty((bh, 1, wl.topk_chunks), dtype=torch.int32, device="cuda")
    gi = torch.empty((bh, 1, wl.topk_groups), dtype=torch.int32, device="cuda")
    out = torch.empty((wl.batch, wl.heads_q, 1, wl.head_dim), device="cuda")
    assert B.hga_device_status() == 0
    old = B.hga_debug_inject(1)
    try:
        B.hga_decode_step(layer, q, pos, cs, gs, n, k, v, ci, gi, out)
        torch.cuda.synchronize()
    finally:
        B.hga_debug_inject(old)
    assert B.hga_device_status() == 5  # HGA_ERR_TIMEOUT
    assert B.hga_device_status() == 0  # read and cleared
    sep, fus = run_both(wl, x)
    check_same_routing_close_output(sep, fus, 1e-2)
    compare_head(wl, x, fus, 0, 0)
