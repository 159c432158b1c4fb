"""hga_decode_step against hga_route + hga_attend and the oracle.

Batches with about one (sequence, KV head) item per SM run the one-launch kernel
(one CTA per item); smaller and larger batches run the routing and attention
kernels through the same call.  The one-launch kernel scores with the routing
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

from gpu_harness import compare_head, layer_of, to_device  # noqa: E402
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
    for b, h in ((0, 0), (7, 3), (15, 7)):
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
    """Batches with about one (sequence, KV head) item per SM take the one-CTA-per-item
    variant; ragged positions, down to a sequence with no candidate chunk."""
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
