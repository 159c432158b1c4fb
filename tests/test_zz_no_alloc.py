"""hga_attend_noalloc against hga_attend, through the C ABI.

hga_attend_noalloc serves callers that cannot allocate device memory (a
framework that owns every device buffer and passes a plugin only its inputs
and outputs, or a loop where cudaMalloc/cudaFree may not run): it keeps the
split-K scratch in a fixed array inside the library.  Its output must match
hga_attend with a caller workspace bit for bit (both run the same kernels on
the same inputs; only the scratch address differs), call after call - also
after a larger call has left more of the array written - and shapes that need
more scratch than the array holds must be refused.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import layer_of, to_device  # noqa: E402
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def _routed(wl, x):
    """Device tensors and routed group ids for one decode step."""
    layer = layer_of(wl)
    n = wl.context
    bh = wl.batch * wl.heads_kv
    q, k, v = (to_device(x[t], wl.dtype) for t in ("q", "k", "v"))
    pos = torch.as_tensor(x["pos"], device="cuda")
    cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device="cuda")
    gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device="cuda")
    ci = torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device="cuda")
    gi = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, cs, gs)
    B.hga_route_chunks(layer, q, 1, pos, cs, n, ci)
    B.hga_route_groups(layer, q, 1, pos, gs, n, ci, gi)
    return layer, q, k, v, pos, gi


def _attend_both(wl, layer, q, k, v, pos, gi):
    """hga_attend with a fresh caller workspace full of NaN bytes, then hga_attend_noalloc."""
    n = wl.context
    shape = (wl.batch, wl.heads_q, 1, wl.head_dim)
    ref, ref_lse = torch.empty(shape, device="cuda"), torch.empty(shape[:3], device="cuda")
    got, got_lse = torch.full(shape, 7.0, device="cuda"), torch.empty(shape[:3], device="cuda")
    wsb = B.hga_workspace_size(layer, n, 1)
    assert wsb > 0  # this shape does use split-K scratch
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")  # reads of unwritten scratch show
    B.hga_attend(layer, q, 1, pos, k, v, n, gi, ref, ref_lse, ws, wsb)
    B.hga_attend_noalloc(layer, q, 1, pos, k, v, n, gi, got, got_lse)
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    return ref.cpu().numpy(), got.cpu().numpy(), ref_lse.cpu().numpy(), got_lse.cpu().numpy()


def _assert_bitwise(ref, got, ref_lse, got_lse):
    assert np.isfinite(got).all() and np.isfinite(got_lse).all()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(got_lse.view(np.uint32), ref_lse.view(np.uint32))


@pytest.mark.parametrize("name,kw", [
    ("llama3_8b_decode_32k", dict(batch=4, context=4096, head_dim=64, n_high_pairs=16)),  # bf16
    ("tiny_f32_1k", dict(batch=3, heads_q=4, heads_kv=2)),                                  # fp32
])
def test_noalloc_matches_workspace_call_twice_in_a_row(name, kw):
    wl = S.workload(name, **kw)
    for call, seed in enumerate((31, 32)):    # two calls in a row, different inputs
        x = S.make_inputs(wl, seed)
        if call == 1:
            x["pos"] = x["pos"] - np.arange(wl.batch) * 7   # ragged positions on the 2nd call
        _assert_bitwise(*_attend_both(wl, *_routed(wl, x)))


def test_noalloc_after_a_call_that_wrote_more_scratch():
    """A small call after a larger one reads none of what the larger call left behind."""
    big = S.workload("llama3_8b_decode_32k", batch=8, context=8192, head_dim=64, n_high_pairs=16)
    small = S.workload("llama3_8b_decode_32k", batch=1, context=2048, head_dim=64, n_high_pairs=16)
    lb, ls = layer_of(big), layer_of(small)
    assert B.hga_workspace_size(lb, big.context, 1) > B.hga_workspace_size(ls, small.context, 1)
    for wl, seed in ((big, 41), (small, 42), (big, 43), (small, 44)):
        _assert_bitwise(*_attend_both(wl, *_routed(wl, S.make_inputs(wl, seed))))


def test_noalloc_refuses_shapes_beyond_its_scratch():
    wl = S.workload("wide_head_decode_64k", batch=256, dtype="f32")  # general split-K kernel
    layer = layer_of(wl)
    assert B.hga_workspace_size(layer, wl.context, 1) > 8 << 20
    with pytest.raises(B.HGAError) as e:
        B.hga_attend_noalloc(layer, 16, 1, 16, 16, 16, wl.context, 16, 16)
    assert e.value.status == 7  # HGA_ERR_WORKSPACE, before touching the (fake) pointers
    assert "8388608" in str(e.value)
