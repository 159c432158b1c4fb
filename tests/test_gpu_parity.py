"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Routed indices must equal the oracle's except where the oracle's own scores put
the differing candidates within a 1e-4 relative window of the k-th score (a
near-tie, then the GPU selection is validated and attention is compared on
it).  Outputs: max-abs 2e-2 for bf16 K/V with fp32 accumulation, 1e-4 for
fp32 inputs.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import compare_head, compare_prefill_blocks, compare_summaries, run_gpu  # noqa: E402
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402
from oracle import hga_oracle as O  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


# ------------------------------------------------------------- tiny fp32 layer

def test_tiny_fp32_decode():
    wl = S.workload("tiny_f32_1k")
    x = S.make_inputs(wl, S.seed_for(0))
    res = run_gpu(wl, x)
    compare_summaries(wl, x, res, 0, 0)
    compare_head(wl, x, res, 0, 0)
    toks = O.visible_tokens(1023, 15, res["group_idx"][0, 0, 0], O.HGAParams(
        head_dim=64, heads_q=1, heads_kv=1, chunk=64, group=16, sink=1, local=2,
        topk_chunks=4, topk_groups=8))
    assert len(toks) == 384


def test_tiny_fp32_prefill_all_blocks():
    wl = S.workload("tiny_f32_1k", prefill=True)
    x = S.make_inputs(wl, S.seed_for(0))
    res = run_gpu(wl, x)
    assert res["chunk_idx"].shape[2] == 16
    compare_head(wl, x, res, 0, 0)


# ------------------------------------------------------- bf16 decode variants

@pytest.mark.parametrize("chunk", [64, 128])
def test_bf16_decode_small_context(chunk):
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=4096, chunk=chunk)
    x = S.make_inputs(wl, 11)
    res = run_gpu(wl, x)
    for b in range(2):
        for h in (0, 5):
            compare_summaries(wl, x, res, b, h)
            compare_head(wl, x, res, b, h)
    # planted needles are routed (sanity)
    for b in range(2):
        for h in range(wl.heads_kv):
            assert set(S.needle_chunks(wl, 11, b, h)) <= set(res["chunk_idx"][b, h, 0])


def test_decode_ragged_positions_and_empty_candidates():
    """Per-sequence positions: mid-chunk, mid-group, and too early for any candidate."""
    wl = S.workload("llama3_8b_decode_32k", batch=5, context=2048, heads_q=8, heads_kv=2,
                    needles=0)
    x = S.make_inputs(wl, 12)
    pos = np.array([2047, 2047 - 37, 700, 100, 5], dtype=np.int64)
    x["pos"] = pos
    res = run_gpu(wl, x)
    for b in range(5):
        for h in range(2):
            compare_head(wl, x, res, b, h)
    assert (res["chunk_idx"][3:] == -1).all()      # cur - local <= sink: no candidates
    assert (res["group_idx"][3:] == -1).all()


@pytest.mark.parametrize("kc,chunk", [(8, 64), (64, 64), (32, 128), (64, 128)])
def test_wide_head_sweep_small(kc, chunk):
    wl = S.workload("wide_head_decode_64k", batch=2, context=16384, topk_chunks=kc,
                    topk_groups=2 * kc, chunk=chunk)
    x = S.make_inputs(wl, 13)
    res = run_gpu(wl, x)
    for b in range(2):
        for h in (0, 7):
            compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("g_heads", [1, 16])
def test_gqa_extremes(g_heads):
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=2048, heads_q=2 * g_heads,
                    heads_kv=2, needles=0, topk_chunks=4, topk_groups=8)
    x = S.make_inputs(wl, 14)
    res = run_gpu(wl, x)
    for b in range(2):
        for h in range(2):
            compare_head(wl, x, res, b, h)


def test_bf16_output_dtype():
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=2048, needles=0)
    x = S.make_inputs(wl, 15)
    res = run_gpu(wl, x, out_dtype=B.HGA_BF16)
    compare_head(wl, x, res, 1, 3)


def test_bf16_prefill_small():
    wl = S.workload("llama3_8b_prefill_64k", context=1024, heads_q=8, heads_kv=2,
                    topk_chunks=4, topk_groups=8)
    x = S.make_inputs(wl, 16)
    res = run_gpu(wl, x)
    for h in range(2):
        compare_head(wl, x, res, 0, h)


# ----------------------------------------------------------- summaries / ABI

def test_incremental_summaries_equal_batch_bitwise():
    """Appending tokens one call at a time writes the same bits as one batch call."""
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=2048, heads_q=8, heads_kv=2,
                    needles=0)
    x = S.make_inputs(wl, 17)
    layer = __import__("gpu_harness").layer_of(wl)
    from gpu_harness import to_device
    k = to_device(x["k"], wl.dtype)
    n = wl.context
    shape_c = (2 * 2, n // 64, 128)
    shape_g = (2 * 2, n // 64, 4, 128)
    cs_a = torch.zeros(shape_c, device="cuda"); gs_a = torch.zeros(shape_g, device="cuda")
    cs_b = torch.zeros(shape_c, device="cuda"); gs_b = torch.zeros(shape_g, device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, cs_a, gs_a)
    start = n - 200
    B.hga_build_summaries(layer, k, n, 0, start, cs_b, gs_b)
    for t in range(start, n):
        B.hga_build_summaries(layer, k, n, t, t + 1, cs_b, gs_b)
    torch.cuda.synchronize()
    assert torch.equal(cs_a, cs_b) and torch.equal(gs_a, gs_b)


def test_invalid_position_sets_device_error_and_recovers():
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=1024, heads_q=8, heads_kv=2,
                    needles=0, topk_chunks=4, topk_groups=8)
    x = S.make_inputs(wl, 18)
    bad = np.array([1023, 1024], dtype=np.int64)   # second sequence past the cache
    res = run_gpu(wl, x, pos=bad, check_status=False)
    assert res["status"] == 6  # HGA_ERR_DEVICE_CHECK
    assert (res["chunk_idx"][1] == -1).all() and (res["group_idx"][1] == -1).all()
    assert np.all(res["out"][1] == 0)
    x["pos"] = np.array([1023, 1023], dtype=np.int64)
    res = run_gpu(wl, x)  # status is clear again
    compare_head(wl, x, res, 1, 1)


def test_host_side_argument_errors():
    layer = B.Layer(batch=1, heads_q=3, heads_kv=2, head_dim=128)
    with pytest.raises(B.HGAError) as e:
        B.hga_workspace_size(layer, 4096, 1)
    assert e.value.status == 2
    layer = B.Layer(batch=1, heads_q=4, heads_kv=2, head_dim=96)
    with pytest.raises(B.HGAError) as e:
        B.hga_workspace_size(layer, 4096, 1)
    assert e.value.status == 3


def test_bf16_head_dim_64_decode():
    """bf16 with D=64 takes the general kernel; parity holds there too."""
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=2048, head_dim=64, n_high_pairs=16,
                    heads_q=8, heads_kv=2, needles=0)
    x = S.make_inputs(wl, 19)
    res = run_gpu(wl, x)
    for b in range(2):
        for h in range(2):
            compare_summaries(wl, x, res, b, h)
            compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cache_past_the_query_is_never_read_into_the_output(dtype):
    """Rows after the query position may hold anything (here NaN): outputs stay exact."""
    wl = S.workload("llama3_8b_decode_32k", batch=2, context=2048, heads_q=8, heads_kv=2,
                    needles=0, dtype=dtype)
    x = S.make_inputs(wl, 20)
    pos = np.array([2047 - 5, 2047 - 16 - 9], dtype=np.int64)
    x["pos"] = pos
    nan = np.uint16(0x7FC0) if dtype == "bf16" else np.float32("nan")
    for b in range(2):
        x["k"][b, :, pos[b] + 1:] = nan
        x["v"][b, :, pos[b] + 1:] = nan
    res = run_gpu(wl, x, summaries_range=(0, int(pos.min()) + 1))
    assert np.isfinite(res["out"]).all()
    for b in range(2):
        for h in range(2):
            compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("context,batch", [(6400, 1), (100 * 64 * 5, 1), (3200, 3)])
def test_router_with_odd_chunk_counts(context, batch):
    """Chunk counts that split unevenly over a CTA cluster; small and large candidate sets."""
    wl = S.workload("llama3_8b_decode_32k", batch=batch, context=context, heads_q=8, heads_kv=2,
                    needles=0)
    x = S.make_inputs(wl, 21)
    res = run_gpu(wl, x)
    for b in range(batch):
        for h in range(2):
            compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("name,kw", [
    ("llama3_8b_decode_32k", dict(batch=3, context=8192)),
    ("wide_head_decode_64k", dict(batch=2, context=8192, chunk=128, topk_chunks=32, topk_groups=64)),
    ("llama3_8b_prefill_64k", dict(context=2048, heads_q=8, heads_kv=2)),
    ("tiny_f32_1k", dict()),
])
def test_fused_route_is_bitwise_the_two_calls(name, kw):
    from gpu_harness import layer_of, to_device
    wl = S.workload(name, **kw)
    x = S.make_inputs(wl, 22)
    layer = layer_of(wl)
    n = wl.context
    q_len = x["q"].shape[2]
    nblk = 1 if q_len == 1 else q_len // wl.chunk
    bh = wl.batch * wl.heads_kv
    q, k = to_device(x["q"], wl.dtype), to_device(x["k"], wl.dtype)
    pos = torch.as_tensor(x["pos"], device="cuda")
    cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device="cuda")
    gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device="cuda")
    B.hga_build_summaries(layer, k, n, 0, n, cs, gs)
    outs = []
    for fused in (False, True):
        ci = torch.full((bh, nblk, wl.topk_chunks), -7, dtype=torch.int32, device="cuda")
        gi = torch.full((bh, nblk, wl.topk_groups), -7, dtype=torch.int32, device="cuda")
        csc = torch.empty((bh, nblk, wl.topk_chunks), device="cuda")
        gsc = torch.empty((bh, nblk, wl.topk_groups), device="cuda")
        if fused:
            B.hga_route(layer, q, q_len, pos, cs, gs, n, ci, gi, csc, gsc)
        else:
            B.hga_route_chunks(layer, q, q_len, pos, cs, n, ci, csc)
            B.hga_route_groups(layer, q, q_len, pos, gs, n, ci, gi, gsc)
        torch.cuda.synchronize()
        outs.append((ci.cpu(), gi.cpu(), csc.cpu(), gsc.cpu()))
    assert B.hga_device_status() == 0
    for a, b in zip(*outs):
        assert torch.equal(a.nan_to_num(nan=-9.0), b.nan_to_num(nan=-9.0))


# --------------------------------------------------------------- prefill (tcgen05)

@pytest.mark.parametrize("heads_q,heads_kv,out_dtype", [(8, 2, B.HGA_F32), (4, 2, B.HGA_F32),
                                                       (8, 2, B.HGA_BF16)])
def test_prefill_tensor_core_path_small(heads_q, heads_kv, out_dtype):
    """64-query blocks on tcgen05 (G*C = 256 or 128 rows), every block and row checked."""
    wl = S.workload("llama3_8b_prefill_64k", context=1024, heads_q=heads_q, heads_kv=heads_kv,
                    topk_chunks=4, topk_groups=8)
    x = S.make_inputs(wl, 23)
    res = run_gpu(wl, x, out_dtype=out_dtype)
    for h in range(heads_kv):
        compare_head(wl, x, res, 0, h)


def test_prefill_suffix_with_ragged_block_count_and_positions():
    """A 13-block prompt continuing a cache (queries start mid-cache), two sequences
    at different positions: the router's blocks-per-CTA grouping has a ragged tail."""
    wl = S.workload("llama3_8b_prefill_64k", batch=2, context=4096, heads_q=8, heads_kv=2,
                    topk_chunks=8, topk_groups=16)
    q_len = 13 * wl.chunk
    x = S.make_inputs(wl, 25, q_len=q_len)
    x["pos"] = np.array([4095, 1535], dtype=np.int64)
    res = run_gpu(wl, x, q_len=q_len)
    for b in range(2):
        for h in range(2):
            compare_prefill_blocks(wl, x, res, b, h, blocks=range(13), rows=(0, 17, 63))


def test_prefill_tensor_core_path_8k_sampled_blocks():
    """Llama-3-8B-shaped prefill at 8K context: many KV tiles per block, all workload k values."""
    wl = S.workload("llama3_8b_prefill_64k", context=8192)
    x = S.make_inputs(wl, 24)
    res = run_gpu(wl, x)
    assert np.isfinite(res["out"]).all()
    for h in (0, 3, 7):
        compare_prefill_blocks(wl, x, res, 0, h, blocks=(0, 1, 4, 5, 6, 37, 127),
                               rows=(0, 9, 40, 63))
