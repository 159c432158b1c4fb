"""Parity at the workloads' full sizes: the routed ids of EVERY (sequence, KV head)
unit (and every prefill block of two KV heads) against the oracle's routing,
recomputed in parallel over the host's cores; the attention output of sampled
units (16 per decode workload, 32 prefill blocks, one block's 64 rows in full)
against the oracle's attention; every unit is checked for size-independent
properties.  hga_route + hga_attend here; the one-launch decode step at full
size is in test_gpu_decode_step.py.
"""

import numpy as np
import pytest

import hga_synth as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU too
    pytest.skip("needs a CUDA device", allow_module_level=True)

from gpu_harness import (check_properties, compare_head, compare_prefill_blocks,  # noqa: E402
                         compare_prefill_routing_all, compare_routing_all, run_gpu, sample_units)
from hierarchical_sparse_attention_hga_b200 import binding as B  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    B.load_library()


def test_llama3_8b_decode_32k_batch16():
    wl = S.workload("llama3_8b_decode_32k")
    x = S.make_inputs(wl, S.seed_for(1))
    res = run_gpu(wl, x, fused=True)
    check_properties(wl, res)
    compare_routing_all(wl, S.seed_for(1), res)   # all 128 units
    for b, h in sample_units(wl, 16):
        compare_head(wl, x, res, b, h)
    for b in range(wl.batch):          # the planted needles are routed for every head
        for h in range(wl.heads_kv):
            assert set(S.needle_chunks(wl, S.seed_for(1), b, h)) <= set(res["chunk_idx"][b, h, 0])


def test_wide_head_decode_64k_batch32():
    wl = S.workload("wide_head_decode_64k")
    x = S.make_inputs(wl, S.seed_for(4))
    res = run_gpu(wl, x, fused=True)
    check_properties(wl, res)
    compare_routing_all(wl, S.seed_for(4), res)   # all 256 units
    for b, h in sample_units(wl, 16, seed=1):
        compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("kc,chunk", [(8, 64), (32, 64), (64, 64), (8, 128), (16, 128), (64, 128)])
def test_wide_head_sweep_full_context(kc, chunk):
    """The top-k / chunk-size sweep at the full 64K context (batch 4)."""
    wl = S.workload("wide_head_decode_64k", batch=4, topk_chunks=kc, topk_groups=2 * kc,
                    chunk=chunk)
    x = S.make_inputs(wl, S.seed_for(4) + kc + chunk)
    res = run_gpu(wl, x, fused=True)
    check_properties(wl, res)
    compare_routing_all(wl, S.seed_for(4) + kc + chunk, res)   # all 32 units
    for b, h in ((0, 1), (3, 6)):
        compare_head(wl, x, res, b, h)


def test_llama3_8b_prefill_64k_sampled_blocks():
    wl = S.workload("llama3_8b_prefill_64k")
    x = S.make_inputs(wl, S.seed_for(2))
    res = run_gpu(wl, x, fused=True, out_dtype=B.HGA_BF16)
    check_properties(wl, res)
    for h in (0, 6):                              # every one of the 1024 blocks
        compare_prefill_routing_all(wl, x, res, 0, h)
    rng = np.random.default_rng(2)
    blocks = sorted({0, 3, 5, 6, 21, 400, 1023} | set(int(j) for j in rng.permutation(1024)[:25]))
    for h in (0, 6):                              # 32 blocks, three rows each
        compare_prefill_blocks(wl, x, res, 0, h, blocks=blocks, rows=(0, 13, 63))
    # the causal edge: every row of one block's current-chunk tile
    compare_prefill_blocks(wl, x, res, 0, 3, blocks=(517,), rows=tuple(range(64)))
