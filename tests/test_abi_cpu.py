"""The C-ABI library builds, loads and exports every symbol include/hga.h declares.

No compute call is made here: only entry points that fail host-side argument
validation (before any CUDA call) or are pure host functions run.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from hierarchical_sparse_attention_hga_b200 import binding as B
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    return B.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hga.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_[a-z_]+)\s*\(", text)))


def test_header_declares_the_four_steps():
    names = declared_symbols()
    for step in ("hga_build_summaries", "hga_route_chunks", "hga_route_groups", "hga_attend"):
        assert step in names


def test_library_exports_every_declared_symbol(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    names = declared_symbols()
    assert sorted(B.SYMBOLS) == names
    for name in names:
        assert getattr(lib, name) is not None


def test_abi_version_and_status_strings(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    assert B.hga_abi_version() == 6
    assert B.hga_status_string(0) == "HGA_OK"
    assert B.hga_status_string(6) == "HGA_ERR_DEVICE_CHECK"
    assert B.hga_status_string(99) == "HGA_ERR_UNKNOWN"


def test_config_struct_layout_matches_header(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    assert ctypes.sizeof(B.HGAConfig) == 14 * 4 + 8
    assert B.HGAConfig.rope_theta.offset == 56


@pytest.mark.parametrize("kw,status", [
    (dict(heads_q=3, heads_kv=2), 2),          # Hq % Hkv
    (dict(head_dim=96), 3),                     # unsupported D
    (dict(chunk=32), 3),                        # unsupported C
    (dict(group=8), 3),                         # unsupported g
    (dict(topk_chunks=0), 1),                   # non-positive k
    (dict(n_high_pairs=65), 2),                 # more pairs than D/2
    (dict(rope_theta=0.5), 1),
    (dict(heads_q=64, heads_kv=2), 3),          # G = 32 > 16
    (dict(dtype=7), 1),
])
def test_host_validation_errors(lib, kw, status):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    base = dict(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    base.update(kw)
    with pytest.raises(B.HGAError) as e:
        B.hga_workspace_size(B.Layer(**base), 4096, 1)
    assert e.value.status == status
    assert B.load_library().hga_last_error()  # detail message is set


def test_shape_errors_of_sizes(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    for n_alloc, q_len, status in [(4000, 1, 2), (4096, 0, 1), (4096, 100, 3), (0, 1, 2)]:
        with pytest.raises(B.HGAError) as e:
            B.hga_workspace_size(layer, n_alloc, q_len)
        assert e.value.status == status


def test_null_pointers_rejected_before_any_cuda_call(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    with pytest.raises(B.HGAError) as e:
        B.hga_build_summaries(layer, None, 4096, 0, 4096, None, None, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_build_summaries(layer, 16, 4096, 10, 5, 16, 16, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_route_chunks(layer, None, 1, None, None, 4096, None, stream=0)
    assert e.value.status == 1
    f32 = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128, dtype=B.HGA_F32)
    with pytest.raises(B.HGAError) as e:
        B.hga_attend(f32, 16, 1, 16, 16, 16, 4096, 16, 16, workspace=None, workspace_bytes=0,
                     stream=0)
    assert e.value.status == 7  # fp32 decode needs split-K workspace


def test_workspace_size_is_zero_for_prefill_and_grows_with_batch(lib):
    from hierarchical_sparse_attention_hga_b200 import binding as B
    f32 = dict(heads_q=32, heads_kv=8, head_dim=128, dtype=B.HGA_F32)
    small = B.hga_workspace_size(B.Layer(batch=1, **f32), 32768, 1)
    big = B.hga_workspace_size(B.Layer(batch=16, **f32), 32768, 1)
    assert 0 < small < big
    assert B.hga_workspace_size(B.Layer(batch=1, **f32), 32768, 1024) == 0
    # bf16, D = 128 decode merges its split-K partials inside a CTA cluster
    assert B.hga_workspace_size(B.Layer(batch=16, heads_q=32, heads_kv=8, head_dim=128), 32768,
                                1) == 0


def test_decode_step_rejects_what_it_does_not_fuse(lib):
    """hga_decode_step: null pointers, fp32 K/V, D = 64 and host-tier K/V are refused on the
    host (no CUDA call is made)."""
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    with pytest.raises(B.HGAError) as e:
        B.hga_decode_step(layer, None, 16, 16, 16, 4096, 16, 16, 16, 16, 16, stream=0)
    assert e.value.status == 1
    for kw in (dict(dtype=B.HGA_F32), dict(head_dim=64, n_high_pairs=16)):
        other = B.Layer(batch=1, heads_q=32, heads_kv=8, **{"head_dim": 128, **kw})
        with pytest.raises(B.HGAError) as e:
            B.hga_decode_step(other, 16, 16, 16, 16, 4096, 16, 16, 16, 16, 16, stream=0)
        assert e.value.status == 3
    host = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    host.kv_loc = B.HGA_KV_HOST_PINNED
    with pytest.raises(B.HGAError) as e:
        B.hga_decode_step(host, 16, 16, 16, 16, 4096, 16, 16, 16, 16, 16, stream=0)
    assert e.value.status == 3


def test_warm_tier_sizes_and_refusals(lib):
    """hga_warm_rows: the window rows plus warm_groups groups; warm_groups below
    topk_groups or above 2048, and null tables, are refused on the host."""
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=2, heads_q=32, heads_kv=8, head_dim=128)
    window = (layer.sink_chunks + layer.local_chunks + 1) * layer.chunk
    assert B.hga_hot_rows(layer) == window + layer.topk_groups * layer.group
    for m in (layer.topk_groups, 100, 2048):
        assert B.hga_warm_rows(layer, m) == window + m * layer.group
    for m in (layer.topk_groups - 1, 2049, -1):
        with pytest.raises(B.HGAError) as e:
            B.hga_warm_rows(layer, m)
        assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_warm_reset(layer, 64, None, 16, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_warm_reset(layer, 64, 16, 16, seq=2, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_gather_warm(layer, 16, 16, 4096, 16, 16, 64, 16, 16, None, 16, 16, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_attend_warm(layer, 16, 16, 16, 16, 4096, 16, 16, 16, 16, stream=0)
    assert e.value.status == 1   # warm_groups 16 < topk_groups
    for fn in (lambda: B.hga_gather_host(layer, 16, 16, 4096, 16, 16, 16, 16, refresh_window=3,
                                         stream=0),
               lambda: B.hga_gather_warm(layer, 16, 16, 4096, 16, 16, 64, 16, 16, 16, 16, 16,
                                         refresh_window=-1, stream=0)):
        with pytest.raises(B.HGAError) as e:
            fn()
        assert e.value.status == 1   # window modes are 0, 1 and 2


def test_paged_pool_refusals(lib):
    """Paged calls check the block-table description on the host: a page size that
    is not a positive multiple of 16, a null table, non-positive sizes, a capacity
    that is not whole chunks, a pool of 2^31 rows or more."""
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=2, heads_q=32, heads_kv=8, head_dim=128)
    cases = [(B.kv_pages(16, 100, 8, 64), 1), (B.kv_pages(None, 100, 64, 64), 1),
             (B.kv_pages(16, 0, 64, 64), 1), (B.kv_pages(16, 100, 64, 0), 1),
             (B.kv_pages(16, 100, 48, 5), 2), (B.kv_pages(16, 1 << 24, 256, 64), 3)]
    for kv, status in cases:
        with pytest.raises(B.HGAError) as e:
            B.hga_decode_step_paged(layer, 16, 16, 16, 16, 16, 16, kv, 16, 16, 16, stream=0)
        assert e.value.status == status, (kv.page_size, kv.n_pages, kv.max_pages)
        with pytest.raises(B.HGAError) as e:
            B.hga_build_summaries_paged(layer, 16, kv, 16, 16, 16, stream=0)
        assert e.value.status == status
    with pytest.raises(B.HGAError) as e:   # null pointers after a valid description
        B.hga_decode_step_paged(layer, None, 16, 16, 16, 16, 16, B.kv_pages(16, 100, 64, 64), 16,
                                16, 16, stream=0)
    assert e.value.status == 1


def test_backward_workspace_and_refusals(lib):
    """The backward pass sizes its workspace on the host and refuses decode shapes,
    fp32 K/V, null pointers and a short workspace before any CUDA call."""
    from hierarchical_sparse_attention_hga_b200 import binding as B
    layer = B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128)
    small = B.hga_attend_backward_workspace_size(layer, 8192, 8192)
    big = B.hga_attend_backward_workspace_size(layer, 65536, 65536)
    assert 0 < small < big
    for args, status in (((layer, 8192, 1), 3),
                         ((B.Layer(batch=1, heads_q=32, heads_kv=8, head_dim=128, dtype=B.HGA_F32),
                           8192, 8192), 3)):
        with pytest.raises(B.HGAError) as e:
            B.hga_attend_backward_workspace_size(*args)
        assert e.value.status == status
    with pytest.raises(B.HGAError) as e:
        B.hga_attend_backward(layer, None, 8192, 16, 16, 16, 8192, 16, 16, 16, 16, 16, 16, 16, 16,
                              small, stream=0)
    assert e.value.status == 1
    with pytest.raises(B.HGAError) as e:
        B.hga_attend_backward(layer, 16, 8192, 16, 16, 16, 8192, 16, 16, 16, 16, 16, 16, 16, 16,
                              small - 1, stream=0)
    assert e.value.status == 7
