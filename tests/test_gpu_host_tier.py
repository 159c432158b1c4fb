"""Host tier: K/V in pinned host memory, routed groups gathered per step.

The working-buffer path must give the oracle's result, and the same bits as
the device-resident path on the same inputs, step after step (the window ring
crosses chunk boundaries).
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


class Runner:
    """Device buffers of one layer, run either device-resident or host-tier."""

    def __init__(self, wl, x):
        self.wl = wl
        n, bh = wl.context, wl.batch * wl.heads_kv
        self.dev_layer = layer_of(wl)
        self.host_layer = layer_of(wl)
        self.host_layer.kv_loc = B.HGA_KV_HOST_PINNED
        self.q = to_device(x["q"], wl.dtype)
        self.k = to_device(x["k"], wl.dtype)
        self.v = to_device(x["v"], wl.dtype)
        self.k_host = self.k.cpu().pin_memory()
        self.v_host = self.v.cpu().pin_memory()
        rows = B.hga_hot_rows(self.host_layer)
        assert rows == (wl.sink + wl.local + 1) * wl.chunk + wl.topk_groups * wl.group
        self.k_work = torch.full((bh, rows, wl.head_dim), float("nan"), dtype=torch.bfloat16,
                                 device="cuda")
        self.v_work = torch.full_like(self.k_work, float("nan"))
        self.cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device="cuda")
        self.gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device="cuda")
        self.ci = torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device="cuda")
        self.gi = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device="cuda")
        self.n = n

    def summaries(self, t0, t1, host):
        src = self.k_host if host else self.k
        lay = self.host_layer if host else self.dev_layer
        B.hga_build_summaries(lay, src, self.n, t0, t1, self.cs, self.gs)

    def step(self, pos, host, refresh=False):
        wl = self.wl
        pos_t = torch.as_tensor(pos, dtype=torch.int64, device="cuda")
        out = torch.empty(wl.batch, wl.heads_q, 1, wl.head_dim, device="cuda")
        lse = torch.empty(wl.batch, wl.heads_q, 1, device="cuda")
        lay = self.host_layer if host else self.dev_layer
        B.hga_route(lay, self.q, 1, pos_t, self.cs, self.gs, self.n, self.ci, self.gi)
        if host:
            B.hga_gather_host(lay, self.k_host, self.v_host, self.n, pos_t, self.gi, self.k_work,
                              self.v_work, refresh_window=refresh)
            B.hga_attend(lay, self.q, 1, pos_t, self.k_work, self.v_work, self.n, self.gi, out, lse)
        else:
            B.hga_attend(lay, self.q, 1, pos_t, self.k, self.v, self.n, self.gi, out, lse)
        torch.cuda.synchronize()
        assert B.hga_device_status() == 0
        return out.cpu().numpy(), lse.cpu().numpy(), self.gi.cpu().numpy().copy()


def test_host_tier_decode_matches_oracle():
    wl = S.workload("host_tier_decode_128k", batch=2, context=8192)
    x = S.make_inputs(wl, 41)
    r = Runner(wl, x)
    r.summaries(0, wl.context, host=True)  # summaries read the host cache directly
    out, lse, gi = r.step(x["pos"], host=True, refresh=True)
    res = dict(chunk_idx=r.ci.cpu().numpy().reshape(2, 8, 1, -1), group_idx=gi.reshape(2, 8, 1, -1),
               out=out, lse=lse)
    for b in range(2):
        for h in (0, 3, 7):
            compare_head(wl, x, res, b, h)


@pytest.mark.parametrize("mode", [0, 2])
def test_host_tier_equals_device_path_step_by_step(mode):
    """Decode steps across chunk boundaries: the window ring and the staged groups
    give the same bits as the device-resident cache (window mode 0: the current
    chunk re-copied each step; 2: only the newest row)."""
    wl = S.workload("host_tier_decode_128k", batch=2, context=4096, heads_q=8, heads_kv=2)
    x = S.make_inputs(wl, 42)
    r = Runner(wl, x)
    start = 4020   # one decode step per position, across the chunk boundaries at 4032 and 4064
    r.summaries(0, start, host=False)
    for step, p in enumerate(range(start, 4096)):
        pos = np.array([p, p - 3], dtype=np.int64)
        r.summaries(p, p + 1, host=False)
        dev_out, dev_lse, dev_gi = r.step(pos, host=False)
        host_out, host_lse, host_gi = r.step(pos, host=True, refresh=1 if step == 0 else mode)
        assert np.array_equal(dev_gi, host_gi)
        assert np.array_equal(dev_out, host_out), f"step at {p}"
        assert np.array_equal(dev_lse, host_lse)


def test_host_tier_rejects_unsupported_shapes():
    wl = S.workload("tiny_f32_1k")
    lay = layer_of(wl)
    lay.kv_loc = B.HGA_KV_HOST_PINNED
    with pytest.raises(B.HGAError) as e:
        B.hga_gather_host(lay, 16, 16, 1024, 16, 16, 16, 16)
    assert e.value.status == 3


def test_host_tier_decode_128k_batch8_full_size():
    """The host-tier workload at full size: 131072 tokens, batch 8, K/V pinned on the host."""
    wl = S.workload("host_tier_decode_128k")
    x = S.make_inputs(wl, S.seed_for(3))
    r = Runner(wl, x)
    r.summaries(0, wl.context, host=True)
    out, lse, gi = r.step(x["pos"], host=True, refresh=True)
    res = dict(chunk_idx=r.ci.cpu().numpy().reshape(8, 8, 1, -1), group_idx=gi.reshape(8, 8, 1, -1),
               out=out, lse=lse)
    assert np.isfinite(out).all()
    compare_routing_all(wl, S.seed_for(3), res)   # all 64 units
    for b, h in sample_units(wl, 16):
        compare_head(wl, x, res, b, h)
