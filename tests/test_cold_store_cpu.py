"""Cold tier host side: the file-backed K/V history and the staging of a warm
step's misses and window rows (runs without a GPU: positioned reads and writes
on the host's file system).  The expected rows are sliced here from the arrays
that were written, following the staging layout documented in include/hga.h.
"""

import numpy as np
import pytest

from hierarchical_sparse_attention_hga_b200 import binding as B


@pytest.fixture(scope="module")
def lib():
    from hierarchical_sparse_attention_hga_b200.build import build
    build()
    return B.load_library()


def _layer(batch=2, hkv=3):
    return B.Layer(batch=batch, heads_q=2 * hkv, heads_kv=hkv, head_dim=128)


def _history(layer, n, seed):
    rng = np.random.default_rng(seed)
    shape = (layer.batch, layer.heads_kv, n, 128)
    return (rng.integers(0, 1 << 16, shape, dtype=np.uint16),
            rng.integers(0, 1 << 16, shape, dtype=np.uint16))


def _window_tokens(layer, pos, mode):
    """Window rows of a query at pos, in staging order (sink, local, current)."""
    c = layer.chunk
    cur = pos // c
    b0 = max(0, cur - layer.local_chunks)
    toks = []
    if mode == 1:
        for ch in range(min(layer.sink_chunks, b0)):
            toks += range(ch * c, (ch + 1) * c)
        toks += range(b0 * c, cur * c)
    toks += range(pos if mode == 2 else cur * c, pos + 1)
    return toks


def _expected(layer, k, v, pos, plan, n_plan, mode):
    kg = layer.topk_groups
    wr = (layer.sink_chunks + layer.local_chunks + 1) * layer.chunk
    units = layer.batch * layer.heads_kv
    out = np.zeros((units, 2 * kg * 16 + 2 * wr, 128), dtype=np.uint16)
    kk = k.reshape(units, -1, 128)
    vv = v.reshape(units, -1, 128)
    for u in range(units):
        for r in range(n_plan[u]):
            gid = plan[u, r, 0]
            out[u, r * 16:(r + 1) * 16] = kk[u, gid * 16:(gid + 1) * 16]
            out[u, (kg + r) * 16:(kg + r + 1) * 16] = vv[u, gid * 16:(gid + 1) * 16]
        toks = _window_tokens(layer, int(pos[u // layer.heads_kv]), mode)
        base = 2 * kg * 16
        out[u, base:base + len(toks)] = kk[u, toks]
        out[u, base + wr:base + wr + len(toks)] = vv[u, toks]
    return out


def _staging(layer):
    nb = B.hga_cold_stage_bytes(layer)
    units = layer.batch * layer.heads_kv
    assert nb % (units * 256) == 0
    return np.zeros((units, nb // units // 256, 128), dtype=np.uint16)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("threads", [1, 6])
def test_stage_reads_the_missed_groups_and_window_rows(lib, tmp_path, mode, threads):
    layer = _layer()
    n = 2048
    k, v = _history(layer, n, seed=mode)
    rng = np.random.default_rng(10 + mode)
    units = layer.batch * layer.heads_kv
    plan = np.full((units, layer.topk_groups, 2), -1, dtype=np.int32)
    n_plan = rng.integers(0, layer.topk_groups + 1, units).astype(np.int32)
    for u in range(units):
        gids = rng.choice(n // 16, n_plan[u], replace=False)
        plan[u, :n_plan[u], 0] = gids
        plan[u, :n_plan[u], 1] = np.arange(n_plan[u])
    pos = np.array([2047, 1000], dtype=np.int64)
    with B.ColdStore(tmp_path / "kv.bin", layer, n, create=True) as st:
        st.write(k, v, 0, n, threads=threads)
        got = _staging(layer)
        st.stage(layer, pos, plan, n_plan, mode, got, threads=threads)
    want = _expected(layer, k, v, pos, plan, n_plan, mode)
    # only the rows the layout assigns are defined: compare those
    kg, wr = layer.topk_groups, (layer.sink_chunks + layer.local_chunks + 1) * layer.chunk
    for u in range(units):
        m = n_plan[u]
        nw = len(_window_tokens(layer, int(pos[u // layer.heads_kv]), mode))
        for lo, hi in ((0, m * 16), (kg * 16, (kg + m) * 16), (2 * kg * 16, 2 * kg * 16 + nw),
                       (2 * kg * 16 + wr, 2 * kg * 16 + wr + nw)):
            assert np.array_equal(got[u, lo:hi], want[u, lo:hi]), (u, lo, hi)


def test_writes_in_pieces_equal_one_write_and_reopen(lib, tmp_path):
    layer = _layer(batch=1, hkv=2)
    n = 1024
    k, v = _history(layer, n, seed=7)
    path = tmp_path / "kv.bin"
    with B.ColdStore(path, layer, n, create=True) as st:
        for t0, t1 in ((0, 300), (300, 301), (301, 1024)):
            st.write(k, v, t0, t1, threads=3)
    raw = np.fromfile(path, dtype=np.uint16).reshape(2, 1, 2, n, 128)
    assert np.array_equal(raw[0], k) and np.array_equal(raw[1], v)
    with B.ColdStore(path, layer, n) as st:   # reopened without create
        plan = np.zeros((2, layer.topk_groups, 2), dtype=np.int32)
        plan[:, 0, 0] = [5, 60]
        n_plan = np.array([1, 1], dtype=np.int32)
        got = _staging(layer)
        st.stage(layer, np.array([1023]), plan, n_plan, 2, got)
    assert np.array_equal(got[1, 0:16], k[0, 1, 60 * 16:61 * 16])


def test_errors_are_status_codes(lib, tmp_path):
    layer = _layer(batch=1, hkv=2)
    n = 1024
    short = tmp_path / "short.bin"
    short.write_bytes(b"\0" * 1000)
    with pytest.raises(B.HGAError) as e:
        B.ColdStore(short, layer, n)
    assert e.value.status == 1 and "holds 1000 bytes" in str(e.value)
    k, v = _history(layer, n, seed=1)
    with B.ColdStore(tmp_path / "kv.bin", layer, n, create=True) as st:
        st.write(k, v, 0, n)
        got = _staging(layer)
        plan = np.zeros((2, layer.topk_groups, 2), dtype=np.int32)
        plan[0, 0, 0] = n // 16           # one past the last group
        with pytest.raises(B.HGAError) as e:
            st.stage(layer, np.array([1023]), plan, np.array([1, 0], dtype=np.int32), 0, got)
        assert e.value.status == 1
        with pytest.raises(B.HGAError) as e:
            st.stage(layer, np.array([1023]), plan, np.array([0, 0], dtype=np.int32), 3, got)
        assert e.value.status == 1
        with pytest.raises(B.HGAError) as e:
            st.stage(_layer(batch=2, hkv=2), np.array([1023, 1023]), plan,
                     np.array([0, 0], dtype=np.int32), 0, got)
        assert e.value.status == 2
        with pytest.raises(B.HGAError) as e:
            st.write(k, v, 10, n + 1)
        assert e.value.status == 1
