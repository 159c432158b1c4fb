"""Thin Python binding of libhga.so (the C ABI in include/hga.h).

Argument marshalling only: every step of the HGA path runs in the library's
CUDA kernels.  Tensors are passed as raw pointers; the caller allocates them
(PyTorch is used for device memory and streams).  If the library is missing,
every call raises - there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhga.so")

HGA_F32, HGA_BF16 = 0, 1
HGA_KV_DEVICE, HGA_KV_HOST_PINNED = 0, 1

STATUS_NAMES = {0: "HGA_OK", 1: "HGA_ERR_INVALID_ARG", 2: "HGA_ERR_SHAPE", 3: "HGA_ERR_UNSUPPORTED",
                4: "HGA_ERR_CUDA", 5: "HGA_ERR_TIMEOUT", 6: "HGA_ERR_DEVICE_CHECK",
                7: "HGA_ERR_WORKSPACE"}

# Exported symbols of the C ABI, in header order.
SYMBOLS = ("hga_abi_version", "hga_status_string", "hga_last_error", "hga_device_status",
           "hga_debug_inject",
           "hga_workspace_size", "hga_build_summaries", "hga_route_chunks", "hga_route_groups",
           "hga_route", "hga_hot_rows", "hga_gather_host", "hga_attend", "hga_decode_step",
           "hga_decode_step_launches", "hga_attend_noalloc", "hga_warm_rows", "hga_warm_reset",
           "hga_gather_warm", "hga_attend_warm", "hga_build_summaries_paged",
           "hga_decode_step_paged", "hga_attend_backward_workspace_size", "hga_attend_backward",
           "hga_cold_open", "hga_cold_close", "hga_cold_write", "hga_cold_stage_bytes",
           "hga_warm_plan", "hga_cold_stage", "hga_warm_fill")


class HGAConfig(ctypes.Structure):
    """Mirror of struct hga_config."""

    _fields_ = [("batch", ctypes.c_int32), ("heads_q", ctypes.c_int32),
                ("heads_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("group", ctypes.c_int32),
                ("sink_chunks", ctypes.c_int32), ("local_chunks", ctypes.c_int32),
                ("topk_chunks", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("n_high_pairs", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("kv_loc", ctypes.c_int32),
                ("rope_theta", ctypes.c_double)]


class HGAKvPages(ctypes.Structure):
    """Mirror of struct hga_kv_pages (a paged K/V pool's block table)."""

    _fields_ = [("block_table", ctypes.c_void_p), ("n_pages", ctypes.c_int64),
                ("page_size", ctypes.c_int32), ("max_pages", ctypes.c_int32)]


class HGAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {detail}")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhga.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libhga.so not found at {path}; build it with "
                           "`python -m hierarchical_sparse_attention_hga_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    C = ctypes.POINTER(HGAConfig)
    KV = ctypes.POINTER(HGAKvPages)
    sig = {
        "hga_abi_version": (I32, []),
        "hga_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hga_last_error": (ctypes.c_char_p, []),
        "hga_device_status": (ctypes.c_int, [P]),
        "hga_workspace_size": (ctypes.c_int, [C, I64, I32, ctypes.POINTER(SZ)]),
        "hga_build_summaries": (ctypes.c_int, [C, P, I64, I64, I64, P, P, P]),
        "hga_route_chunks": (ctypes.c_int, [C, P, I32, P, P, I64, P, P, P]),
        "hga_route_groups": (ctypes.c_int, [C, P, I32, P, P, I64, P, P, P, P]),
        "hga_route": (ctypes.c_int, [C, P, I32, P, P, P, I64, P, P, P, P, P]),
        "hga_hot_rows": (ctypes.c_int, [C, ctypes.POINTER(I64)]),
        "hga_gather_host": (ctypes.c_int, [C, P, P, I64, P, P, P, P, I32, P]),
        "hga_attend": (ctypes.c_int, [C, P, I32, P, P, P, I64, P, P, P, P, SZ, P]),
        "hga_decode_step": (ctypes.c_int, [C, P, P, P, P, I64, P, P, P, P, P, P, P, P, I32, P]),
        "hga_debug_inject": (I32, [I32]),
        "hga_decode_step_launches": (ctypes.c_int, [C, I64, ctypes.POINTER(I32)]),
        "hga_attend_noalloc": (ctypes.c_int, [C, P, I32, P, P, P, I64, P, P, P, P]),
        "hga_warm_rows": (ctypes.c_int, [C, I32, ctypes.POINTER(I64)]),
        "hga_warm_reset": (ctypes.c_int, [C, I32, P, P, I32, P]),
        "hga_gather_warm": (ctypes.c_int, [C, P, P, I64, P, P, I32, P, P, P, P, P, I32, P, P]),
        "hga_attend_warm": (ctypes.c_int, [C, P, P, P, P, I64, P, P, I32, P, P, P]),
        "hga_build_summaries_paged": (ctypes.c_int, [C, P, KV, P, P, P, P]),
        "hga_decode_step_paged": (ctypes.c_int, [C, P, P, P, P, P, P, KV, P, P, P, P, P, P, I32,
                                                 P]),
        "hga_attend_backward_workspace_size": (ctypes.c_int, [C, I64, I32, ctypes.POINTER(SZ)]),
        "hga_attend_backward": (ctypes.c_int, [C, P, I32, P, P, P, I64, P, P, P, P, P, P, P, P,
                                               SZ, P]),
        "hga_cold_open": (ctypes.c_int, [ctypes.c_char_p, C, I64, I32, ctypes.POINTER(P)]),
        "hga_cold_close": (ctypes.c_int, [P]),
        "hga_cold_write": (ctypes.c_int, [P, P, P, I64, I64, I32]),
        "hga_cold_stage_bytes": (ctypes.c_int, [C, ctypes.POINTER(SZ)]),
        "hga_warm_plan": (ctypes.c_int, [C, I64, P, P, I32, P, P, P, P, P, P, P]),
        "hga_cold_stage": (ctypes.c_int, [P, C, P, P, P, I32, P, I32]),
        "hga_warm_fill": (ctypes.c_int, [C, I64, P, P, P, P, I32, I32, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise HGAError(status, where, load_library().hga_last_error().decode())


def _ptr(x):
    """Raw address of a tensor (or an int address, or None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if not x.flags["C_CONTIGUOUS"]:  # a numpy array (host-side calls)
        raise ValueError("host arrays passed to the library must be C-contiguous")
    return x.ctypes.data


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclass
class Layer:
    """Shape and method parameters of one layer; ``config()`` gives the C struct."""

    batch: int
    heads_q: int
    heads_kv: int
    head_dim: int
    chunk: int = 64
    group: int = 16
    sink_chunks: int = 1
    local_chunks: int = 4
    topk_chunks: int = 16
    topk_groups: int = 32
    n_high_pairs: int = 32
    rope_theta: float = 500000.0
    dtype: int = HGA_BF16
    out_dtype: int = HGA_F32
    kv_loc: int = HGA_KV_DEVICE

    def config(self) -> HGAConfig:
        return HGAConfig(self.batch, self.heads_q, self.heads_kv, self.head_dim, self.chunk,
                         self.group, self.sink_chunks, self.local_chunks, self.topk_chunks,
                         self.topk_groups, self.n_high_pairs, self.dtype, self.out_dtype,
                         self.kv_loc, float(self.rope_theta))


def _cfg(cfg) -> HGAConfig:
    return cfg.config() if isinstance(cfg, Layer) else cfg


def hga_abi_version() -> int:
    return load_library().hga_abi_version()


def hga_status_string(status: int) -> str:
    return load_library().hga_status_string(status).decode()


def hga_device_status(stream=None) -> int:
    """Status of the device-side argument checks since the last call (clears them)."""
    return load_library().hga_device_status(_stream(stream))


def hga_workspace_size(cfg, n_alloc: int, q_len: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().hga_workspace_size(ctypes.byref(_cfg(cfg)), n_alloc, q_len,
                                             ctypes.byref(out)), "hga_workspace_size")
    return out.value


def hga_build_summaries(cfg, k, n_alloc: int, t_begin: int, t_end: int, chunk_sum, group_sum,
                        stream=None) -> None:
    _check(load_library().hga_build_summaries(ctypes.byref(_cfg(cfg)), _ptr(k), n_alloc, t_begin,
                                              t_end, _ptr(chunk_sum), _ptr(group_sum),
                                              _stream(stream)), "hga_build_summaries")


def hga_route_chunks(cfg, q, q_len: int, pos, chunk_sum, n_alloc: int, chunk_idx,
                     chunk_score=None, stream=None) -> None:
    _check(load_library().hga_route_chunks(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos),
                                           _ptr(chunk_sum), n_alloc, _ptr(chunk_idx),
                                           _ptr(chunk_score), _stream(stream)), "hga_route_chunks")


def hga_route_groups(cfg, q, q_len: int, pos, group_sum, n_alloc: int, chunk_idx, group_idx,
                     group_score=None, stream=None) -> None:
    _check(load_library().hga_route_groups(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos),
                                           _ptr(group_sum), n_alloc, _ptr(chunk_idx),
                                           _ptr(group_idx), _ptr(group_score), _stream(stream)),
           "hga_route_groups")


def hga_route(cfg, q, q_len: int, pos, chunk_sum, group_sum, n_alloc: int, chunk_idx, group_idx,
              chunk_score=None, group_score=None, stream=None) -> None:
    """Both routing levels in one launch (same results as the two separate calls)."""
    _check(load_library().hga_route(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos),
                                    _ptr(chunk_sum), _ptr(group_sum), n_alloc, _ptr(chunk_idx),
                                    _ptr(chunk_score), _ptr(group_idx), _ptr(group_score),
                                    _stream(stream)), "hga_route")


def hga_hot_rows(cfg) -> int:
    """Rows per (sequence, KV head) of the host tier's device working buffers."""
    out = ctypes.c_int64(0)
    _check(load_library().hga_hot_rows(ctypes.byref(_cfg(cfg)), ctypes.byref(out)), "hga_hot_rows")
    return out.value


def hga_decode_step_launches(cfg, n_alloc: int) -> int:
    """1 when hga_decode_step runs as one kernel for this shape, 2 when it launches two."""
    out = ctypes.c_int32(0)
    _check(load_library().hga_decode_step_launches(ctypes.byref(_cfg(cfg)), n_alloc,
                                                    ctypes.byref(out)), "hga_decode_step_launches")
    return out.value


def hga_gather_host(cfg, k_host, v_host, n_alloc: int, pos, group_idx, k_work, v_work,
                    refresh_window: int = 0, stream=None) -> None:
    """Host tier: stage the routed groups and window rows (refresh_window 0: the current
    chunk up to pos, 1: the whole window, 2: the row at pos only) from pinned host K/V."""
    _check(load_library().hga_gather_host(ctypes.byref(_cfg(cfg)), _ptr(k_host), _ptr(v_host),
                                          n_alloc, _ptr(pos), _ptr(group_idx), _ptr(k_work),
                                          _ptr(v_work), int(refresh_window),
                                          _stream(stream)), "hga_gather_host")


def hga_warm_rows(cfg, warm_groups: int) -> int:
    """Rows per (sequence, KV head) of the warm tier's device working buffers."""
    out = ctypes.c_int64(0)
    _check(load_library().hga_warm_rows(ctypes.byref(_cfg(cfg)), warm_groups, ctypes.byref(out)),
           "hga_warm_rows")
    return out.value


def hga_warm_reset(cfg, warm_groups: int, tags, stamps, seq: int = -1, stream=None) -> None:
    """Empty the warm tables of one sequence (or of all, seq=-1)."""
    _check(load_library().hga_warm_reset(ctypes.byref(_cfg(cfg)), warm_groups, _ptr(tags),
                                         _ptr(stamps), seq, _stream(stream)), "hga_warm_reset")


def hga_gather_warm(cfg, k_host, v_host, n_alloc: int, pos, group_idx, warm_groups: int, tags,
                    stamps, slot_map, k_work, v_work, refresh_window: int = 0, counters=None,
                    stream=None) -> None:
    """Warm tier step: LRU lookup/eviction, then only the missed groups from host K/V."""
    _check(load_library().hga_gather_warm(ctypes.byref(_cfg(cfg)), _ptr(k_host), _ptr(v_host),
                                          n_alloc, _ptr(pos), _ptr(group_idx), warm_groups,
                                          _ptr(tags), _ptr(stamps), _ptr(slot_map), _ptr(k_work),
                                          _ptr(v_work), int(refresh_window),
                                          _ptr(counters), _stream(stream)), "hga_gather_warm")


def hga_attend_warm(cfg, q, pos, k_work, v_work, n_alloc: int, group_idx, slot_map,
                    warm_groups: int, out, lse=None, stream=None) -> None:
    """Decode attention over the warm working buffers (routed groups via slot_map)."""
    _check(load_library().hga_attend_warm(ctypes.byref(_cfg(cfg)), _ptr(q), _ptr(pos),
                                          _ptr(k_work), _ptr(v_work), n_alloc, _ptr(group_idx),
                                          _ptr(slot_map), warm_groups, _ptr(out), _ptr(lse),
                                          _stream(stream)), "hga_attend_warm")


def hga_attend(cfg, q, q_len: int, pos, k, v, n_alloc: int, group_idx, out, lse=None,
               workspace=None, workspace_bytes: int = 0, stream=None) -> None:
    _check(load_library().hga_attend(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos), _ptr(k),
                                     _ptr(v), n_alloc, _ptr(group_idx), _ptr(out), _ptr(lse),
                                     _ptr(workspace), workspace_bytes, _stream(stream)),
           "hga_attend")


def hga_decode_step(cfg, q, pos, chunk_sum, group_sum, n_alloc: int, k, v, chunk_idx, group_idx,
                    out, lse=None, chunk_score=None, group_score=None, append: bool = False,
                    stream=None) -> None:
    """One decode step: the summary append (if asked), routing and attention."""
    _check(load_library().hga_decode_step(ctypes.byref(_cfg(cfg)), _ptr(q), _ptr(pos),
                                          _ptr(chunk_sum), _ptr(group_sum), n_alloc, _ptr(k),
                                          _ptr(v), _ptr(chunk_idx), _ptr(chunk_score),
                                          _ptr(group_idx), _ptr(group_score), _ptr(out),
                                          _ptr(lse), 1 if append else 0, _stream(stream)),
           "hga_decode_step")


def kv_pages(block_table, n_pages: int, page_size: int, max_pages: int) -> HGAKvPages:
    """A paged pool's description: block_table (device int32 [B, max_pages]) and sizes."""
    return HGAKvPages(_ptr(block_table), n_pages, page_size, max_pages)


def hga_build_summaries_paged(cfg, k_pages, kv: HGAKvPages, seq_len, chunk_sum, group_sum,
                              stream=None) -> None:
    """Summaries of a ragged batch over a paged pool: sequence b's rows up to seq_len[b]."""
    _check(load_library().hga_build_summaries_paged(ctypes.byref(_cfg(cfg)), _ptr(k_pages),
                                                    ctypes.byref(kv), _ptr(seq_len),
                                                    _ptr(chunk_sum), _ptr(group_sum),
                                                    _stream(stream)), "hga_build_summaries_paged")


def hga_decode_step_paged(cfg, q, pos, chunk_sum, group_sum, k_pages, v_pages, kv: HGAKvPages,
                          chunk_idx, group_idx, out, lse=None, chunk_score=None, group_score=None,
                          append: bool = False, stream=None) -> None:
    """hga_decode_step over a paged pool (one launch)."""
    _check(load_library().hga_decode_step_paged(ctypes.byref(_cfg(cfg)), _ptr(q), _ptr(pos),
                                                _ptr(chunk_sum), _ptr(group_sum), _ptr(k_pages),
                                                _ptr(v_pages), ctypes.byref(kv), _ptr(chunk_idx),
                                                _ptr(chunk_score), _ptr(group_idx),
                                                _ptr(group_score), _ptr(out), _ptr(lse),
                                                1 if append else 0, _stream(stream)),
           "hga_decode_step_paged")


def hga_attend_backward_workspace_size(cfg, n_alloc: int, q_len: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().hga_attend_backward_workspace_size(ctypes.byref(_cfg(cfg)), n_alloc,
                                                             q_len, ctypes.byref(out)),
           "hga_attend_backward_workspace_size")
    return out.value


def hga_attend_backward(cfg, q, q_len: int, pos, k, v, n_alloc: int, group_idx, out, lse, d_out,
                        dq, dk, dv, workspace, workspace_bytes: int, stream=None) -> None:
    """dQ, dK, dV of a prefill attention over its routed index sets."""
    _check(load_library().hga_attend_backward(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos),
                                              _ptr(k), _ptr(v), n_alloc, _ptr(group_idx),
                                              _ptr(out), _ptr(lse), _ptr(d_out), _ptr(dq),
                                              _ptr(dk), _ptr(dv), _ptr(workspace),
                                              workspace_bytes, _stream(stream)),
           "hga_attend_backward")


class ColdStore:
    """A file-backed K/V history (the cold tier); close() or use as a context manager."""

    def __init__(self, path: str, cfg, n_alloc: int, create: bool = False):
        self.handle = ctypes.c_void_p()
        _check(load_library().hga_cold_open(str(path).encode(), ctypes.byref(_cfg(cfg)), n_alloc,
                                            1 if create else 0, ctypes.byref(self.handle)),
               "hga_cold_open")

    def write(self, k, v, t0: int, t1: int, threads: int = 8) -> None:
        _check(load_library().hga_cold_write(self.handle, _ptr(k), _ptr(v), t0, t1, threads),
               "hga_cold_write")

    def stage(self, cfg, pos, plan, n_plan, window_mode: int, staging, threads: int = 8) -> None:
        _check(load_library().hga_cold_stage(self.handle, ctypes.byref(_cfg(cfg)), _ptr(pos),
                                             _ptr(plan), _ptr(n_plan), window_mode, _ptr(staging),
                                             threads), "hga_cold_stage")

    def close(self) -> None:
        if self.handle:
            _check(load_library().hga_cold_close(self.handle), "hga_cold_close")
            self.handle = ctypes.c_void_p()

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def hga_cold_stage_bytes(cfg) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().hga_cold_stage_bytes(ctypes.byref(_cfg(cfg)), ctypes.byref(out)),
           "hga_cold_stage_bytes")
    return out.value


def hga_warm_plan(cfg, n_alloc: int, pos, group_idx, warm_groups: int, tags, stamps, slot_map,
                  plan, n_plan, counters=None, stream=None) -> None:
    """The warm tier's table update alone: misses as (group, slot) pairs for a cold store."""
    _check(load_library().hga_warm_plan(ctypes.byref(_cfg(cfg)), n_alloc, _ptr(pos),
                                        _ptr(group_idx), warm_groups, _ptr(tags), _ptr(stamps),
                                        _ptr(slot_map), _ptr(plan), _ptr(n_plan), _ptr(counters),
                                        _stream(stream)), "hga_warm_plan")


def hga_warm_fill(cfg, n_alloc: int, pos, staging, plan, n_plan, warm_groups: int,
                  window_mode: int, k_work, v_work, stream=None) -> None:
    """Copies a cold store's staged rows into the warm working buffers."""
    _check(load_library().hga_warm_fill(ctypes.byref(_cfg(cfg)), n_alloc, _ptr(pos),
                                        _ptr(staging), _ptr(plan), _ptr(n_plan), warm_groups,
                                        window_mode, _ptr(k_work), _ptr(v_work), _stream(stream)),
           "hga_warm_fill")


def hga_debug_inject(flags: int) -> int:
    """Test hook: sets the library's debug flags for later launches; returns the old flags."""
    return load_library().hga_debug_inject(flags)


def hga_attend_noalloc(cfg, q, q_len: int, pos, k, v, n_alloc: int, group_idx, out, lse=None,
                       stream=None) -> None:
    """hga_attend without a caller workspace, for callers that cannot allocate.

    Frameworks that own all device memory and hand a plugin only its inputs and
    outputs, or loops where cudaMalloc/cudaFree (which may synchronise the
    device) is not allowed, can use this call: the split-K scratch lives in a
    fixed 8 MiB array inside the library.  Larger shapes raise HGAError
    (HGA_ERR_WORKSPACE).  The first call on a device looks up the array's
    address, so make it before any stream capture; calls that overlap on the
    GPU share the array and race.
    """
    _check(load_library().hga_attend_noalloc(ctypes.byref(_cfg(cfg)), _ptr(q), q_len, _ptr(pos),
                                             _ptr(k), _ptr(v), n_alloc, _ptr(group_idx),
                                             _ptr(out), _ptr(lse), _stream(stream)),
           "hga_attend_noalloc")
