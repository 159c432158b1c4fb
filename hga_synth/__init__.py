"""Seeded synthetic inputs for the HGA hot path.

This module is shared by the tests, the benchmark, the oracle side and the
CUDA side.  It holds no step of the method's arithmetic: it only draws random
tensors, plants the synthetic structure the workloads call for (needle chunks,
log-normal key norms) and stores values once in their storage type, so that
both sides read identical bytes.

Every tensor slice has its own counter-derived stream
``numpy.random.default_rng([seed, tensor_id, b, h])``, so one (sequence, KV
head) slice can be regenerated alone, at any context length, without drawing
the rest.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

# tensor ids of the sub-streams
_Q, _K, _V, _NEEDLE, _LOGNORM, _DRIFT, _REQ = 0, 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    """Shape and method parameters of one synthetic attention layer."""

    name: str
    batch: int
    heads_q: int
    heads_kv: int
    head_dim: int
    context: int               # N, tokens already in the cache (decode query at N-1)
    dtype: str                 # "f32" or "bf16": storage type of q, k, v
    rope_theta: float
    n_high_pairs: int
    chunk: int = 64
    group: int = 16
    sink: int = 1
    local: int = 4
    topk_chunks: int = 16
    topk_groups: int = 32
    needles: int = 0           # planted needle chunks per (sequence, KV head)
    needle_cos: float = 0.9
    lognormal_sigma: float = 0.0
    prefill: bool = False      # queries cover the whole context in blocks of C

    @property
    def gqa(self) -> int:
        return self.heads_q // self.heads_kv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the hot path, by what they are.
WORKLOADS = {
    # Tiny single-layer check: 1 query head, 1 KV head, D=64, 1024 tokens, fp32.
    "tiny_f32_1k": Workload("tiny_f32_1k", batch=1, heads_q=1, heads_kv=1, head_dim=64,
                            context=1024, dtype="f32", rope_theta=1e4, n_high_pairs=16,
                            chunk=64, group=16, sink=1, local=2, topk_chunks=4, topk_groups=8),
    # Llama-3-8B-shaped decode layer at 32K context (GQA 32/8, D=128), 2 needles per head.
    "llama3_8b_decode_32k": Workload("llama3_8b_decode_32k", batch=16, heads_q=32, heads_kv=8,
                                     head_dim=128, context=32768, dtype="bf16", rope_theta=5e5,
                                     n_high_pairs=32, needles=2),
    # Chunked prefill of the same layer shape at 64K context, batch 1.
    "llama3_8b_prefill_64k": Workload("llama3_8b_prefill_64k", batch=1, heads_q=32, heads_kv=8,
                                      head_dim=128, context=65536, dtype="bf16", rope_theta=5e5,
                                      n_high_pairs=32, prefill=True),
    # Host-tier decode at 128K context, batch 8: full K/V in pinned host memory.
    "host_tier_decode_128k": Workload("host_tier_decode_128k", batch=8, heads_q=32, heads_kv=8,
                                      head_dim=128, context=131072, dtype="bf16", rope_theta=5e5,
                                      n_high_pairs=32),
    # Wide-head decode stress: 64/8 heads, 64K context, batch 32, log-normal key norms.
    "wide_head_decode_64k": Workload("wide_head_decode_64k", batch=32, heads_q=64, heads_kv=8,
                                     head_dim=128, context=65536, dtype="bf16", rope_theta=5e5,
                                     n_high_pairs=32, lognormal_sigma=0.5),
}


def workload(name: str, **overrides) -> Workload:
    return WORKLOADS[name].with_(**overrides)


# ------------------------------------------------------------- storage types

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def store(x: np.ndarray, dtype: str) -> np.ndarray:
    """Store float values in the workload's storage type (float32, or bf16 bits as uint16)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))
    raise ValueError(dtype)


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored values as float64 (exact)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64)
    return bf16_bits_to_f32(x).astype(np.float64)


# ------------------------------------------------------------------ generators

def _rng(seed: int, tensor: int, *idx: int) -> np.random.Generator:
    return np.random.default_rng([seed, tensor, *idx])


def query_slice(wl: Workload, seed: int, b: int, q_len: int | None = None) -> np.ndarray:
    """Stored post-RoPE queries of sequence b: [Hq, q_len, D] ~ N(0,1)."""
    q_len = (wl.context if wl.prefill else 1) if q_len is None else q_len
    z = _rng(seed, _Q, b).standard_normal((wl.heads_q, q_len, wl.head_dim), dtype=np.float32)
    return store(z, wl.dtype)


def needle_chunks(wl: Workload, seed: int, b: int, h: int) -> np.ndarray:
    """The planted needle chunks of (b, h): distinct intermediate-context chunks of the decode query."""
    cur = (wl.context - 1) // wl.chunk
    lo, hi = wl.sink, cur - wl.local
    if wl.needles == 0 or hi - lo < wl.needles:
        return np.zeros(0, dtype=np.int64)
    return np.sort(_rng(seed, _NEEDLE, b, h).choice(np.arange(lo, hi), size=wl.needles, replace=False))


def key_slice(wl: Workload, seed: int, b: int, h: int, q_stored: np.ndarray | None = None) -> np.ndarray:
    """Stored post-RoPE keys of (b, h): [N, D].

    N(0,1) entries; with ``lognormal_sigma`` every key row is scaled by
    exp(sigma * z), z ~ N(0,1); with ``needles`` the keys of the planted chunks
    are turned towards the decode query direction (cosine ``needle_cos``),
    keeping each key's norm:  k = |k| (c * u + sqrt(1 - c^2) * w), where u is
    the unit mean of the stored queries of the G heads sharing KV head h and w
    a random unit vector orthogonal to u.
    """
    n, d = wl.context, wl.head_dim
    k = _rng(seed, _K, b, h).standard_normal((n, d), dtype=np.float32)
    if wl.lognormal_sigma:
        z = _rng(seed, _LOGNORM, b, h).standard_normal(n).astype(np.float32)
        k *= np.exp(np.float32(wl.lognormal_sigma) * z)[:, None]
    chunks = needle_chunks(wl, seed, b, h)
    if len(chunks):
        if q_stored is None:
            q_stored = query_slice(wl, seed, b, q_len=1)
        g = wl.gqa
        u = widen(q_stored[h * g:(h + 1) * g, -1], wl.dtype).mean(axis=0)
        u /= np.linalg.norm(u)
        rng = _rng(seed, _NEEDLE, b, h, 1)
        c = wl.needle_cos
        for ch in chunks:
            rows = slice(ch * wl.chunk, (ch + 1) * wl.chunk)
            kk = k[rows].astype(np.float64)
            w = rng.standard_normal(kk.shape)
            w -= (w @ u)[:, None] * u[None, :]
            w /= np.linalg.norm(w, axis=1, keepdims=True)
            norm = np.linalg.norm(kk, axis=1, keepdims=True)
            k[rows] = (norm * (c * u[None, :] + math.sqrt(1.0 - c * c) * w)).astype(np.float32)
    return store(k, wl.dtype)


def value_slice(wl: Workload, seed: int, b: int, h: int) -> np.ndarray:
    """Stored values of (b, h): [N, D] ~ N(0,1)."""
    z = _rng(seed, _V, b, h).standard_normal((wl.context, wl.head_dim), dtype=np.float32)
    return store(z, wl.dtype)


def make_inputs(wl: Workload, seed: int, q_len: int | None = None) -> dict:
    """All stored inputs of a workload.

    Returns q [B, Hq, q_len, D], k and v [B, Hkv, N, D] (float32 arrays, or
    uint16 bf16 bits) and pos [B] int64, the position of each sequence's last
    query (N-1).
    """
    q_len = (wl.context if wl.prefill else 1) if q_len is None else q_len
    qs = [query_slice(wl, seed, b, q_len) for b in range(wl.batch)]
    q1 = [query_slice(wl, seed, b, 1) if q_len != 1 else qs[b] for b in range(wl.batch)]
    k = np.stack([np.stack([key_slice(wl, seed, b, h, q1[b]) for h in range(wl.heads_kv)])
                  for b in range(wl.batch)])
    v = np.stack([np.stack([value_slice(wl, seed, b, h) for h in range(wl.heads_kv)])
                  for b in range(wl.batch)])
    pos = np.full(wl.batch, wl.context - 1, dtype=np.int64)
    return dict(q=np.stack(qs), k=k, v=v, pos=pos)


def drifting_queries(wl: Workload, seed: int, steps: int, rho: float) -> np.ndarray:
    """Stored decode queries of `steps` consecutive steps: [steps, B, Hq, 1, D].

    Step 0 is query_slice's query; every next one keeps a share rho of the last:
    q_t = rho * q_{t-1} + sqrt(1 - rho^2) * z_t, z_t ~ N(0,1) (a stationary
    AR(1) walk, drawn in float64 and stored once per step), so that
    consecutive decode steps route to overlapping groups as a real decode
    does."""
    out = np.empty((steps, wl.batch, wl.heads_q, 1, wl.head_dim),
                   dtype=np.uint16 if wl.dtype == "bf16" else np.float32)
    c = math.sqrt(max(0.0, 1.0 - rho * rho))
    for b in range(wl.batch):
        cur = widen(query_slice(wl, seed, b, 1), wl.dtype)
        out[0, b] = store(cur, wl.dtype)
        rng = _rng(seed, _DRIFT, b)
        for t in range(1, steps):
            cur = rho * cur + c * rng.standard_normal(cur.shape)
            out[t, b] = store(cur, wl.dtype)
    return out


def group_requests(wl: Workload, seed: int, steps: int, pos: np.ndarray, keep: float,
                   kg: int | None = None) -> np.ndarray:
    """Synthetic level-2 selections for the warm tier: [steps, B, Hkv, kg] int32.

    Every row holds kg distinct groups of candidate chunks of pos[b] (chunk c
    with sink <= c < pos[b] // C - local), ascending, padded with -1 when fewer
    exist; from one step to the next each group stays with probability `keep`
    and the others are drawn afresh from the candidates."""
    kg = wl.topk_groups if kg is None else kg
    gpc = wl.chunk // wl.group
    out = np.full((steps, wl.batch, wl.heads_kv, kg), -1, dtype=np.int32)
    for b in range(wl.batch):
        lo, hi = wl.sink * gpc, max(wl.sink, int(pos[b]) // wl.chunk - wl.local) * gpc
        cand = np.arange(lo, hi)
        n = min(kg, len(cand))
        for h in range(wl.heads_kv):
            rng = _rng(seed, _REQ, b, h)
            cur = np.sort(rng.choice(cand, n, replace=False)) if n else cand[:0]
            for t in range(steps):
                if t:
                    stay = cur[rng.random(len(cur)) < keep]
                    pool = np.setdiff1d(cand, stay)
                    cur = np.sort(np.concatenate([stay, rng.choice(pool, n - len(stay),
                                                                   replace=False)]))
                out[t, b, h, :n] = cur
    return out


def seed_for(index: int) -> int:
    """Seed of the i-th workload (1000 + i)."""
    return 1000 + index
