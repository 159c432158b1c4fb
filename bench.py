"""Benchmark of the HGA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--batch B]
    python bench.py --impl reference ...      # the float64 CPU oracle, timed on host cores

One step = one decode step of one attention layer for the whole batch: append
the new token's summary rows, route chunks, route groups, attend (steps 1-5 of
the HGA hot path), on inputs already resident in HBM.  The append writes rows
of the current chunk only, which the same step never routes, so it runs on a
side stream beside the routing/attention chain (one CUDA graph per step).  L2 is flushed (a 256 MB
write) before every timed step, outside the timed events.  Prints one JSON line.

Multi-GPU (torchrun, one process per GPU): every rank decodes its own batch of
independent sequences (weak scaling, no collective on the data path); the
step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hga_synth as S  # noqa: E402

METRIC = "HGA decode tokens/s + attn µs/layer at 32K–128K ctx; % HBM roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--workload", default="llama3_8b_decode_32k")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--context", type=int, default=None, help="override the context length")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def profile_traffic(kernel: str, wl: S.Workload):
    """DRAM bytes per launch of `kernel` from a committed ncu capture (profiles/*.md).

    The capture may be of a smaller case of the same workload; its bytes are
    scaled by the units processed (the line's `scale`: batch, or batch*context).
    Returns None when no capture covers the kernel or when its source file has
    changed since the counters were taken.
    """
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(path):
            if not line.startswith("traffic:"):
                continue
            kv = dict(x.split("=", 1) for x in line.split()[1:])
            if kv.get("kernel") != kernel or kv.get("workload") != wl.name:
                continue
            src = os.path.join(ROOT, kv["source"])
            if not os.path.exists(src):
                return None
            if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != kv["sha256_16"]:
                return None  # the kernel changed since the counters were taken
            ratio = wl.batch / int(kv["batch"])
            if kv.get("scale") == "batch*context":
                ratio *= wl.context / int(kv["context"])
            return int(float(kv["dram_bytes"]) * ratio)
    return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------- byte counts

def step_bytes(wl: S.Workload) -> dict:
    """Algorithmic HBM bytes of one decode step per kernel (whole batch).

    route_chunks: the candidate chunk-summary rows (fp32) + the G query rows;
    route_groups: the groups of the kc selected chunks + query rows + chunk ids;
    attend: K and V rows of the T routed tokens + query rows + output (fp32);
    summaries: the closing chunk's and group's key rows + the rows written.
    """
    e = 2 if wl.dtype == "bf16" else 4
    d, g = wl.head_dim, wl.gqa
    p = wl.context - 1
    cur = p // wl.chunk
    n_cand = max(0, cur - wl.local - wl.sink)
    kc = min(wl.topk_chunks, n_cand)
    ng = wl.chunk // wl.group
    kg = min(wl.topk_groups, kc * ng)
    forced = (min(wl.sink, max(0, cur - wl.local)) * wl.chunk + (p - max(0, cur - wl.local) * wl.chunk + 1))
    t = forced + kg * wl.group
    units = wl.batch * wl.heads_kv
    qrow = g * d * e
    closes_chunk = (p + 1) % wl.chunk == 0
    closes_group = (p + 1) % wl.group == 0
    summ = 0
    if closes_chunk:
        summ = wl.chunk * d * e + (d + ng * d) * 4
    elif closes_group:
        summ = wl.group * d * e + d * 4
    return dict(
        summaries=units * summ,
        route_chunks=units * (n_cand * d * 4 + qrow),
        route_groups=units * (kc * ng * d * 4 + qrow + wl.topk_chunks * 4),
        attend=units * (t * d * e * 2 + qrow + g * d * 4 + wl.topk_groups * 4),
        tokens=t,
    )


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv:
            self._t.join()

    def report(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ ranks (N > 1)

class Ranks:
    """Cross-rank plumbing of the timed region (one process per GPU).

    Every rank takes the same steps in the same order: a barrier before and
    after the timed steps, and a MAX reduction of each time it reports.  With
    one rank every call is a no-op.  The data path itself has no collective:
    the ranks decode independent sequences (weak scaling).
    """

    def __init__(self, world: int, device):
        self.world = world
        self.device = device
        self.dist = None
        if world > 1:
            import torch.distributed as dist
            self.dist = dist

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def max(self, value: float) -> float:
        if not self.dist:
            return value
        import torch
        t = torch.tensor([value], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())


def init_ranks(backend: str) -> tuple[int, int]:
    """Joins the process group torchrun describes in the environment."""
    import datetime

    import torch.distributed as dist
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if world > 1:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def rank_seed(workload: str, rank: int) -> int:
    """Input seed of one rank: each rank's sequences are distinct."""
    return S.seed_for(list(S.WORKLOADS).index(workload)) + 7919 * rank


def job_rate(units_per_rank: float, world: int, ms_step: float) -> float:
    """Whole-job throughput: the units all ranks processed over the max-over-ranks time."""
    return units_per_rank * world / (ms_step * 1e-3)


# ------------------------------------------------------------------ CUDA arm

def run_hga(args, rank: int, world: int):
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B
    from hierarchical_sparse_attention_hga_b200.build import build

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    build()
    B.load_library()
    wl = S.workload(args.workload)
    if args.batch:
        wl = wl.with_(batch=args.batch)
    if args.context:
        wl = wl.with_(context=args.context)
    if wl.prefill:
        return run_prefill(args, rank, world, wl)
    dev = torch.device("cuda")
    seed = rank_seed(args.workload, rank)
    x = S.make_inputs(wl, seed)
    n = wl.context
    p = n - 1

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16 if wl.dtype == "bf16" else np.float32))
        return (t.view(torch.bfloat16) if wl.dtype == "bf16" else t).to(dev)

    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    pos = torch.as_tensor(x["pos"], device=dev)
    layer = B.Layer(batch=wl.batch, heads_q=wl.heads_q, heads_kv=wl.heads_kv, head_dim=wl.head_dim,
                    chunk=wl.chunk, group=wl.group, sink_chunks=wl.sink, local_chunks=wl.local,
                    topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                    n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta,
                    dtype=B.HGA_BF16 if wl.dtype == "bf16" else B.HGA_F32, out_dtype=B.HGA_F32)
    bh = wl.batch * wl.heads_kv
    nc, ng = n // wl.chunk, wl.chunk // wl.group
    # Host tier: the whole K/V cache in pinned host memory; the GPU keeps the
    # summaries and a working buffer (windows + the step's routed groups).
    hot = wl.name.startswith("host_tier")
    if hot:
        layer.kv_loc = B.HGA_KV_HOST_PINNED
        k_host, v_host = k.cpu().pin_memory(), v.cpu().pin_memory()
        del k, v
        torch.cuda.empty_cache()
        rows = B.hga_hot_rows(layer)
        k_work = torch.empty(bh, rows, wl.head_dim, dtype=torch.bfloat16, device=dev)
        v_work = torch.empty_like(k_work)
        k_src, v_src = k_host, v_host
    else:
        k_src, v_src = k, v
    cs = torch.empty(bh, nc, wl.head_dim, device=dev)
    gs = torch.empty(bh, nc, ng, wl.head_dim, device=dev)
    ci = torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device=dev)
    gi = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device=dev)
    out = torch.empty(wl.batch, wl.heads_q, 1, wl.head_dim, device=dev)
    lse = torch.empty(wl.batch, wl.heads_q, 1, device=dev)
    wsb = B.hga_workspace_size(layer, n, 1)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    # prefix summaries (setup, untimed): every row closed before the new token
    B.hga_build_summaries(layer, k_src, n, 0, p, cs, gs, stream=sh)
    if hot:  # fill the working buffer's windows once
        B.hga_route(layer, q, 1, pos, cs, gs, n, ci, gi, stream=sh)
        B.hga_gather_host(layer, k_host, v_host, n, pos, gi, k_work, v_work, refresh_window=True,
                          stream=sh)

    parts = {
        "summaries": lambda st: B.hga_build_summaries(layer, k_src, n, p, p + 1, cs, gs, stream=st),
        "route": lambda st: B.hga_route(layer, q, 1, pos, cs, gs, n, ci, gi, stream=st),
        "attend": lambda st: B.hga_attend(layer, q, 1, pos, k_work if hot else k_src,
                                          v_work if hot else v_src, n, gi, out, lse, ws, wsb,
                                          stream=st),
        "route_chunks": lambda st: B.hga_route_chunks(layer, q, 1, pos, cs, n, ci, stream=st),
        "route_groups": lambda st: B.hga_route_groups(layer, q, 1, pos, gs, n, ci, gi, stream=st),
    }
    if hot:
        parts["gather"] = lambda st: B.hga_gather_host(layer, k_host, v_host, n, pos, gi, k_work,
                                                       v_work, stream=st)
    # routing and attention in one launch (bf16, D = 128, K/V in device memory)
    fused = not hot and wl.dtype == "bf16" and wl.head_dim == 128 and wl.group == 16 and wl.gqa <= 16
    if fused:  # the whole step: summary append, routing and attention
        parts["decode_step"] = lambda st: B.hga_decode_step(layer, q, pos, cs, gs, n, k_src, v_src,
                                                            ci, gi, out, lse, append=True,
                                                            stream=st)

    side = torch.cuda.Stream()

    def make_step(chain):
        def step(st):
            # The rows the new token closes belong to the current chunk, which
            # this step never routes (it is always visible), so the append runs
            # on a side stream, concurrently with routing and attention.
            main = torch.cuda.current_stream()
            side.wait_stream(main)
            with torch.cuda.stream(side):
                parts["summaries"](side.cuda_stream)
            for name in chain:
                parts[name](st)
            main.wait_stream(side)
        return step

    if hot:
        step = make_step(("route", "gather", "attend"))
        step2 = step
        step4 = make_step(("route_chunks", "route_groups", "gather", "attend"))
    else:
        # The timed step: hga_decode_step with the summary append (one launch when the
        # batch has at least half a (sequence, KV head) item per SM, else the append,
        # routing and attention kernels); the two-call and four-call steps (append on a
        # side stream) are reported beside it.
        step2 = make_step(("route", "attend"))
        step = parts["decode_step"] if fused else step2
        step4 = make_step(("route_chunks", "route_groups", "attend"))

    # eager warm-up, then one CUDA graph for the whole step and one per call
    for _ in range(max(1, args.warmup)):
        step(sh)
    torch.cuda.synchronize()
    assert B.hga_device_status(sh) == 0
    graphs = {}
    steps = [("step", step), ("step2", step2), ("step4", step4)]
    for name, fn in list(parts.items()) + steps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(torch.cuda.current_stream().cuda_stream)
        graphs[name] = g
    torch.cuda.synchronize()

    def timed(g, iters):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(iters)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(iters)]
        for i in range(iters):
            flush.zero_()              # L2 flush, outside the timed events
            starts[i].record(stream)
            g.replay()
            ends[i].record(stream)
        return starts, ends

    for _ in range(args.warmup):
        flush.zero_()
        graphs["step"].replay()
    ranks = Ranks(world, dev)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        starts, ends = timed(graphs["step"], args.steps)
        torch.cuda.synchronize()
    ranks.barrier()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms_step = sum(step_ms) / len(step_ms)
    a4, b4 = timed(graphs["step4"], min(args.steps, 200))
    torch.cuda.synchronize()
    ms_step4 = sum(x.elapsed_time(y) for x, y in zip(a4, b4)) / len(a4)
    a2, b2 = timed(graphs["step2"], min(args.steps, 200))
    torch.cuda.synchronize()
    ms_step2 = sum(x.elapsed_time(y) for x, y in zip(a2, b2)) / len(a2)
    ms_step = ranks.max(ms_step)
    assert B.hga_device_status(sh) == 0
    # timing floor: an empty graph-sized launch measured the same way
    g_floor = torch.cuda.CUDAGraph()
    dummy = torch.zeros(1, device=dev)
    with torch.cuda.graph(g_floor):
        dummy.add_(1)
    a_, b_ = timed(g_floor, 50)
    torch.cuda.synchronize()
    floor_us = 1e3 * sum(x.elapsed_time(y) for x, y in zip(a_, b_)) / len(a_)
    # per-call breakdown: each call's graph replayed alone after an L2 flush
    ms = {}
    for name in parts:
        a_, b_ = timed(graphs[name], min(args.steps, 200))
        torch.cuda.synchronize()
        ms[name] = sum(x.elapsed_time(y) for x, y in zip(a_, b_)) / len(a_)

    # ---- e2e: host (pinned) q and new K/V rows in, output back, every step
    q_host = torch.from_numpy(np.ascontiguousarray(x["q"]).view(np.int16)).pin_memory() \
        if wl.dtype == "bf16" else torch.from_numpy(x["q"]).pin_memory()
    kv_new = torch.empty(2, wl.batch, wl.heads_kv, wl.head_dim, dtype=torch.bfloat16).pin_memory()
    kv_new[0].copy_(k_src[:, :, p].cpu())
    kv_new[1].copy_(v_src[:, :, p].cpu())
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    qv = q.view(torch.int16) if wl.dtype == "bf16" else q
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = []
    for i in range(args.warmup + min(args.steps, 200)):
        flush.zero_()
        e0.record(stream)
        qv.copy_(q_host, non_blocking=True)
        if hot:  # the new token's K/V goes into the host cache, a host-side write
            k_host[:, :, p].copy_(kv_new[0])
            v_host[:, :, p].copy_(kv_new[1])
        else:
            k_src[:, :, p].copy_(kv_new[0], non_blocking=True)
            v_src[:, :, p].copy_(kv_new[1], non_blocking=True)
        graphs["step"].replay()
        out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= args.warmup:
            e2e.append(e0.elapsed_time(e1))
    ms_e2e = sum(e2e) / len(e2e)
    ms_e2e = ranks.max(ms_e2e)
    h2d = q_host.numel() * q_host.element_size() + (0 if hot else kv_new.numel() * kv_new.element_size())
    d2h = out_host.numel() * out_host.element_size()

    nb = step_bytes(wl)
    nb["route"] = nb["route_chunks"] + nb["route_groups"]
    # one launch reads the query rows once
    nb["decode_step"] = nb["summaries"] + nb["route"] + nb["attend"] - \
        2 * wl.batch * wl.heads_kv * wl.gqa * wl.head_dim * (2 if wl.dtype == "bf16" else 4)
    # the library says whether hga_decode_step is its one-launch kernel for this shape
    one_launch = fused and B.hga_decode_step_launches(layer, n) == 1
    kern = "decode_step" if one_launch else max(("route", "attend"), key=lambda kk: ms[kk])
    kernel_name = {"decode_step": "decode_step_kernel", "route": "route_decode_kernel",
                   "attend": "attend_decode_bf16_kernel"}[kern]
    # The roofline kernel's duration: CUDA events on the launch stream around a direct
    # launch queued behind the L2 flush (the host enqueues the call while the flush
    # runs, so the events bracket the GPU work, without the graph launch latency
    # that the per-call graph replays above include).
    n_direct = min(args.steps, 200)
    ds = [torch.cuda.Event(enable_timing=True) for _ in range(n_direct)]
    de = [torch.cuda.Event(enable_timing=True) for _ in range(n_direct)]
    for i in range(n_direct):
        flush.zero_()
        ds[i].record(stream)
        parts[kern](sh)
        de[i].record(stream)
    torch.cuda.synchronize()
    kern_ms = ranks.max(sum(x.elapsed_time(y) for x, y in zip(ds, de)) / n_direct)
    assert B.hga_device_status(sh) == 0
    hbm, peak_kind = peaks()
    achieved = nb[kern] / (kern_ms * 1e-3) / 1e9
    total_bytes = nb["summaries"] + nb["route"] + nb["attend"]
    if one_launch:
        launches_per_step = 1  # the decode step, summary append included
    elif fused:
        launches_per_step = 3  # summary append, routing, attention
    else:
        # summaries, route, (gather,) attend (+ the split-K combine when a workspace is used)
        launches_per_step = 3 + (1 if wsb > 0 else 0) + (1 if hot else 0)
    tokens = wl.batch  # per rank
    line = {
        "metric": METRIC,
        "value": job_rate(tokens, world, ms_step),
        "unit": "decode tokens/s (one attention layer)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step,
        "attn_us_per_layer": ms_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 K/V, fp32 accumulation" if wl.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) q/k/v" +
                (f"; {wl.needles} needle chunks per KV head" if wl.needles else "") +
                (f"; log-normal key norms, sigma {wl.lognormal_sigma}" if wl.lognormal_sigma else "") +
                ("; K/V in pinned host memory" if hot else "") + ")",
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": n,
                   "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
                   "chunk": wl.chunk, "group": wl.group, "sink": wl.sink, "local": wl.local,
                   "topk_chunks": wl.topk_chunks, "topk_groups": wl.topk_groups,
                   "tokens_attended_per_kv_head": nb["tokens"],
                   "l2": "flushed (256 MB write) before every timed step",
                   "parallelism": f"replicas x{world} (independent sequences per GPU)"},
        "per_kernel_us": {kk: ms[kk] * 1e3 for kk in parts},
        "two_call_step_us": ms_step2 * 1e3,
        "four_call_step_us": ms_step4 * 1e3,
        "timing_floor_us": floor_us,
        "step_hbm_bytes": total_bytes,
        "step_hbm_gbs": total_bytes / (ms_step * 1e-3) / 1e9,
        "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": profile_traffic(kernel_name, wl),
                     "algorithmic_bytes": nb[kern], "kernel_us": kern_ms * 1e3,
                     "graph_replay_us": ms[kern] * 1e3,
                     "duration": "CUDA events on the launch stream around a direct launch of the "
                                 "call, queued behind the L2 flush (mean of the timed launches); "
                                 "graph_replay_us is the call's CUDA graph replayed the same way"},
        "e2e": {"value": job_rate(tokens, world, ms_e2e), "unit": "decode tokens/s (one attention layer)",
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "host_link": host_link_report(wl, ms, dev) if hot else None,
        "timing": "CUDA graph of the step replayed per timed step; CUDA events on the launch stream",
        "clocks": clk.report(),
    }
    return line, wl, seed, x


def host_link_report(wl: S.Workload, ms: dict, dev) -> dict:
    """Host-tier traffic over the host link per step, against a pinned H2D copy probe."""
    import torch
    cur = (wl.context - 1) // wl.chunk
    cur_rows = wl.context - 1 - cur * wl.chunk + 1
    row = wl.head_dim * 2 * 2  # K and V, bf16
    units = wl.batch * wl.heads_kv
    routed = units * wl.topk_groups * wl.group * row
    window = units * cur_rows * row
    src = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = 0.0
    for _ in range(5):
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        e1.synchronize()
        best = max(best, src.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    gbs = (routed + window) / (ms["gather"] * 1e-3) / 1e9
    return {"bytes_per_step": routed + window, "routed_bytes": routed, "window_bytes": window,
            "gather_us": ms["gather"] * 1e3, "achieved_gbs": gbs, "h2d_copy_probe_gbs": best,
            "frac_of_probe": gbs / best}


# ------------------------------------------------------------------ prefill

def prefill_flops(wl: S.Workload) -> float:
    """Algorithmic FLOPs of the prefill attention (masked work excluded).

    Per (sequence, KV head, block j) every query row sees the forced chunks
    before the block, the routed groups and the causal part of its own chunk;
    each visible (row, key) pair costs 4*D flops (Q K^T and P V).
    """
    c, g = wl.chunk, wl.group
    ng = c // g
    total_keys = 0
    for j in range(wl.context // c):
        b0 = max(0, j - wl.local)
        forced = (min(wl.sink, b0) + (j - b0)) * c
        n_cand = max(0, j - wl.local - wl.sink)
        routed = min(wl.topk_groups, ng * min(wl.topk_chunks, n_cand)) * g
        total_keys += c * (forced + routed) + c * (c + 1) // 2
    return 4.0 * wl.head_dim * wl.gqa * total_keys * wl.batch * wl.heads_kv


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (burst)"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def run_prefill(args, rank: int, world: int, wl: S.Workload):
    """One prefill step of one layer: summaries of the whole prompt, routing of
    every 64-query block, attention of every query (steps 1-5)."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = torch.device("cuda")
    seed = rank_seed(args.workload, rank)
    x = S.make_inputs(wl, seed)
    n = wl.context
    nblk = n // wl.chunk

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
        return t.view(torch.bfloat16).to(dev)

    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    pos = torch.as_tensor(x["pos"], device=dev)
    layer = B.Layer(batch=wl.batch, heads_q=wl.heads_q, heads_kv=wl.heads_kv, head_dim=wl.head_dim,
                    chunk=wl.chunk, group=wl.group, sink_chunks=wl.sink, local_chunks=wl.local,
                    topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                    n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta, dtype=B.HGA_BF16,
                    out_dtype=B.HGA_BF16)
    bh = wl.batch * wl.heads_kv
    cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device=dev)
    gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device=dev)
    ci = torch.empty(bh, nblk, wl.topk_chunks, dtype=torch.int32, device=dev)
    gi = torch.empty(bh, nblk, wl.topk_groups, dtype=torch.int32, device=dev)
    out = torch.empty(wl.batch, wl.heads_q, n, wl.head_dim, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.batch, wl.heads_q, n, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    parts = {
        "summaries": lambda: B.hga_build_summaries(layer, k, n, 0, n, cs, gs),
        "route": lambda: B.hga_route(layer, q, n, pos, cs, gs, n, ci, gi),
        "attend": lambda: B.hga_attend(layer, q, n, pos, k, v, n, gi, out, lse),
    }

    def step():
        for fn in parts.values():
            fn()

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert B.hga_device_status() == 0
    graphs = {}
    for name, fn in list(parts.items()) + [("step", step)]:
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            fn()
        graphs[name] = g_
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def timed(g_, iters):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(iters)]
        for a_, b_ in ev:
            flush.zero_()
            a_.record(stream)
            g_.replay()
            b_.record(stream)
        torch.cuda.synchronize()
        return sum(a_.elapsed_time(b_) for a_, b_ in ev) / iters

    ranks = Ranks(world, dev)
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms_step = timed(graphs["step"], args.steps)
    ranks.barrier()
    ms_step = ranks.max(ms_step)
    ms = {name: timed(graphs[name], max(3, min(args.steps, 20))) for name in parts}
    assert B.hga_device_status() == 0

    # e2e: host q in (pinned), host output back, every step; k/v resident
    q_host = torch.from_numpy(np.ascontiguousarray(x["q"]).view(np.int16)).pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = []
    for i in range(1 + min(args.steps, 5)):
        flush.zero_()
        e0.record(stream)
        q.view(torch.int16).copy_(q_host, non_blocking=True)
        graphs["step"].replay()
        out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i:
            e2e.append(e0.elapsed_time(e1))
    ms_e2e = ranks.max(sum(e2e) / len(e2e))

    flops = prefill_flops(wl)
    peak, peak_kind = tensor_peak()
    achieved = flops / (ms["attend"] * 1e-3) / 1e12
    tokens = wl.batch * n  # per rank
    line = {
        "metric": METRIC + " (prefill)",
        "value": job_rate(tokens, world, ms_step),
        "unit": "prefill tokens/s (one attention layer)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "attn_us_per_layer": ms_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 q/k/v, fp32 accumulation (tcgen05)",
        "data": "synthetic (seeded N(0,1) q/k/v)",
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": n,
                   "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
                   "chunk": wl.chunk, "query_block": wl.chunk, "topk_chunks": wl.topk_chunks,
                   "topk_groups": wl.topk_groups,
                   "l2": "flushed (256 MB write) before every timed step",
                   "parallelism": f"replicas x{world}"},
        "per_kernel_us": {kk: vv * 1e3 for kk, vv in ms.items()},
        "attend_flops": flops,
        "roofline": {"kernel": "attend", "bound": "tensor", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": profile_traffic("attend_prefill_kernel", wl),
                     "algorithmic_flops": flops},
        "e2e": {"value": job_rate(tokens, world, ms_e2e), "unit": "prefill tokens/s (one attention layer)",
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": q_host.numel() * 2,
                "d2h_bytes_per_step": out_host.numel() * 2},
        "gpu_launches": 3 * args.steps,
        "timing": "CUDA graph of the step replayed per timed step; CUDA events on the launch stream",
        "clocks": clk.report(),
    }
    return line, wl, seed, x


def oracle_prefill_rate(wl: S.Workload, seed: int, budget_s: float, x=None):
    """Oracle prefill on a bounded sample of (KV head, query block) units: routing
    of the block and attention of its G*C query rows.  Returns prompt tokens/s."""
    from threadpoolctl import threadpool_limits

    from oracle import hga_oracle as O
    prm = O.HGAParams(head_dim=wl.head_dim, heads_q=wl.heads_q, heads_kv=wl.heads_kv,
                      chunk=wl.chunk, group=wl.group, sink=wl.sink, local=wl.local,
                      topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                      n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta)
    g, c = wl.gqa, wl.chunk
    nblk = wl.context // c
    rng = np.random.default_rng(0)
    units = [(h, int(j)) for h in range(wl.heads_kv) for j in rng.permutation(nblk)[:8]]
    times, spent = [], 0.0
    with threadpool_limits(limits=1):
        cache = {}
        for h, j in units:
            if spent >= budget_s:
                break
            if h not in cache:
                kb = x["k"][0, h] if x is not None else S.key_slice(wl, seed, 0, h)
                vb = x["v"][0, h] if x is not None else S.value_slice(wl, seed, 0, h)
                k64, v64 = S.widen(kb, wl.dtype), S.widen(vb, wl.dtype)
                cache = {h: (k64, v64, O.build_summaries(k64, prm))}
            k64, v64, (cs, gs) = cache[h]
            qb = (x["q"][0, h * g:(h + 1) * g, j * c:(j + 1) * c] if x is not None else
                  S.query_slice(wl, seed, 0)[h * g:(h + 1) * g, j * c:(j + 1) * c])
            q64 = S.widen(qb, wl.dtype)
            t0 = time.perf_counter()
            qbar = O.routing_query(q64)
            cidx, _, _ = O.route_chunks(qbar, cs, j, prm)
            gidx, _, _ = O.route_groups(qbar, gs, cidx, prm)
            for i in range(c):
                toks = O.visible_tokens(j * c + i, j, gidx, prm)
                for hh in range(g):
                    O.attend(q64[hh, i], k64, v64, toks)
            dt = time.perf_counter() - t0
            times.append(dt)
            spent += dt
    per_unit = sum(times) / len(times)
    step_s = per_unit * wl.heads_kv * nblk * wl.batch
    sample = (f"{len(times)} (KV head, 64-query block) units of the {wl.context}-token prefill "
              f"(routing + attention of every row), extrapolated ({sum(times):.1f} s of oracle time)")
    return wl.batch * wl.context / step_s, sample, 1


# ------------------------------------------------------------ oracle (CPU) arm

def oracle_decode_rate(wl: S.Workload, seed: int, budget_s: float, x=None):
    """Oracle decode step, timed per (sequence, KV head) unit on a bounded sample.

    Per unit: summaries of the rows the new token closes, level-1 and level-2
    routing, token set and exact attention of the G query heads.  The prefix
    summaries are built before timing (they are state, not step work).
    Returns (tokens/s for the whole batch, sample description, threads used).
    """
    from threadpoolctl import threadpool_limits

    from oracle import hga_oracle as O
    prm = O.HGAParams(head_dim=wl.head_dim, heads_q=wl.heads_q, heads_kv=wl.heads_kv,
                      chunk=wl.chunk, group=wl.group, sink=wl.sink, local=wl.local,
                      topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                      n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta)
    p = wl.context - 1
    cur = p // wl.chunk
    g = wl.gqa
    times = []
    spent = 0.0
    units = [(b, h) for b in range(wl.batch) for h in range(wl.heads_kv)]
    # A few (sequence, KV head) units, prepared once (their prefix summaries are
    # state, not step work), then timed in turn until the budget is spent.
    sample_units = units[:: max(1, len(units) // 4)][:4]
    prepared = []
    with threadpool_limits(limits=1):
        for b, h in sample_units:
            if x is not None:
                qb, kb, vb = x["q"][b, h * g:(h + 1) * g], x["k"][b, h], x["v"][b, h]
            else:
                q1 = S.query_slice(wl, seed, b, 1)
                qb = q1[h * g:(h + 1) * g]
                kb, vb = S.key_slice(wl, seed, b, h, q1), S.value_slice(wl, seed, b, h)
            q64, k64, v64 = S.widen(qb, wl.dtype), S.widen(kb, wl.dtype), S.widen(vb, wl.dtype)
            cs, gs = O.build_summaries(k64[:cur * wl.chunk], prm)
            cs = np.concatenate([cs, np.full((1, wl.head_dim), np.nan)])
            gs = np.concatenate([gs, np.full((1, gs.shape[1], wl.head_dim), np.nan)])
            prepared.append((q64, k64, v64, cs, gs))
        i = 0
        while spent < budget_s or not times:
            q64, k64, v64, cs0, gs0 = prepared[i % len(prepared)]
            cs, gs = cs0.copy(), gs0.copy()
            t0 = time.perf_counter()
            c0 = cur * wl.chunk
            cs[cur] = O.span_summary(k64[c0:c0 + wl.chunk], c0, prm.n_high_pairs, prm.rope_theta)
            g0 = p + 1 - wl.group
            gs[cur, -1] = O.span_summary(k64[g0:p + 1], g0, prm.n_high_pairs, prm.rope_theta)
            qbar = O.routing_query(q64[:, 0])
            cidx, _, _ = O.route_chunks(qbar, cs, cur, prm)
            gidx, _, _ = O.route_groups(qbar, gs, cidx, prm)
            toks = O.visible_tokens(p, cur, gidx, prm)
            for hh in range(g):
                O.attend(q64[hh, 0], k64, v64, toks)
            dt = time.perf_counter() - t0
            times.append(dt)
            spent += dt
            i += 1
    per_unit = sum(times) / len(times)
    step_s = per_unit * len(units)
    sample = (f"{len(times)} timed runs over {len(prepared)} of the {len(units)} (sequence, KV "
              f"head) units of a decode step at position {p}; mean per unit times the batch's "
              f"units ({sum(times):.1f} s of oracle time)")
    return wl.batch / step_s, sample, 1


def run_reference(args, rank: int):
    """The oracle arm: the float64 CPU oracle timed on the host cores, rank 0 only.

    Each step is a bounded sample of the same workload (sized so the whole
    run stays within a few minutes), extrapolated to the arm's unit.
    """
    if rank != 0:
        return None
    wl = S.workload(args.workload)
    if args.batch:
        wl = wl.with_(batch=args.batch)
    if args.context:
        wl = wl.with_(context=args.context)
    seed = rank_seed(args.workload, 0)
    rate_fn = oracle_prefill_rate if wl.prefill else oracle_decode_rate
    rates = []
    budget = max(0.02, min(args.cpu_seconds / 10, 150.0 / (args.warmup + args.steps)))
    for i in range(args.warmup + args.steps):
        r, sample, cores = rate_fn(wl, seed, budget_s=budget)
        if i >= args.warmup:
            rates.append(r)
    value = statistics.median(rates)
    kind = "prefill" if wl.prefill else "decode"
    unit = f"{kind} tokens/s (one attention layer)"
    tokens_per_step = wl.batch * (wl.context if wl.prefill else 1)
    return {"impl": "reference", "metric": METRIC + (" (prefill)" if wl.prefill else ""),
            "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": len(rates), "warmup": args.warmup,
            "ms_per_step": tokens_per_step / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same generator)",
            "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": wl.context},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        line = run_reference(args, rank)
        if line:
            print(json.dumps(line))
        return
    if world > 1:
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        rank, world = init_ranks("nccl")
    line, wl, seed, x = run_hga(args, rank, world)
    if rank == 0:
        if not args.no_cpu_baseline:
            rate = oracle_prefill_rate if wl.prefill else oracle_decode_rate
            val, sample, cores = rate(wl, seed, args.cpu_seconds, x)
            line["cpu_baseline"] = {"value": val, "unit": line["unit"], "cores": cores,
                                    "kind": "oracle", "sample": sample}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
