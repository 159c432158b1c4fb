"""Benchmark of the HGA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--batch B]
                    [--layers L] [--no-workloads]
    python bench.py --impl reference ...      # the float64 CPU oracle, timed on host cores

One step = one decode step of a stack of L attention layers for the whole batch:
in every layer, append the new token's summary rows, route chunks, route groups
and attend (steps 1-5 of the HGA hot path), on inputs already resident in HBM.
Every layer has its own K/V cache and summary tables, so no layer reads what
another one brought into L2; the layers run back to back in one CUDA graph, as
a model's decode step runs them, and the attention time per layer is the step
time over L.  L2 is flushed (a 256 MB write, then a 256 MB read so that no dirty
line is left to write back) before every timed step, outside the timed events.
Prints one JSON line; with one GPU and the default workload it also carries a
`workloads` key with the prefill, wide-head, host-tier and small-batch decode
workloads, each measured the same way.

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
    ap.add_argument("--dtype", default=None, choices=["bf16", "f32"],
                    help="override the K/V storage type (f32 runs the general attention kernels)")
    ap.add_argument("--layers", type=int, default=0,
                    help="attention layers per decode step (0: 4, or 1 for the host tier)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--sub", default=None,
                    help="run one of the additional workloads alone (its record is printed)")
    ap.add_argument("--warm-slots", type=int, default=0,
                    help="warm-tier group slots per (sequence, KV head) (0: 4 x topk_groups)")
    ap.add_argument("--cold-dir", default=None,
                    help="directory of the cold tier's history file (default: the system's "
                         "temporary directory)")
    ap.add_argument("--warm-steps", type=int, default=64,
                    help="consecutive decode steps of the warm-tier runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workloads' sub-records")
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

def step_bytes(wl: S.Workload, positions=None) -> dict:
    """Algorithmic HBM bytes of one decode step per kernel (whole batch).

    route_chunks: the candidate chunk-summary rows (fp32) + the G query rows;
    route_groups: the groups of the kc selected chunks + query rows + chunk ids;
    attend: K and V rows of the T routed tokens + query rows + output (fp32);
    summaries: the closing chunk's and group's key rows + the rows written.
    positions: each sequence's query position (default: the last row, context-1);
    "tokens" is T of the first sequence.
    """
    e = 2 if wl.dtype == "bf16" else 4
    d, g = wl.head_dim, wl.gqa
    ng = wl.chunk // wl.group
    qrow = g * d * e
    positions = [wl.context - 1] * wl.batch if positions is None else [int(x) for x in positions]
    tot = dict(summaries=0, route_chunks=0, route_groups=0, attend=0)
    first_t = None
    for p in positions:
        cur = p // wl.chunk
        n_cand = max(0, cur - wl.local - wl.sink)
        kc = min(wl.topk_chunks, n_cand)
        kg = min(wl.topk_groups, kc * ng)
        forced = (min(wl.sink, max(0, cur - wl.local)) * wl.chunk +
                  (p - max(0, cur - wl.local) * wl.chunk + 1))
        t = forced + kg * wl.group
        first_t = t if first_t is None else first_t
        summ = 0
        if (p + 1) % wl.chunk == 0:
            summ = wl.chunk * d * e + (d + ng * d) * 4
        elif (p + 1) % wl.group == 0:
            summ = wl.group * d * e + d * 4
        tot["summaries"] += wl.heads_kv * summ
        tot["route_chunks"] += wl.heads_kv * (n_cand * d * 4 + qrow)
        tot["route_groups"] += wl.heads_kv * (kc * ng * d * 4 + qrow + wl.topk_chunks * 4)
        tot["attend"] += wl.heads_kv * (t * d * e * 2 + qrow + g * d * 4 + wl.topk_groups * 4)
    tot["tokens"] = first_t
    return tot


def decode_step_bytes(wl: S.Workload, positions=None) -> int:
    """Bytes of the one-launch decode step: append + routing + attention, less the
    query rows the routing and the attention would each read again."""
    nb = step_bytes(wl, positions)
    e = 2 if wl.dtype == "bf16" else 4
    return (nb["summaries"] + nb["route_chunks"] + nb["route_groups"] + nb["attend"] -
            2 * wl.batch * wl.heads_kv * wl.gqa * wl.head_dim * e)


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


# ------------------------------------------------------------------ inputs

L2_NOTE = ("flushed before every timed step: a 256 MB write, then a 256 MB read "
           "(no dirty line left for the timed step to write back)")


class Flush:
    """Evicts L2 (126 MB) before a timed step: writes one buffer larger than L2,
    then reads another, so the timed step starts with a clean L2 holding none of
    its inputs."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def host_to_device(a, wl, dev):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16 if wl.dtype == "bf16" else np.float32))
    return (t.view(torch.bfloat16) if wl.dtype == "bf16" else t).to(dev)


def device_inputs(wl: S.Workload, seed: int, dev):
    """Inputs of the workload's shape drawn on the device (torch's generator): q, k,
    v ~ N(0,1) stored as bf16, with the workload's log-normal key norms.  Used
    for the large sub-workloads, whose host generation would take minutes; the
    work of a step does not depend on the values (the routing always keeps kc
    chunks and kg groups)."""
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    bf = torch.bfloat16
    q_len = wl.context if wl.prefill else 1
    q = torch.empty(wl.batch, wl.heads_q, q_len, wl.head_dim, dtype=bf, device=dev)
    k = torch.empty(wl.batch, wl.heads_kv, wl.context, wl.head_dim, dtype=bf, device=dev)
    v = torch.empty_like(k)
    for b in range(wl.batch):
        q[b] = torch.randn(q[b].shape, generator=gen, device=dev).to(bf)
        kb = torch.randn(k[b].shape, generator=gen, device=dev)
        if wl.lognormal_sigma:
            kb *= torch.exp(wl.lognormal_sigma *
                            torch.randn(wl.heads_kv, wl.context, 1, generator=gen, device=dev))
        k[b] = kb.to(bf)
        v[b] = torch.randn(v[b].shape, generator=gen, device=dev).to(bf)
    pos = torch.full((wl.batch,), wl.context - 1, dtype=torch.int64, device=dev)
    return q, k, v, pos


def make_layer(B, wl, out_dtype):
    return B.Layer(batch=wl.batch, heads_q=wl.heads_q, heads_kv=wl.heads_kv, head_dim=wl.head_dim,
                   chunk=wl.chunk, group=wl.group, sink_chunks=wl.sink, local_chunks=wl.local,
                   topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                   n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta,
                   dtype=B.HGA_BF16 if wl.dtype == "bf16" else B.HGA_F32, out_dtype=out_dtype)


def timed_graph(g, iters, flush, stream):
    """Mean ms of `iters` replays of graph g, each after an L2 flush (outside the events)."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for a_, b_ in ev:
        flush()
        a_.record(stream)
        g.replay()
        b_.record(stream)
    torch.cuda.synchronize()
    return sum(a_.elapsed_time(b_) for a_, b_ in ev) / iters


def decode_record(args, wl: S.Workload, layers: int, steps: int, warmup: int, world: int,
                  ranks, seed: int, x=None, compare: bool = True) -> dict:
    """One decode workload: the timed L-layer step, per-call times, the roofline of
    the dominant kernel, the end-to-end rate through host buffers and clocks."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = torch.device("cuda")
    n = wl.context
    p = n - 1
    hot = wl.name.startswith("host_tier")
    if x is not None:
        q0, k0, v0 = (host_to_device(x[t], wl, dev) for t in ("q", "k", "v"))
        pos = torch.as_tensor(x["pos"], device=dev)
        data = ("synthetic (seeded N(0,1) q/k/v from the host generator" +
                (f"; {wl.needles} needle chunks per KV head" if wl.needles else "") + ")")
    else:
        q0, k0, v0, pos = device_inputs(wl, seed, dev)
        data = ("synthetic (N(0,1) q/k/v drawn on the device" +
                (f"; log-normal key norms, sigma {wl.lognormal_sigma}" if wl.lognormal_sigma else "") + ")")
    layer = make_layer(B, wl, B.HGA_F32)
    bh = wl.batch * wl.heads_kv
    nc, ng = n // wl.chunk, wl.chunk // wl.group
    flush = Flush(dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    # every layer: its own caches, summaries, routing buffers and outputs; the layers'
    # queries (and the new K/V rows, see e2e) share one device input buffer and their
    # outputs one output buffer, so a step moves its inputs and results in one copy each
    kv_dtype = k0.dtype
    q_bytes = layers * q0.numel() * q0.element_size()
    kv_bytes = 0 if hot else layers * 2 * wl.batch * wl.heads_kv * wl.head_dim * k0.element_size()
    dev_in = torch.empty(q_bytes + kv_bytes, dtype=torch.uint8, device=dev)
    qs_all = dev_in[:q_bytes].view(q0.dtype).view((layers,) + tuple(q0.shape))
    kv_dev = None if hot else dev_in[q_bytes:].view(kv_dtype).view(
        layers, 2, wl.batch, wl.heads_kv, wl.head_dim)
    outs_all = torch.empty(layers, wl.batch, wl.heads_q, 1, wl.head_dim, device=dev)
    L_ = []
    for li in range(layers):
        k, v = (k0, v0) if li == 0 else (k0.clone(), v0.clone())
        qs_all[li].copy_(q0)
        d = dict(q=qs_all[li], k=k, v=v,
                 cs=torch.empty(bh, nc, wl.head_dim, device=dev),
                 gs=torch.empty(bh, nc, ng, wl.head_dim, device=dev),
                 ci=torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device=dev),
                 gi=torch.empty(bh, wl.topk_groups, dtype=torch.int32, device=dev),
                 out=outs_all[li],
                 lse=torch.empty(wl.batch, wl.heads_q, 1, device=dev))
        L_.append(d)
    del q0, k0, v0
    if hot:  # the whole K/V cache in pinned host memory; the GPU keeps summaries and windows
        layer.kv_loc = B.HGA_KV_HOST_PINNED
        d = L_[0]
        d["k_host"], d["v_host"] = d["k"].cpu().pin_memory(), d["v"].cpu().pin_memory()
        del d["k"], d["v"]
        torch.cuda.empty_cache()
        rows = B.hga_hot_rows(layer)
        d["k_work"] = torch.empty(bh, rows, wl.head_dim, dtype=torch.bfloat16, device=dev)
        d["v_work"] = torch.empty_like(d["k_work"])
    wsb = B.hga_workspace_size(layer, n, 1)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
    for d in L_:  # prefix summaries (setup, untimed): every row closed before the new token
        k_src = d["k_host"] if hot else d["k"]
        B.hga_build_summaries(layer, k_src, n, 0, p, d["cs"], d["gs"], stream=sh)
    if hot:
        d = L_[0]
        B.hga_route(layer, d["q"], 1, pos, d["cs"], d["gs"], n, d["ci"], d["gi"], stream=sh)
        B.hga_gather_host(layer, d["k_host"], d["v_host"], n, pos, d["gi"], d["k_work"],
                          d["v_work"], refresh_window=True, stream=sh)

    # the one-call decode step takes bf16, D = 128; other shapes (fp32 caches, D = 64)
    # run the append, routing and general attention calls
    try:
        fusable = not hot and B.hga_decode_step_launches(layer, n) >= 1
    except B.HGAError:
        fusable = False

    def parts_of(d):
        k_src, v_src = (d["k_host"], d["v_host"]) if hot else (d["k"], d["v"])
        k_att, v_att = (d["k_work"], d["v_work"]) if hot else (d["k"], d["v"])
        pr = {
            "summaries": lambda st: B.hga_build_summaries(layer, k_src, n, p, p + 1, d["cs"], d["gs"],
                                                          stream=st),
            "route": lambda st: B.hga_route(layer, d["q"], 1, pos, d["cs"], d["gs"], n, d["ci"],
                                            d["gi"], stream=st),
            "attend": lambda st: B.hga_attend(layer, d["q"], 1, pos, k_att, v_att, n, d["gi"],
                                              d["out"], d["lse"], ws, wsb, stream=st),
            "route_chunks": lambda st: B.hga_route_chunks(layer, d["q"], 1, pos, d["cs"], n, d["ci"],
                                                          stream=st),
            "route_groups": lambda st: B.hga_route_groups(layer, d["q"], 1, pos, d["gs"], n, d["ci"],
                                                          d["gi"], stream=st),
        }
        if hot:
            pr["gather"] = lambda st: B.hga_gather_host(layer, d["k_host"], d["v_host"], n, pos,
                                                        d["gi"], d["k_work"], d["v_work"], stream=st)
        elif fusable:
            # the whole step in one call: summary append, routing and attention
            pr["decode_step"] = lambda st: B.hga_decode_step(layer, d["q"], pos, d["cs"], d["gs"], n,
                                                             d["k"], d["v"], d["ci"], d["gi"],
                                                             d["out"], d["lse"], append=True,
                                                             stream=st)
        return pr

    parts_l = [parts_of(d) for d in L_]
    parts = parts_l[0]
    side = torch.cuda.Stream()

    def chain_step(pr, chain):
        """The append on a side stream beside a routing/attention chain (the rows the
        new token closes belong to the current chunk, which the step never routes)."""
        def step(st):
            main_s = torch.cuda.current_stream()
            side.wait_stream(main_s)
            with torch.cuda.stream(side):
                pr["summaries"](side.cuda_stream)
            for name in chain:
                pr[name](st)
            main_s.wait_stream(side)
        return step

    if hot:
        one_layer = chain_step(parts, ("route", "gather", "attend"))
        step = one_layer
        comparisons = {"four_call_step_us": chain_step(parts, ("route_chunks", "route_groups",
                                                                "gather", "attend"))}
    elif fusable:
        def step(st):
            for pr in parts_l:
                pr["decode_step"](st)
        comparisons = {"two_call_step_us": chain_step(parts, ("route", "attend")),
                       "four_call_step_us": chain_step(parts, ("route_chunks", "route_groups",
                                                               "attend"))} if compare else {}
    else:
        layer_steps = [chain_step(pr, ("route", "attend")) for pr in parts_l]

        def step(st):
            for ls in layer_steps:
                ls(st)
        comparisons = {}

    for _ in range(max(1, warmup)):
        step(sh)
    torch.cuda.synchronize()
    assert B.hga_device_status(sh) == 0
    graphs = {}
    for name, fn in [("step", step)] + list(comparisons.items()) + list(parts.items()):
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            fn(torch.cuda.current_stream().cuda_stream)
        graphs[name] = g_
    torch.cuda.synchronize()
    for _ in range(warmup):
        flush()
        graphs["step"].replay()
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms_step = timed_graph(graphs["step"], steps, flush, stream)
    ranks.barrier()
    ms_step = ranks.max(ms_step)
    assert B.hga_device_status(sh) == 0
    n_side = min(steps, 100)
    side_ms = {name: timed_graph(graphs[name], n_side, flush, stream) for name in comparisons}
    ms = {name: timed_graph(graphs[name], n_side, flush, stream) for name in parts}

    # roofline kernel: CUDA events around direct launches queued behind the flush
    # (the host enqueues them while the flush runs, so the events bracket GPU work)
    nb = step_bytes(wl)
    nb["route"] = nb["route_chunks"] + nb["route_groups"]
    nb["decode_step"] = decode_step_bytes(wl)
    one_launch = fusable and B.hga_decode_step_launches(layer, n) == 1
    if one_launch:
        kern = "decode_step"
    else:
        kern = max(("route", "attend"), key=lambda kk: ms[kk])
    kernel_name = {"decode_step": "decode_step_kernel", "route": "route_decode_kernel",
                   "attend": "attend_decode_bf16_kernel" if wl.dtype == "bf16" and
                   wl.head_dim == 128 else "attend_kernel + combine_kernel"}[kern]
    lay = layers if kern == "decode_step" else 1
    ds = [torch.cuda.Event(enable_timing=True) for _ in range(n_side)]
    de = [torch.cuda.Event(enable_timing=True) for _ in range(n_side)]
    for i in range(n_side):
        flush()
        ds[i].record(stream)
        for pr in parts_l[:lay]:
            pr[kern](sh)
        de[i].record(stream)
    torch.cuda.synchronize()
    kern_ms = ranks.max(sum(a_.elapsed_time(b_) for a_, b_ in zip(ds, de)) / n_side / lay)
    assert B.hga_device_status(sh) == 0
    hbm, peak_kind = peaks()
    achieved = nb[kern] / (kern_ms * 1e-3) / 1e9

    # e2e: every step, the new token's q and K/V rows of every layer come in from
    # pinned host memory (one copy into the shared input buffer; the K/V rows then
    # go to their cache rows on the device) and every layer's output goes back (one
    # copy of the shared output buffer)
    host_in = torch.empty(dev_in.shape, dtype=torch.uint8).pin_memory()
    host_in.copy_(dev_in)
    kv_new = None if hot else host_in[q_bytes:].view(kv_dtype).view(kv_dev.shape)
    kv_rows = torch.empty(layers, 2, wl.batch, wl.heads_kv, wl.head_dim, dtype=kv_dtype)
    for li, d in enumerate(L_):
        kv_rows[li, 0].copy_((d["k_host"] if hot else d["k"])[:, :, p].cpu())
        kv_rows[li, 1].copy_((d["v_host"] if hot else d["v"])[:, :, p].cpu())
    if not hot:
        kv_new.copy_(kv_rows)
    out_host = torch.empty(outs_all.shape, dtype=outs_all.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = []
    for i in range(warmup + min(steps, 100)):
        flush()
        e0.record(stream)
        dev_in.copy_(host_in, non_blocking=True)
        for li, d in enumerate(L_):
            if hot:  # the new token's K/V goes into the host cache, a host-side write
                d["k_host"][:, :, p].copy_(kv_rows[li, 0])
                d["v_host"][:, :, p].copy_(kv_rows[li, 1])
            else:
                d["k"][:, :, p].copy_(kv_dev[li, 0])
                d["v"][:, :, p].copy_(kv_dev[li, 1])
        graphs["step"].replay()
        out_host.copy_(outs_all, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= warmup:
            e2e.append(e0.elapsed_time(e1))
    ms_e2e = ranks.max(sum(e2e) / len(e2e))
    h2d = q_bytes + kv_bytes
    d2h = out_host.numel() * out_host.element_size()

    per_layer_ms = ms_step / layers
    total_bytes = nb["summaries"] + nb["route"] + nb["attend"]
    if one_launch:
        launches = layers
    else:  # append, route, (gather,) attend (+ the split-K combine with a workspace)
        launches = layers * (3 + (1 if wsb > 0 else 0) + (1 if hot else 0))
    unit = "decode tokens/s (one attention layer)"
    rec = {
        "value": job_rate(wl.batch, world, per_layer_ms),
        "unit": unit,
        "ms_per_step": ms_step,
        "attn_us_per_layer": per_layer_ms * 1e3,
        "layers_per_step": layers,
        "data": data,
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": n,
                   "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
                   "chunk": wl.chunk, "group": wl.group, "sink": wl.sink, "local": wl.local,
                   "topk_chunks": wl.topk_chunks, "topk_groups": wl.topk_groups,
                   "tokens_attended_per_kv_head": nb["tokens"], "layers_per_step": layers,
                   "l2": L2_NOTE, "parallelism": f"replicas x{world} (independent sequences per GPU)"},
        "per_kernel_us": {kk: ms[kk] * 1e3 for kk in parts},
        **{name: t * 1e3 for name, t in side_ms.items()},
        "step_hbm_bytes_per_layer": total_bytes,
        "step_hbm_gbs": total_bytes / (per_layer_ms * 1e-3) / 1e9,
        "roofline": {"kernel": kernel_name, "bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": profile_traffic(kernel_name, wl),
                     "algorithmic_bytes": nb[kern], "kernel_us": kern_ms * 1e3,
                     "duration": ("CUDA events on the launch stream around " +
                                  (f"{lay} back-to-back launches (one per layer), divided by {lay}"
                                   if lay > 1 else "one direct launch") +
                                  ", queued behind the L2 flush; per_kernel_us holds each call's "
                                  "one-layer CUDA graph replayed the same way")},
        "e2e": {"value": job_rate(wl.batch, world, ms_e2e / layers), "unit": unit,
                "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches * steps,
        "timing": (f"CUDA graph of the {layers}-layer step replayed per timed step; CUDA events on "
                   "the launch stream; attention time per layer = step time / layers"),
        "clocks": clk.report(),
    }
    if hot:
        rec["host_link"] = host_link_report(wl, ms, dev)
        rec["warm_tier"] = warm_tier_report(args, wl, layer, L_[0], flush, stream)
    del L_, graphs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def ragged_positions(wl: S.Workload, seed: int) -> np.ndarray:
    """A serving batch's mix of context lengths: each sequence's position drawn
    log-uniform in [2048, context), seeded."""
    rng = np.random.default_rng([seed, 77])
    return np.exp(rng.uniform(np.log(2048), np.log(wl.context), wl.batch)).astype(np.int64)


def make_pool(k, v, pos: np.ndarray, page: int, seed: int):
    """Scatter each sequence's pages up to its position into a shuffled page pool
    (the layout a serving engine's allocator leaves): pools [n_pages, Hkv, page,
    D] and the block table [B, context/page], -1 past each sequence's last page."""
    import torch
    b_, h, n, d = k.shape
    mp = n // page
    need = pos // page + 1
    total = int(need.sum())
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(seed))
    bt = torch.full((b_, mp), -1, dtype=torch.int32)
    kp = torch.empty(total, h, page, d, dtype=k.dtype, device=k.device)
    vp = torch.empty_like(kp)
    kb, vb = k.view(b_, h, mp, page, d), v.view(b_, h, mp, page, d)
    at = 0
    for b in range(b_):
        m = int(need[b])
        ids = perm[at:at + m]
        at += m
        bt[b, :m] = ids.to(torch.int32)
        dst = ids.to(k.device)
        kp[dst] = kb[b, :, :m].permute(1, 0, 2, 3)
        vp[dst] = vb[b, :, :m].permute(1, 0, 2, 3)
    return kp, vp, bt.to(k.device), total


def paged_record(args, wl: S.Workload, layers: int, steps: int, warmup: int, world: int, ranks,
                 seed: int, pages=(16, 64, 256)) -> dict:
    """A ragged serving batch over paged K/V: every sequence at its own position
    (ragged_positions), the pages of every layer scattered through a shuffled
    pool, the one-launch paged decode step of `layers` layers back to back (each
    its own pool and tables) against the dense one-launch step on the same rows
    and positions.  Same timing method as the decode records; the headline is
    the first page size, the others are reported beside it; outputs of every
    arm checked bit for bit against the dense step."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = torch.device("cuda")
    n = wl.context
    pos_np = ragged_positions(wl, seed)
    pos = torch.as_tensor(pos_np, device=dev)
    layer = make_layer(B, wl, B.HGA_F32)
    bh = wl.batch * wl.heads_kv
    nc, ng = n // wl.chunk, wl.chunk // wl.group
    flush = Flush(dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    def tables():
        return dict(cs=torch.zeros(bh, nc, wl.head_dim, device=dev),
                    gs=torch.zeros(bh, nc, ng, wl.head_dim, device=dev),
                    ci=torch.empty(bh, wl.topk_chunks, dtype=torch.int32, device=dev),
                    gi=torch.empty(bh, wl.topk_groups, dtype=torch.int32, device=dev),
                    out=torch.empty(wl.batch, wl.heads_q, 1, wl.head_dim, device=dev),
                    lse=torch.empty(wl.batch, wl.heads_q, 1, device=dev))

    L_ = []
    for li in range(layers):
        q, k, v, _ = device_inputs(wl, seed + li, dev)
        d = dict(q=q, k=k, v=v, dense=tables())
        B.hga_build_summaries(layer, k, n, 0, n, d["dense"]["cs"], d["dense"]["gs"], stream=sh)
        L_.append(d)

    def run(d, page, st):
        t = d[page]
        if page == "dense":
            B.hga_decode_step(layer, d["q"], pos, t["cs"], t["gs"], n, d["k"], d["v"], t["ci"],
                              t["gi"], t["out"], t["lse"], append=True, stream=st)
        else:
            B.hga_decode_step_paged(layer, d["q"], pos, t["cs"], t["gs"], t["kp"], t["vp"],
                                    t["kv"], t["ci"], t["gi"], t["out"], t["lse"], append=True,
                                    stream=st)

    def graph_of(page):
        for _ in range(max(1, warmup)):
            for d in L_:
                run(d, page, sh)
        torch.cuda.synchronize()
        g_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_):
            cs_ = torch.cuda.current_stream().cuda_stream
            for d in L_:
                run(d, page, cs_)
        torch.cuda.synchronize()
        assert B.hga_device_status(sh) == 0
        return g_

    g_dense = graph_of("dense")
    ms_dense = timed_graph(g_dense, steps, flush, stream)
    del g_dense
    hbm, peak_kind = peaks()
    arms = {}
    for i, page in enumerate(pages):
        for li, d in enumerate(L_):
            kp, vp, bt, n_pages = make_pool(d["k"], d["v"], pos_np, page, seed + li)
            t = dict(tables(), kp=kp, vp=vp, bt=bt, kv=B.kv_pages(bt, n_pages, page, n // page))
            B.hga_build_summaries_paged(layer, kp, t["kv"], pos, t["cs"], t["gs"], stream=sh)
            d[page] = t
        g_ = graph_of(page)
        for d in L_:   # same routing and the same output bits as the dense step
            assert torch.equal(d["dense"]["gi"], d[page]["gi"])
            assert torch.equal(d["dense"]["out"].view(torch.int32), d[page]["out"].view(torch.int32))
        for _ in range(warmup):
            flush()
            g_.replay()
        ranks.barrier()
        torch.cuda.synchronize()
        if i == 0:
            with ClockSampler(torch.cuda.current_device()) as clk:
                ms = timed_graph(g_, steps, flush, stream)
        else:
            ms = timed_graph(g_, steps, flush, stream)
        ranks.barrier()
        ms = ranks.max(ms)
        # roofline: events around the layers' direct launches, queued behind the flush
        n_side = min(steps, 100)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_side)]
        for a_, b_ in ev:
            flush()
            a_.record(stream)
            for d in L_:
                run(d, page, sh)
            b_.record(stream)
        torch.cuda.synchronize()
        assert B.hga_device_status(sh) == 0
        kern_ms = ranks.max(sum(a_.elapsed_time(b_) for a_, b_ in ev) / n_side / layers)
        nbytes = decode_step_bytes(wl, pos_np) + bh * (n // page) * 4   # + the block-table rows
        arms[page] = dict(ms=ms, kern_ms=kern_ms, nbytes=nbytes)
        del g_
        for d in L_:
            del d[page]
        torch.cuda.empty_cache()

    head = arms[pages[0]]
    achieved = head["nbytes"] / (head["kern_ms"] * 1e-3) / 1e9
    per_layer = head["ms"] / layers
    unit = "decode tokens/s (one attention layer)"
    rec = {
        "value": job_rate(wl.batch, world, per_layer), "unit": unit, "ms_per_step": head["ms"],
        "attn_us_per_layer": per_layer * 1e3, "dense_us_per_layer": ms_dense / layers * 1e3,
        "page_sizes_us_per_layer": {str(pg): a["ms"] / layers * 1e3 for pg, a in arms.items()},
        "layers_per_step": layers,
        "data": "synthetic (N(0,1) q/k/v drawn on the device; pages shuffled through the pool)",
        "config": {"workload": "paged_ragged_decode", "batch_per_gpu": wl.batch,
                   "capacity": n, "page_size": pages[0], "positions": {
                       "min": int(pos_np.min()), "median": int(np.median(pos_np)),
                       "max": int(pos_np.max()), "recipe": "log-uniform in [2048, capacity)"},
                   "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
                   "topk_chunks": wl.topk_chunks, "topk_groups": wl.topk_groups,
                   "l2": L2_NOTE},
        "roofline": {"kernel": "decode_step_kernel (paged)", "bound": "hbm", "achieved": achieved,
                     "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": None, "algorithmic_bytes": head["nbytes"],
                     "kernel_us": head["kern_ms"] * 1e3},
        "gpu_launches": layers * steps,
        "parity": "every arm's routed ids and outputs equal the dense step's bit for bit (checked here)",
        "clocks": clk.report(),
    }
    del L_
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def training_record(args, wl: S.Workload, steps: int, warmup: int, world: int, ranks,
                    seed: int) -> dict:
    """One training step of one attention layer at the prefill shape: the forward
    (summaries, routing of every 64-query block, attention) and the backward over
    the forward's index sets (hga_attend_backward: dQ, dK, dV) for a synthetic
    upstream gradient.  Same timing method as the prefill record."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = torch.device("cuda")
    n = wl.context
    nblk = n // wl.chunk
    q, k, v, pos = device_inputs(wl, seed, dev)
    layer = make_layer(B, wl, B.HGA_BF16)
    bh = wl.batch * wl.heads_kv
    cs = torch.empty(bh, n // wl.chunk, wl.head_dim, device=dev)
    gs = torch.empty(bh, n // wl.chunk, wl.chunk // wl.group, wl.head_dim, device=dev)
    ci = torch.empty(bh, nblk, wl.topk_chunks, dtype=torch.int32, device=dev)
    gi = torch.empty(bh, nblk, wl.topk_groups, dtype=torch.int32, device=dev)
    out = torch.empty(wl.batch, wl.heads_q, n, wl.head_dim, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.batch, wl.heads_q, n, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 1)
    dout = torch.randn(out.shape, generator=gen, device=dev).to(torch.bfloat16)
    dq = torch.empty(out.shape, device=dev)
    dk = torch.empty(k.shape, device=dev)
    dv = torch.empty(v.shape, device=dev)
    bwb = B.hga_attend_backward_workspace_size(layer, n, n)
    bws = torch.empty(bwb, dtype=torch.uint8, device=dev)
    flush = Flush(dev)
    parts = {
        "forward": lambda: (B.hga_build_summaries(layer, k, n, 0, n, cs, gs),
                            B.hga_route(layer, q, n, pos, cs, gs, n, ci, gi),
                            B.hga_attend(layer, q, n, pos, k, v, n, gi, out, lse)),
        "backward": lambda: B.hga_attend_backward(layer, q, n, pos, k, v, n, gi, out, lse, dout,
                                                  dq, dk, dv, bws, bwb),
    }

    def step():
        for fn in parts.values():
            fn()

    for _ in range(max(1, warmup)):
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
    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms_step = timed_graph(graphs["step"], steps, flush, stream)
    ranks.barrier()
    ms_step = ranks.max(ms_step)
    ms = {name: timed_graph(graphs[name], max(3, min(steps, 20)), flush, stream) for name in parts}
    assert B.hga_device_status() == 0
    assert bool(torch.isfinite(dq).all()) and bool(torch.isfinite(dk).all())
    # algorithmic flops per visible (query row, key) pair: forward 4D (S, PV);
    # backward 14D (dQ pass: S, dP, dS K; dK/dV pass: S, dP, P^T dO, dS^T Q)
    fwd_flops = prefill_flops(wl)
    bwd_flops = fwd_flops * 14 / 4
    peak, peak_kind = tensor_peak()
    achieved = bwd_flops / (ms["backward"] * 1e-3) / 1e12
    tokens = wl.batch * n
    rec = {
        "value": job_rate(tokens, world, ms_step),
        "unit": "training tokens/s (one attention layer, forward + backward)",
        "ms_per_step": ms_step, "forward_ms": ms["forward"], "backward_ms": ms["backward"],
        "layers_per_step": 1,
        "dtype": "bf16 q/k/v/dO, fp32 accumulation and gradients",
        "data": "synthetic (N(0,1) q/k/v and upstream gradient drawn on the device)",
        "config": {"workload": wl.name + " (training step)", "batch_per_gpu": wl.batch,
                   "context": n, "heads_q": wl.heads_q, "heads_kv": wl.heads_kv,
                   "head_dim": wl.head_dim, "chunk": wl.chunk, "topk_chunks": wl.topk_chunks,
                   "topk_groups": wl.topk_groups, "l2": L2_NOTE},
        "roofline": {"kernel": "hga_attend_backward (dq_kernel + dkdv_kernel + helpers)",
                     "bound": "tensor", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None, "algorithmic_flops": bwd_flops,
                     "kernel_us": ms["backward"] * 1e3,
                     "note": "mma.sync m16n8k16 kernels; timed as the whole backward call"},
        "gpu_launches": steps * (3 + 5),
        "clocks": clk.report(),
    }
    del q, k, v, dq, dk, dv, bws, graphs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


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


def warm_tier_report(args, wl: S.Workload, layer, d: dict, flush, stream) -> dict:
    """The warm tier in front of the host tier, against the cold host tier.

    T consecutive decode steps at positions n-T .. n-1 (every sequence), each
    with its own query: q_t = rho q_{t-1} + sqrt(1 - rho^2) z_t drawn on the
    device (a stationary AR(1) walk from the workload's query, stored bf16), so
    that consecutive steps route to overlapping groups.  Each arm runs one
    untimed step at n-T-1 that fills the windows (and, warm, the table after a
    reset), then the T steps: the summary append, routing, the gather (warm:
    hga_gather_warm, cold: hga_gather_host; both copy only the newest window
    row, the previous step having been at the position before) and the
    attention (warm: hga_attend_warm), all on the launch stream.  CUDA events around every step
    and around its gather, L2 flushed before each step."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = d["q"].device
    sh = stream.cuda_stream
    n, T = wl.context, args.warm_steps
    M = args.warm_slots or 4 * wl.topk_groups
    bh = wl.batch * wl.heads_kv
    group_bytes = wl.group * wl.head_dim * 2 * 2      # K and V rows of one group, bf16
    rows = B.hga_warm_rows(layer, M)
    kw = torch.empty(bh, rows, wl.head_dim, dtype=torch.bfloat16, device=dev)
    vw = torch.empty_like(kw)
    tags = torch.empty(bh, M, dtype=torch.int32, device=dev)
    stamps = torch.empty_like(tags)
    smap = torch.empty(bh, wl.topk_groups, dtype=torch.int32, device=dev)
    counters = torch.zeros(2, dtype=torch.int64, device=dev)
    pos_all = torch.arange(n - T - 1, n, device=dev).repeat_interleave(wl.batch).view(T + 1, wl.batch)

    def queries(rho):
        gen = torch.Generator(device=dev)
        gen.manual_seed(int(rho * 1000))
        cur = d["q"].float()
        out = [cur.to(torch.bfloat16)]
        c = (1.0 - rho * rho) ** 0.5
        for _ in range(T):
            cur = rho * cur + c * torch.randn(cur.shape, generator=gen, device=dev)
            out.append(cur.to(torch.bfloat16))
        return out

    def run(qs, warm):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(T)]
        if warm:
            B.hga_warm_reset(layer, M, tags, stamps, stream=sh)
        for t in range(T + 1):
            pos = pos_all[t]
            p = n - T - 1 + t
            if t:
                flush()
                ev[t - 1][0].record(stream)
            B.hga_build_summaries(layer, d["k_host"], n, p, p + 1, d["cs"], d["gs"], stream=sh)
            B.hga_route(layer, qs[t], 1, pos, d["cs"], d["gs"], n, d["ci"], d["gi"], stream=sh)
            if t:
                ev[t - 1][1].record(stream)
            if warm:
                B.hga_gather_warm(layer, d["k_host"], d["v_host"], n, pos, d["gi"], M, tags,
                                  stamps, smap, kw, vw, refresh_window=1 if t == 0 else 2,
                                  counters=counters if t else None, stream=sh)
            else:
                B.hga_gather_host(layer, d["k_host"], d["v_host"], n, pos, d["gi"], d["k_work"],
                                  d["v_work"], refresh_window=1 if t == 0 else 2, stream=sh)
            if t:
                ev[t - 1][2].record(stream)
            if warm:
                B.hga_attend_warm(layer, qs[t], pos, kw, vw, n, d["gi"], smap, M, d["out"],
                                  d["lse"], stream=sh)
            else:
                B.hga_attend(layer, qs[t], 1, pos, d["k_work"], d["v_work"], n, d["gi"],
                             d["out"], d["lse"], stream=sh)
            if t:
                ev[t - 1][3].record(stream)
        torch.cuda.synchronize()
        assert B.hga_device_status(sh) == 0
        step = sum(e[0].elapsed_time(e[3]) for e in ev) / T
        gather = sum(e[1].elapsed_time(e[2]) for e in ev) / T
        return step * 1e3, gather * 1e3

    runs = []
    for rho in (0.9, 0.95, 0.99):
        qs = queries(rho)
        counters.zero_()
        w_step, w_gather = run(qs, True)
        hits, misses = (int(v) for v in counters.cpu())
        c_step, c_gather = run(qs, False)
        runs.append({"rho": rho, "hit_rate": hits / max(1, hits + misses),
                     "routed_host_bytes_per_step": {"warm": misses * group_bytes / T,
                                                    "cold": (hits + misses) * group_bytes / T},
                     "step_us": {"warm": w_step, "cold": c_step},
                     "gather_us": {"warm": w_gather, "cold": c_gather}})
    # the cold tier: the same steps with the history in a file, read per step by
    # host threads (plan on the GPU, stage on the host, fill on the GPU)
    qs = queries(0.95)
    cold = {}
    try:
        cold = cold_tier_run(args, B, wl, layer, d, qs, pos_all, M, tags, stamps, smap, kw, vw,
                             counters, group_bytes, sh)
    except (B.HGAError, OSError) as e:   # e.g. no room for the history file
        cold = {"unavailable": str(e)}
    return {"slots_per_kv_head": M, "steps": T, "cold_tier": cold,
            "hbm_bytes": 2 * bh * rows * wl.head_dim * 2 + 2 * tags.numel() * 4,
            "timing": ("CUDA events around each of T direct-launch steps (summary append, route, "
                       "gather, attention) on the launch stream, L2 flushed before each; one "
                       "untimed step fills the windows first"),
            "runs": runs}


def cold_tier_run(args, B, wl, layer, d, qs, pos_all, M, tags, stamps, smap, kw, vw, counters,
                  group_bytes, sh) -> dict:
    """The warm-tier steps with the history in a file (the cold tier): plan on the
    GPU, stage the misses and the newest window row from the file with host
    threads, fill and attend on the GPU."""
    import tempfile
    import torch
    n, T = wl.context, args.warm_steps
    bh = wl.batch * wl.heads_kv
    dev = d["q"].device
    rho = 0.95
    plan = torch.empty(bh, wl.topk_groups, 2, dtype=torch.int32, device=dev)
    n_plan = torch.empty(bh, dtype=torch.int32, device=dev)
    plan_h = torch.empty(plan.shape, dtype=torch.int32).pin_memory()
    n_plan_h = torch.empty(n_plan.shape, dtype=torch.int32).pin_memory()
    staging = torch.zeros(B.hga_cold_stage_bytes(layer), dtype=torch.uint8).pin_memory()
    with tempfile.TemporaryDirectory(dir=args.cold_dir) as tmp:
        with B.ColdStore(os.path.join(tmp, "kv.bin"), layer, n, create=True) as store:
            store.write(d["k_host"], d["v_host"], 0, n, threads=16)
            B.hga_warm_reset(layer, M, tags, stamps, stream=sh)
            counters.zero_()
            step_ms, stage_ms, groups = [], [], 0
            for t in range(T + 1):
                pos = pos_all[t]
                p = n - T - 1 + t
                mode = 1 if t == 0 else 2
                torch.cuda.synchronize()
                t0 = time.perf_counter()
                B.hga_build_summaries(layer, d["k_host"], n, p, p + 1, d["cs"], d["gs"], stream=sh)
                B.hga_route(layer, qs[t], 1, pos, d["cs"], d["gs"], n, d["ci"], d["gi"], stream=sh)
                B.hga_warm_plan(layer, n, pos, d["gi"], M, tags, stamps, smap, plan, n_plan,
                                counters=counters, stream=sh)
                plan_h.copy_(plan, non_blocking=True)
                n_plan_h.copy_(n_plan, non_blocking=True)
                torch.cuda.synchronize()
                s0 = time.perf_counter()
                store.stage(layer, np.full(wl.batch, p, dtype=np.int64), plan_h.numpy(),
                            n_plan_h.numpy(), mode, staging, threads=16)
                s1 = time.perf_counter()
                B.hga_warm_fill(layer, n, pos, staging, plan, n_plan, M, mode, kw, vw, stream=sh)
                B.hga_attend_warm(layer, qs[t], pos, kw, vw, n, d["gi"], smap, M, d["out"],
                                  d["lse"], stream=sh)
                torch.cuda.synchronize()
                t1 = time.perf_counter()
                if t:
                    step_ms.append((t1 - t0) * 1e3)
                    stage_ms.append((s1 - s0) * 1e3)
                    groups += int(n_plan_h.sum())
            assert B.hga_device_status(sh) == 0
            hits, misses = (int(v) for v in counters.cpu())
            read = groups * group_bytes + T * bh * d["k_host"].shape[-1] * 2 * 2
            return {"rho": rho, "hit_rate": hits / max(1, hits + misses),
                    "file_bytes_read_per_step": read / T,
                    "step_ms": sum(step_ms) / T, "stage_ms": sum(stage_ms) / T,
                    "stage_gbs": read / (sum(stage_ms) * 1e-3) / 1e9,
                    "timing": ("host wall clock around each step (the plan's device-to-host "
                               "copy and the file reads make the step synchronous), 16 host "
                               "threads; the file was just written, so the page cache may "
                               "serve the reads")}


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


def prefill_record(args, wl: S.Workload, steps: int, warmup: int, world: int, ranks,
                   seed: int, x=None) -> dict:
    """One prefill step of one layer: summaries of the whole prompt, routing of
    every 64-query block, attention of every query (steps 1-5)."""
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B

    dev = torch.device("cuda")
    n = wl.context
    nblk = n // wl.chunk
    if x is not None:
        q, k, v = (host_to_device(x[t], wl, dev) for t in ("q", "k", "v"))
        pos = torch.as_tensor(x["pos"], device=dev)
    else:
        q, k, v, pos = device_inputs(wl, seed, dev)
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
    flush = Flush(dev)
    parts = {
        "summaries": lambda: B.hga_build_summaries(layer, k, n, 0, n, cs, gs),
        "route": lambda: B.hga_route(layer, q, n, pos, cs, gs, n, ci, gi),
        "attend": lambda: B.hga_attend(layer, q, n, pos, k, v, n, gi, out, lse),
    }

    def step():
        for fn in parts.values():
            fn()

    for _ in range(max(1, warmup)):
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
        return timed_graph(g_, iters, flush, stream)

    ranks.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms_step = timed(graphs["step"], steps)
    ranks.barrier()
    ms_step = ranks.max(ms_step)
    ms = {name: timed(graphs[name], max(3, min(steps, 20))) for name in parts}
    assert B.hga_device_status() == 0

    # e2e: host q in (pinned), host output back, every step; k/v resident
    q_host = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    q_host.copy_(q)
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e = []
    for i in range(1 + min(steps, 5)):
        flush()
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
    rec = {
        "value": job_rate(tokens, world, ms_step),
        "unit": "prefill tokens/s (one attention layer)",
        "ms_per_step": ms_step, "attn_us_per_layer": ms_step * 1e3, "layers_per_step": 1,
        "dtype": "bf16 q/k/v, fp32 accumulation (tcgen05)",
        "data": ("synthetic (seeded N(0,1) q/k/v from the host generator)" if x is not None else
                 "synthetic (N(0,1) q/k/v drawn on the device)"),
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": n,
                   "heads_q": wl.heads_q, "heads_kv": wl.heads_kv, "head_dim": wl.head_dim,
                   "chunk": wl.chunk, "query_block": wl.chunk, "topk_chunks": wl.topk_chunks,
                   "topk_groups": wl.topk_groups,
                   "l2": L2_NOTE,
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
        "gpu_launches": 3 * steps,
        "timing": "CUDA graph of the step replayed per timed step; CUDA events on the launch stream",
        "clocks": clk.report(),
    }
    del q, k, v, out, graphs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


# ------------------------------------------------------------ oracle (CPU) arm

def _oracle_worker(task):
    """One oracle process: prepares its units from the seeded host generator (the
    prefix summaries are state, not step work, so they are built untimed), then
    times the oracle's work on them in turn, `rounds` times for `budget` seconds.
    Decode unit (b, h): the summary rows the new token closes, level-1 and
    level-2 routing, the token set and exact attention of the G query heads.
    Prefill unit (h, j): routing of query block j and attention of its G*C rows.
    Returns [(runs, seconds)] per round."""
    from threadpoolctl import threadpool_limits

    from oracle import hga_oracle as O
    kind, wl, seed, units, budget, rounds = task
    prm = O.HGAParams(head_dim=wl.head_dim, heads_q=wl.heads_q, heads_kv=wl.heads_kv,
                      chunk=wl.chunk, group=wl.group, sink=wl.sink, local=wl.local,
                      topk_chunks=wl.topk_chunks, topk_groups=wl.topk_groups,
                      n_high_pairs=wl.n_high_pairs, rope_theta=wl.rope_theta)
    g, c = wl.gqa, wl.chunk
    out = []
    with threadpool_limits(limits=1):
        prepared = []
        for u in units:
            if kind == "decode":
                b, h = u
                q1 = S.query_slice(wl, seed, b, 1)
                kb, vb = S.key_slice(wl, seed, b, h, q1), S.value_slice(wl, seed, b, h)
                q64 = S.widen(q1[h * g:(h + 1) * g], wl.dtype)
                k64, v64 = S.widen(kb, wl.dtype), S.widen(vb, wl.dtype)
                cur = (wl.context - 1) // c
                cs, gs = O.build_summaries(k64[:cur * c], prm)
                cs = np.concatenate([cs, np.full((1, wl.head_dim), np.nan)])
                gs = np.concatenate([gs, np.full((1, gs.shape[1], wl.head_dim), np.nan)])
                prepared.append((q64, k64, v64, cs, gs))
            else:
                h, j = u
                k64 = S.widen(S.key_slice(wl, seed, 0, h), wl.dtype)
                v64 = S.widen(S.value_slice(wl, seed, 0, h), wl.dtype)
                # the block's queries: N(0,1) rows of the stored type (the whole
                # prompt's query tensor is not drawn for one block)
                rng = np.random.default_rng([seed, 99, h, j])
                q64 = S.widen(S.store(rng.standard_normal((g, c, wl.head_dim), dtype=np.float32),
                                      wl.dtype), wl.dtype)
                prepared.append((q64, k64, v64, O.build_summaries(k64, prm), j))
        for _ in range(rounds):
            runs, spent, i = 0, 0.0, 0
            while spent < budget or runs == 0:
                t0 = time.perf_counter()
                if kind == "decode":
                    q64, k64, v64, cs0, gs0 = prepared[i % len(prepared)]
                    p = wl.context - 1
                    cur = p // c
                    cs, gs = cs0.copy(), gs0.copy()
                    c0 = cur * c
                    if (p + 1) % c == 0:
                        cs[cur] = O.span_summary(k64[c0:c0 + c], c0, prm.n_high_pairs, prm.rope_theta)
                    if (p + 1) % wl.group == 0:
                        g0 = p + 1 - wl.group
                        gs[cur, (p % c) // wl.group] = O.span_summary(k64[g0:p + 1], g0,
                                                                      prm.n_high_pairs, prm.rope_theta)
                    qbar = O.routing_query(q64[:, 0])
                    cidx, _, _ = O.route_chunks(qbar, cs, cur, prm)
                    gidx, _, _ = O.route_groups(qbar, gs, cidx, prm)
                    toks = O.visible_tokens(p, cur, gidx, prm)
                    for hh in range(g):
                        O.attend(q64[hh, 0], k64, v64, toks)
                else:
                    q64, k64, v64, (cs, gs), j = prepared[i % len(prepared)]
                    qbar = O.routing_query(q64)
                    cidx, _, _ = O.route_chunks(qbar, cs, j, prm)
                    gidx, _, _ = O.route_groups(qbar, gs, cidx, prm)
                    for r in range(c):
                        toks = O.visible_tokens(j * c + r, j, gidx, prm)
                        for hh in range(g):
                            O.attend(q64[hh, r], k64, v64, toks)
                spent += time.perf_counter() - t0
                runs += 1
                i += 1
            out.append((runs, spent))
    return out


def oracle_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rates(wl: S.Workload, seed: int, budget: float, rounds: int = 1, max_procs: int = 64):
    """The oracle on the host's cores: one single-threaded process per core (spawned),
    each timing a few of the workload's independent units.  Returns (per-round
    tokens/s, sample description, processes)."""
    import multiprocessing as mp
    kind = "prefill" if wl.prefill else "decode"
    nblk = wl.context // wl.chunk
    if kind == "decode":
        all_units = [(b, h) for b in range(wl.batch) for h in range(wl.heads_kv)]
        units_per_step, tokens_per_step = len(all_units), wl.batch
    else:
        rng = np.random.default_rng(0)
        all_units = [(h, int(j)) for h in range(wl.heads_kv) for j in rng.permutation(nblk)[:8]]
        units_per_step, tokens_per_step = wl.heads_kv * nblk * wl.batch, wl.batch * wl.context
    # memory per process grows with the context: fewer processes for long ones
    procs = max(1, min(oracle_cores(), max_procs, 16 if wl.context > 65536 else max_procs,
                       len(all_units)))
    per = [all_units[i::procs][:2] for i in range(procs)]
    tasks = [(kind, wl, seed, u, budget, rounds) for u in per]
    with mp.get_context("spawn").Pool(procs) as pool:
        res = pool.map(_oracle_worker, tasks)
    rates = []
    for r in range(rounds):
        units_per_s = sum(w[r][0] / w[r][1] for w in res)
        rates.append(units_per_s / units_per_step * tokens_per_step)
    n_runs = sum(w[r][0] for w in res for r in range(rounds))
    what = ("(sequence, KV head) units of a decode step at position "
            f"{wl.context - 1}" if kind == "decode" else
            f"(KV head, 64-query block) units of the {wl.context}-token prefill")
    sample = (f"{procs} single-threaded processes, {n_runs} timed runs over "
              f"{sum(len(u) for u in per)} {what}, each process timing its units for "
              f"{budget:.1f} s per round; throughput summed over the processes and scaled "
              f"to the step's {units_per_step} units")
    return rates, sample, procs


def cpu_baseline(wl, seed, budget, unit):
    rates, sample, procs = oracle_rates(wl, seed, budget)
    return {"value": rates[0], "unit": unit, "cores": procs, "kind": "oracle", "sample": sample}


def workload_of(args) -> S.Workload:
    wl = S.workload(args.workload)
    if args.batch:
        wl = wl.with_(batch=args.batch)
    if args.context:
        wl = wl.with_(context=args.context)
    if args.dtype:
        wl = wl.with_(dtype=args.dtype)
    return wl


def run_reference(args, rank: int):
    """The oracle arm: the float64 CPU oracle timed on the host cores, rank 0 only.

    Each step is a bounded sample of the same workload (sized so the whole run
    stays within a few minutes), extrapolated to the arm's unit.
    """
    if rank != 0:
        return None
    wl = workload_of(args)
    seed = rank_seed(args.workload, 0)
    rounds = args.warmup + args.steps
    budget = max(0.05, min(args.cpu_seconds / 4, 120.0 / rounds))
    rates, sample, procs = oracle_rates(wl, seed, budget, rounds=rounds)
    timed = rates[args.warmup:] or rates
    value = statistics.median(timed)
    kind = "prefill" if wl.prefill else "decode"
    unit = f"{kind} tokens/s (one attention layer)"
    tokens_per_step = wl.batch * (wl.context if wl.prefill else 1)
    return {"impl": "reference", "metric": METRIC + (" (prefill)" if wl.prefill else ""),
            "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": len(timed), "warmup": args.warmup,
            "ms_per_step": tokens_per_step / value * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, same generator)",
            "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "context": wl.context},
            "cpu_baseline": {"value": value, "unit": unit, "cores": procs, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# Other workloads measured beside the headline (one GPU, default workload only):
# name, workload, attention layers per step.
SUB_WORKLOADS = (
    ("llama3_8b_prefill_64k", S.workload("llama3_8b_prefill_64k"), 1),
    ("wide_head_decode_64k_b32", S.workload("wide_head_decode_64k"), 2),
    ("host_tier_decode_128k_b8", S.workload("host_tier_decode_128k"), 1),
    ("llama3_8b_decode_32k_b4", S.workload("llama3_8b_decode_32k", batch=4, needles=0), 4),
    ("llama3_8b_decode_32k_b1", S.workload("llama3_8b_decode_32k", batch=1, needles=0), 4),
    ("paged_ragged_decode_32k_b16", S.workload("llama3_8b_decode_32k", needles=0), 4),
    ("training_step_64k", S.workload("llama3_8b_prefill_64k"), 1),
)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        line = run_reference(args, rank)
        if line:
            print(json.dumps(line))
        return
    import torch
    from hierarchical_sparse_attention_hga_b200 import binding as B
    from hierarchical_sparse_attention_hga_b200.build import build

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    if world > 1:
        rank, world = init_ranks("nccl")
    build()
    B.load_library()
    dev = torch.device("cuda")
    ranks = Ranks(world, dev)
    if args.sub:
        name, swl, layers = next(t for t in SUB_WORKLOADS if t[0] == args.sub)
        if args.batch:
            swl = swl.with_(batch=args.batch)
        if args.context:
            swl = swl.with_(context=args.context)
        seed = rank_seed(swl.name, rank)
        if name.startswith("training"):
            r = training_record(args, swl, args.steps, args.warmup, world, ranks, seed)
        elif swl.prefill:
            r = prefill_record(args, swl, args.steps, args.warmup, world, ranks, seed)
        elif name.startswith("paged"):
            r = paged_record(args, swl, layers, args.steps, args.warmup, world, ranks, seed)
        else:
            r = decode_record(args, swl, layers, args.steps, args.warmup, world, ranks, seed,
                              compare=False)
        if rank == 0:
            print(json.dumps({"workload": name, "n_gpus": world, "steps": args.steps,
                              "warmup": args.warmup, **r}))
        return
    wl = workload_of(args)
    seed = rank_seed(args.workload, rank)
    x = S.make_inputs(wl, seed)
    if wl.prefill:
        rec = prefill_record(args, wl, args.steps, args.warmup, world, ranks, seed, x)
    else:
        layers = args.layers or (1 if wl.name.startswith("host_tier") else 4)
        rec = decode_record(args, wl, layers, args.steps, args.warmup, world, ranks, seed, x)
    line = {"metric": METRIC + (" (prefill)" if wl.prefill else ""), "value": rec.pop("value"),
            "unit": rec.pop("unit"), "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": rec.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": rec.pop("dtype", "bf16 K/V, fp32 accumulation" if wl.dtype == "bf16" else "f32"),
            **rec}
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, seed, args.cpu_seconds, line["unit"])
    default_run = (args.workload == "llama3_8b_decode_32k" and not args.batch and not args.context
                   and not args.dtype)
    if world == 1 and default_run and not args.no_workloads:
        del x
        subs = {}
        sub_steps = max(3, min(args.steps, 20))
        for i, (name, swl, layers) in enumerate(SUB_WORKLOADS):
            sseed = rank_seed(swl.name, 0) + 17 * (i + 1)
            if name.startswith("training"):
                r = training_record(args, swl, sub_steps, args.warmup, world, ranks, sseed)
            elif swl.prefill:
                r = prefill_record(args, swl, sub_steps, args.warmup, world, ranks, sseed)
            elif name.startswith("paged"):
                r = paged_record(args, swl, layers, sub_steps, args.warmup, world, ranks, sseed)
            else:
                r = decode_record(args, swl, layers, sub_steps, args.warmup, world, ranks, sseed,
                                  compare=False)
            r["steps"] = sub_steps
            if not args.no_cpu_baseline and not name.startswith(("paged", "training")):
                r["cpu_baseline"] = cpu_baseline(swl, sseed, 3.0, r["unit"])
            subs[name] = r
        line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
