"""The benchmark's multi-process path on CPU: two ranks over gloo.

The data path has no collective (the ranks decode independent sequences), so
what is tested here is the plumbing around it: every rank joins the group,
takes the same barriers, reports the MAX of the ranks' times, and the job's
value counts the units of all ranks.  The oracle arm under torchrun prints one
line, from rank 0, and the other rank exits 0 without work.
"""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import hga_synth as S  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w = bench.init_ranks("gloo")
    ranks = bench.Ranks(w, "cpu")
    ranks.barrier()
    step_ms = 0.5 + rank          # a slower rank must set the job's time
    m = ranks.max(step_ms)
    ranks.barrier()
    wl = S.workload("llama3_8b_decode_32k", batch=1, context=2048)
    seed = bench.rank_seed(wl.name, r)
    q = S.query_slice(wl, seed, 0, 1)
    res = dict(rank=r, world=w, max_ms=m, seed=seed, rate=bench.job_rate(wl.batch, w, m),
               q0=float(np.asarray(q, dtype=np.float64).ravel()[0]))
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_job_rate(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [x["rank"] for x in res] == [0, 1] and all(x["world"] == 2 for x in res)
    # every rank reports the slowest rank's time
    assert all(x["max_ms"] == pytest.approx(1.5) for x in res)
    # value = units of all ranks over that time: 2 sequences / 1.5 ms
    assert all(x["rate"] == pytest.approx(2 / 1.5e-3) for x in res)
    # ranks decode different sequences
    assert res[0]["seed"] != res[1]["seed"] and res[0]["q0"] != res[1]["q0"]


def test_single_rank_plumbing_is_a_no_op():
    ranks = bench.Ranks(1, "cpu")
    ranks.barrier()
    assert ranks.max(3.25) == 3.25
    assert bench.job_rate(16, 1, 2.0) == pytest.approx(8000.0)


def _torchrun(args, nproc, timeout=240):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py")] + args
    env = dict(os.environ, OMP_NUM_THREADS="1")
    return subprocess.run(cmd, capture_output=True, text=True, timeout=timeout, env=env, cwd=ROOT)


def test_oracle_arm_under_torchrun_prints_one_line_from_rank0():
    r = _torchrun(["--impl", "reference", "--gpus", "2", "--workload", "tiny_f32_1k",
                   "--steps", "3", "--warmup", "3", "--cpu-seconds", "0.2"], nproc=2)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 3
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_oracle_arm_prefill_workload():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "llama3_8b_prefill_64k", "--context", "2048", "--steps", "3",
           "--warmup", "3", "--cpu-seconds", "0.2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["unit"].startswith("prefill") and line["config"]["context"] == 2048
    assert line["ms_per_step"] == pytest.approx(2048 / line["value"] * 1e3)
