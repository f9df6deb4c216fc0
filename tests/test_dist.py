"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo (127.0.0.1).

The data path has no collective (each rank runs its own sequences); what is shared between ranks
is the timing and the unit count: the maximum of the per-rank times and the sum of the per-rank
units, and that only rank 0 prints.  Those are checked here without a GPU.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import torch.distributed as dist
import bench
rank = int(os.environ["RANK"])
dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
t = bench.reduce_max(10.0 * (rank + 1), 2)
u = bench.reduce_sum(1000.0 + rank, 2)
bench.barrier(2)
print(json.dumps({"rank": rank, "max": t, "sum": u}))
dist.destroy_process_group()
"""


def _port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, port: int) -> dict:
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port), REPO_ROOT=ROOT)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    return env


def test_max_time_and_summed_units_over_two_gloo_ranks():
    port = _port()
    procs = [subprocess.Popen([sys.executable, "-c", WORKER], env=_env(r, port), stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["max"] == 20.0  # time = max over ranks
        assert o["sum"] == 2001.0  # units = sum over ranks


def test_reference_arm_prints_on_rank_zero_only():
    port = _port()
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--config", "c1",
           "--steps", "1", "--warmup", "0"]
    r1 = subprocess.run(cmd, env=_env(1, port), capture_output=True, text=True, timeout=300)
    assert r1.returncode == 0, r1.stderr[-2000:]
    assert r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=_env(0, port), capture_output=True, text=True, timeout=300)
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [ln for ln in r0.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
