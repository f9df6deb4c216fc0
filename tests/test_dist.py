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


# ------------------------------------------------------------------ a context split over two ranks
SPLIT_WORKER = r"""
import datetime, json, math, os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import numpy as np
import torch
import torch.distributed as dist
import oracle
from long_context_decode_kv1b_b200 import context_split as cs
rank, world = int(os.environ["RANK"]), 2
dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
rng = np.random.default_rng(7)                     # every rank draws the same sequence and queries
L, G = 3001, 4
K = rng.standard_normal((L, 128)).astype(np.float32)
V = rng.standard_normal((L, 128)).astype(np.float32)
q = rng.standard_normal((G, 128)).astype(np.float32)
D = oracle.signs(11)
t0, t1 = cs.shard_bounds(L, world, rank)
enc = oracle.encode(K[t0:t1], V[t0:t1], D)         # this rank's token range only
part = np.zeros((G, 130), np.float32)
for j in range(G):
    m, l, o = oracle.attend_partial(enc, q[j], D, 0.3)
    part[j, 0], part[j, 1], part[j, 2:] = m, l, o
parts = cs.exchange(torch.from_numpy(part)).numpy()   # [world, G, 130]
M = parts[:, :, 0].max(axis=0)
w = np.exp2(parts[:, :, 0] - M).astype(np.float64)
out = (w[..., None] * parts[:, :, 2:]).sum(0) / (w * parts[:, :, 1]).sum(0)[:, None]
print(json.dumps({"rank": rank, "range": [t0, t1], "out": out.tolist(),
                  "first": parts[0, 0, :4].tolist(), "second": parts[1, 0, :4].tolist()}))
dist.destroy_process_group()
"""


def test_context_split_over_two_gloo_ranks_matches_the_whole_sequence():
    # each rank encodes and attends over its own token range; the exchanged log-sum-exp rows merge
    # into the attention over the whole context (the oracle's, at the 1e-3 bar, here ~1e-6)
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle

    port = _port()
    procs = [subprocess.Popen([sys.executable, "-c", SPLIT_WORKER], env=_env(r, port), stdout=subprocess.PIPE,
                              stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert outs[0]["range"] == [0, 1501] and outs[1]["range"] == [1501, 3001]
    assert outs[0]["first"] == outs[1]["first"] and outs[0]["second"] == outs[1]["second"]  # same gather
    rng = np.random.default_rng(7)
    K = rng.standard_normal((3001, 128)).astype(np.float32)
    V = rng.standard_normal((3001, 128)).astype(np.float32)
    q = rng.standard_normal((4, 128)).astype(np.float32)
    D = oracle.signs(11)
    enc = oracle.encode(K, V, D)
    ref = np.stack([oracle.attend(enc, q[j], D, 0.3) for j in range(4)])
    for o in outs:
        got = np.asarray(o["out"])
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_shard_bounds_cover_the_context_once():
    sys.path.insert(0, ROOT)
    from long_context_decode_kv1b_b200 import context_split as cs

    for length in (0, 1, 7, 1024, 1048577):
        for world in (1, 2, 3, 8):
            spans = [cs.shard_bounds(length, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == length
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    assert cs.append_rank(4) == 3
