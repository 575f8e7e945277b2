"""The N > 1 path of bench.py on the CPU: two ranks as separate processes over
gloo (127.0.0.1), no GPU.

* the timing aggregation uses the slowest rank (max over ranks) and counts
  the work of every rank (weak scaling);
* the barrier and the max-over-ranks collective run with real collectives;
* each rank draws its own seeded inputs (same shapes, different values);
* the reference arm prints one JSON line on rank 0 and nothing elsewhere.
"""

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["REPO"])
import torch, torch.distributed as dist
import bench
from factorized_block_sparse_b200 import synth
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", init_method="env://", rank=rank, world_size=world)
bench.barrier(world)
local_ms = 10.0 if rank == 0 else 25.0   # rank 1 is the slow one
value, tok_s, ms_step = bench.whole_job(world, 1e12, 1000, local_ms, 5, torch.device("cpu"))
x = synth.inputs(1, 1, 64, 32, seed_offset=rank)
bench.barrier(world)
print(json.dumps({"rank": rank, "value": value, "tok_s": tok_s, "ms_step": ms_step,
                  "q0": float(x["q"].float()[0, 0, 0, 0])}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), REPO=ROOT)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    return env


def test_two_ranks_over_gloo():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", CHILD], env=_env(r, 2, port), cwd=ROOT,
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    a, b = sorted(outs, key=lambda d: d["rank"])
    # slowest rank: 25 ms over 5 steps = 5 ms per step; both ranks' work counted
    for d in (a, b):
        assert abs(d["ms_step"] - 5.0) < 1e-12
        assert abs(d["value"] - 2 * 1e12 / 5e-3 / 1e12) < 1e-9
        assert abs(d["tok_s"] - 2 * 1000 / 5e-3) < 1e-6
    assert a["q0"] != b["q0"]  # each rank has its own data


def test_reference_arm_prints_on_rank_zero_only():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny-strided",
           "--steps", "1", "--warmup", "3", "--gpus", "2"]
    r1 = subprocess.run(cmd, env=_env(1, 2, _free_port()), cwd=ROOT, capture_output=True, text=True, timeout=240)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = subprocess.run(cmd, env=_env(0, 2, _free_port()), cwd=ROOT, capture_output=True, text=True, timeout=240)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
