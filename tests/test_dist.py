"""Multi-process host logic of the benchmark (world size 2, gloo, CPU): the
rank plumbing, the per-rank workloads and the whole-job aggregation."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import json, os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench, synth
world, rank, local = bench.dist_init("gloo")
w = bench.rank_workload(synth.WORKLOADS["llama1b_stack16_b8_128k"], rank)
# each rank reports a different "elapsed" time; the job takes the slowest
mx = bench.max_over_ranks(10.0 + rank, world)
sm = bench.sum_over_ranks(1.0, world)
bench.barrier(world)
v = bench.aggregate_value(64, mx, world)
q = synth.queries(w, 0, 1, B=1, h_q=2)
print(json.dumps({"rank": rank, "world": world, "seed": w.seed, "max": mx, "sum": sm,
                  "value": v, "q0": int(q[0, 0, 0, 0])}))
import torch.distributed as dist
dist.destroy_process_group()
'''


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gloo():
    import json
    port = free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=240)
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    outs.sort(key=lambda d: d["rank"])
    assert [d["world"] for d in outs] == [2, 2]
    assert all(d["max"] == 11.0 and d["sum"] == 2.0 for d in outs)
    assert all(abs(d["value"] - 2 * 64 / 0.011) < 1e-6 for d in outs)
    # rank 0 keeps the canonical workload, rank 1 draws an independent batch
    import synth
    assert outs[0]["seed"] == synth.WORKLOADS["llama1b_stack16_b8_128k"].seed
    assert outs[1]["seed"] != outs[0]["seed"] and outs[1]["q0"] != outs[0]["q0"]


def test_reference_arm_only_rank0_prints(tmp_path):
    """Under torchrun the oracle arm runs on rank 0 alone; other ranks exit 0
    silently."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "2", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_single_process():
    import json
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("RANK", None); env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_f32", "--steps", "3", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "steps/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_starts_the_ranks_it_is_asked_for():
    """bench.py --gpus 2 outside torchrun starts two ranks (gloo on CPU here)
    and rank 0 alone prints one line, with n_gpus 2."""
    import json
    import subprocess
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--workload", "tiny_f32", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"
