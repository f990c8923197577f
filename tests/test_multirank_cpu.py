"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1 agree on the
max-over-ranks step time, and replicas count every rank's work in the whole-job flops."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json
sys.path.insert(0, sys.argv[1])
import bench
rank, world, _ = bench.dist_setup(2)
ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
bench.barrier(world)
slowest = bench.max_over_ranks(ms, world)
import types, torch, synth
w = synth.Workload("rep", 1, 1, 32, 5, 40, (40,), 1.0, False)
prob = bench.Problem(None, w, types.SimpleNamespace(seed=0, split_mode="separate"), rank, world, "replicas",
                     torch.device("cpu"))
value = prob.flops_job / (slowest * 1e-3) / 1e12
print(json.dumps({"rank": rank, "world": world, "slowest": slowest, "value": value,
                  "flops_total": prob.flops_total}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_gloo_ranks_take_the_max_and_count_all_work(tmp_path):
    import json
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2 and o["slowest"] == 15.0
        assert o["flops_total"] == 4.0 * 1 * 5 * 40 * 32
        assert abs(o["value"] - 2 * o["flops_total"] / 15e-3 / 1e12) < 1e-12


def test_reference_arm_runs_on_host_cores():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "3", "--cpu-seconds", "0.5"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT,
                         env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert out.returncode == 0, out.stderr
    import json
    rec = json.loads(out.stdout.strip().splitlines()[-1])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["higher_is_better"] is True


def test_reference_arm_takes_the_host_cores_back_from_torchrun_s_default():
    """torchrun starts every rank with OMP_NUM_THREADS=1; the reference arm (rank 0 alone)
    still times the oracle on every core the process may use."""
    import json
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "3", "--cpu-seconds", "0.5"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr
    rec = json.loads(out.stdout.strip().splitlines()[-1])
    assert rec["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))
