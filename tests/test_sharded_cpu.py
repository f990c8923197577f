"""Key-sharded attention across ranks, host side, on two gloo ranks (CPU).

The exchange step of the sequence-parallel scheme ("Add sequence-parallel multi-GPU
inference ...", section "Sequence-parallel inference") is sharded.gather_partials:
every rank's partial (O_r, lse_r) stacked in rank order. It is tested here with the
oracle standing in for the two GPU steps (the per-shard partial and the combine).
Shards are unequal in size, and one batch element has an empty shard on rank 1. The
sharded result must equal the unsharded oracle over all the keys.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
import oracle, synth
from key_prefix_masked_b200 import sharded

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world,
                        init_method="tcp://127.0.0.1:" + os.environ["MASTER_PORT"])
B, H, Tq, Tk, D = 2, 2, 9, 100, 16
kv_full = [100, 40]
c = synth.random_case(B, H, Tq, Tk, D, tuple(kv_full), seed=5)   # same draw on every rank
scale = 0.25
bounds = [(0, 60), (60, 100)]                 # unequal shards; element 1 has none on rank 1
lo, hi = bounds[rank]
k_loc = c["k"][:, :, lo:hi].contiguous()
v_loc = c["v"][:, :, lo:hi].contiguous()
kv_loc = [max(0, min(n - lo, hi - lo)) for n in kv_full]
po, pl = oracle.attn_prefix(c["q"], k_loc, v_loc, kv_loc, scale)   # stands in for local_partial
po = torch.from_numpy(po)[None]
pl = torch.from_numpy(pl)[None]
go, gl = sharded.gather_partials(po, pl)
assert go.shape == (world, B, H, Tq, D) and gl.shape == (world, B, H, Tq)
out, lse = oracle.lse_combine(go.numpy(), gl.numpy())             # stands in for combine
ref_out, ref_lse = oracle.attn_prefix(c["q"], c["k"], c["v"], kv_full, scale)
err_out = float(np.abs(out - ref_out).max())
err_lse = float(np.abs(lse - ref_lse).max())
own = bool(torch.equal(go[rank], po[0]) and torch.equal(gl[rank], pl[0]))   # rank order kept
print(json.dumps({"rank": rank, "err_out": err_out, "err_lse": err_lse, "own_slot": own,
                  "empty_shard_lse": float(gl[1, 1].max())}), flush=True)
dist.destroy_process_group()
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_gloo_ranks_key_sharded_equals_unsharded(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["err_out"] < 1e-12 and o["err_lse"] < 1e-12
        assert o["own_slot"]
        assert o["empty_shard_lse"] == float("-inf")
