"""bench.py's multi-GPU modes on two gloo ranks (CPU), with the oracle standing in for the
kernels.

bench.Problem cuts one workload across ranks and runs the step the benchmark times:
  - query sharding: each rank takes a contiguous block of query rows and all keys, and
    nothing crosses ranks (each row's softmax depends on its own scores only);
  - key sharding: each rank takes a contiguous block of key slots, cuts it into
    chunks, and the chunk partials of all ranks cross in one all-gather before the
    exact log-sum-exp combine ("Add sequence-parallel multi-GPU inference ...",
    section "Sequence-parallel inference").
Here every kernel call of the step is answered by the fp64 oracle on the same
arguments, so the test checks the partition and the exchange: the rows assembled from
the ranks (query sharding) and every rank's combined output (key sharding) must equal
the unsharded oracle.  Shapes are ragged: the row and key blocks are unequal, one batch
element's prefix ends inside rank 0's key block, so rank 1 holds no valid key of it.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import os, sys, json, math, types
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
import bench, oracle, synth

rank, world, _ = bench.dist_setup(2)


def chunk_len(Tk, C):
    # the documented split rule of attn_split_chunk_len: ceil(Tk / C) rounded up to 128 keys
    per = -(-Tk // C)
    return -(-per // 128) * 128


class OracleKP:
    """The kernel calls of bench.Problem.step, answered by the oracle."""
    ATTN_OK = 0

    def attn_prefix_fwd(self, q, k, v, kv, scale, out, lse):
        o, l = oracle.attn_prefix(q, k, v, kv.tolist(), scale)
        out.copy_(torch.from_numpy(o))
        lse.copy_(torch.from_numpy(l))

    def attn_prefix_fwd_split(self, q, k, v, kv, C, scale, po, pl):
        L = chunk_len(k.shape[2], C)
        for c in range(C):
            o, l = oracle.attn_chunk(q, k, v, kv.tolist(), scale, c * L, (c + 1) * L)
            po[c].copy_(torch.from_numpy(o))
            pl[c].copy_(torch.from_numpy(l))

    def attn_lse_combine(self, po, pl, out, lse):
        o, l = oracle.lse_combine(po.double().numpy(), pl.double().numpy())
        out.copy_(torch.from_numpy(o))
        lse.copy_(torch.from_numpy(l))


args = types.SimpleNamespace(seed=3, split_mode="separate")
res = {}
# prefix workload, query-sharded: 37 rows -> blocks of 19 and 18
wq = synth.Workload("shard_q", 2, 2, 32, 37, 300, (300, 170), 1.0, True)
pq = bench.Problem(OracleKP(), wq, args, rank, world, "queries", torch.device("cpu"))
pq.step()
blocks = [None] * world
dist.all_gather_object(blocks, (pq.r0, pq.r1, pq.out.float().numpy(), pq.lse.numpy()))
ref_o, ref_l = oracle.attn_prefix(pq.case["q"], pq.case["k"], pq.case["v"], pq.case["kv_len_list"],
                                  pq.case["scale"])
ranges = [(b[0], b[1]) for b in blocks]
got_o = np.concatenate([b[2] for b in blocks], axis=2)
got_l = np.concatenate([b[3] for b in blocks], axis=2)
res["q_ranges"] = ranges
res["q_err_out"] = float(np.abs(got_o - ref_o).max())
res["q_lse_ninf_same"] = bool(np.array_equal(np.isneginf(got_l), np.isneginf(ref_l)))
fin = np.isfinite(ref_l)
res["q_err_lse"] = float(np.abs(got_l[fin] - ref_l[fin]).max())
res["q_flops_job"] = pq.flops_job
res["q_in_bytes_ok"] = bench.input_bytes(wq, rank, world, "queries") == sum(
    t.numel() * t.element_size() for t in (pq.q, pq.k, pq.v))
res["q_flops_total"] = pq.flops_total
# split-KV workload, key-sharded: 700 key slots -> blocks of 384 and 316 (3 and 3 tiles);
# element 1's prefix (200) ends inside rank 0's block
wk = synth.Workload("shard_k", 2, 2, 32, 21, 700, (650, 200), 1.0, True, num_splits=4)
pk = bench.Problem(OracleKP(), wk, args, rank, world, "keys", torch.device("cpu"))
pk.step()
ref_o, ref_l = oracle.attn_prefix(pk.case["q"], pk.case["k"], pk.case["v"], pk.case["kv_len_list"],
                                  pk.case["scale"])
res["k_bounds"] = (pk.k0, pk.k1)
res["k_kv_local"] = pk.kv_list
res["k_chunks"] = pk.c_local
res["k_err_out"] = float(np.abs(pk.out.float().numpy() - ref_o).max())
res["k_err_lse"] = float(np.abs(pk.lse.numpy() - ref_l).max())
res["k_flops_rank"] = pk.flops_rank
res["k_in_bytes_ok"] = bench.input_bytes(wk, rank, world, "keys") == sum(
    t.numel() * t.element_size() for t in (pk.q, pk.k, pk.v))
res["k_flops_total"] = pk.flops_total
print(json.dumps({"rank": rank, **res}), flush=True)
dist.destroy_process_group()
'''


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_gloo_ranks_shard_queries_and_keys(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER)
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script), ROOT], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    outs.sort(key=lambda o: o["rank"])
    for o in outs:
        # query sharding: the blocks tile [0, Tq) in rank order, and the assembled rows
        # are the unsharded result (bf16 output rounding only)
        assert [tuple(r) for r in o["q_ranges"]] == [(0, 19), (19, 37)]
        assert o["q_err_out"] < 1e-2 and o["q_err_lse"] < 1e-6 and o["q_lse_ninf_same"]
        assert o["q_flops_job"] == o["q_flops_total"]
        # the L2-flush decision and the configs both arms print use these shard sizes
        assert o["q_in_bytes_ok"] and o["k_in_bytes_ok"]
        # key sharding: every rank holds the exact combined result
        assert o["k_err_out"] < 1e-2 and o["k_err_lse"] < 1e-6
        assert o["k_chunks"] == 2
    assert tuple(outs[0]["k_bounds"]) == (0, 384) and tuple(outs[1]["k_bounds"]) == (384, 700)
    assert outs[0]["k_kv_local"] == [384, 200] and outs[1]["k_kv_local"] == [266, 0]
    # the ranks' key-sharded work adds up to the whole problem's
    assert abs(outs[0]["k_flops_rank"] + outs[1]["k_flops_rank"] - outs[0]["k_flops_total"]) < 1e-6


def test_shard_blocks_cover_every_row_and_key_once():
    sys.path.insert(0, ROOT)
    from key_prefix_masked_b200 import sharded
    for T, world in ((110000, 8), (37, 2), (5, 8), (1024, 3)):
        rows = [sharded.query_rows(T, r, world) for r in range(world)]
        assert rows[0][0] == 0 and rows[-1][1] == T
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
        assert max(b - a for a, b in rows) - min(b - a for a, b in rows) <= 1
    for Tk, world in ((1000000, 8), (700, 2), (100352, 3)):
        ks = [sharded.key_bounds(Tk, r, world) for r in range(world)]
        assert ks[0][0] == 0 and ks[-1][1] == Tk
        assert all(a[1] == b[0] and a[1] % 128 == 0 for a, b in zip(ks, ks[1:]))
    assert sharded.shard_kv_len([650, 200, 0, 700], 384, 700) == [266, 0, 0, 316]


def test_reference_arm_names_the_same_config():
    """The reference arm's `config` is the one the GPU arm prints for the same workload,
    so the two lines name the same work (its value comes from a bounded oracle sample)."""
    import types
    sys.path.insert(0, ROOT)
    import bench
    import synth
    for name in ("tiny", "unmasked_8v"):
        w = synth.WORKLOADS[name]
        args = types.SimpleNamespace(workload=name, seed=0, cpu_seconds=0.2, steps=1, warmup=3,
                                     shard="auto", split_mode="separate")
        rec = bench.run_reference(args, 0, 1)
        case = synth.make_inputs(w, device="cpu", seed=0)
        ours = {**bench.workload_config(w, case, args, 1, "single", bench.needs_flush(w, 0, 1, "single")),
                "parallelism": bench.PARALLELISM["single"].format(n=1)}
        assert rec["config"] == ours
        assert rec["scaling"] == "weak" and rec["impl"] == "reference"


def test_traffic_of_a_changed_kernel_is_null(tmp_path, monkeypatch):
    """A committed traffic summary counts only while it was taken on the current kernel."""
    import json as _json
    sys.path.insert(0, ROOT)
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k_w_traffic.json").write_text(_json.dumps({"dram_bytes_per_launch": 123}))
    (prof / "k_old_traffic.json").write_text(_json.dumps({"dram_bytes_per_launch": 456, "current": False}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profile("w", "k") == 123
    assert bench.traffic_from_profile("old", "k") is None
    assert bench.traffic_from_profile("missing", "k") is None
