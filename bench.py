"""Benchmark: prefix-masked attention forward on B200, TFLOP/s over valid keys.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload icl] [--impl ours|reference]

One step = one pass of the hot path over one batch of the workload, inputs resident in
HBM: for the single-pass workloads one attn_prefix_fwd launch (key-range selection,
TMA staging, QK^T, prefix mask, online softmax, PV, epilogue); for `splitkv` the split
partial launch plus the LSE combine launch (`--split-mode fused`: one launch whose last
chunk per query tile runs the combine, attn_prefix_fwd_split_fused).  FLOPs counted = sum_b 4*H*Tq*kv_len[b]*D.

The default workload is the in-context-learning shape: B=1, H=8, D=256, 110000 queries
against 100000 valid keys in a 100352-row padded key buffer.  Its inputs (1.27 GB) are
larger than the 126 MB L2, so no flush is needed between steps.  A workload whose
q, k and v together are smaller than twice the L2 (the D=64 shapes) gets a 252 MB buffer
written before every timed step, outside that step's CUDA events; its value then comes
from the per-step events.

After the headline line's workload, the same run times every other workload of the
pages at one GPU (tiny, the three unmasked D=64 sizes, ragged, split-KV) and reports each
under `configs`, with its roofline, clocks, oracle check and oracle time.

Multi-GPU (torchrun, one process per GPU; --shard): by default the query rows of the one
problem are split across ranks with no exchange (strong scaling); split-KV workloads
split the key slots instead, and the partials cross ranks in one all-gather before the
exact log-sum-exp combine.  --shard replicas runs one whole replica per rank (weak
scaling).  The step time is the max over ranks; the value counts the whole job's work.

`--impl reference` times the fp64 CPU oracle on this machine's host cores instead (the
only reference this method has), on a bounded sample of query rows of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "attention fwd TFLOP/s (valid keys only) and % of BF16 tensor peak on one B200"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_flops(w: synth.Workload, kv_list) -> float:
    return float(sum(4.0 * w.H * w.Tq * n * w.D for n in kv_list))


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clock sampling
class ClockMonitor:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "power": float(parts[3]) if parts[3] not in ("", "[N/A]") else 0.0,
                             "active": parts[4], "hw": parts[5], "hwt": parts[6], "swt": parts[7],
                             "pcap": parts[8]})
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r["power"] for r in rows)
        loaded = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows),
                "power_w_max": pmax, "samples": len(rows), "samples_under_load": len(loaded),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ our arm
# Sharding of one workload across ranks (torchrun, one process per GPU):
#   queries  rank r takes a contiguous block of query rows and every key; no exchange.
#   keys     rank r takes a contiguous block of key slots and every query row; the
#            partials cross ranks in one all-gather (NCCL) and combine exactly.
#   replicas every rank runs the whole workload (weak scaling).
# "auto" picks keys for the split-KV workload (short query block, huge context) and
# queries for the others.  With one rank all three are the single-GPU step.
def resolve_shard(shard: str, w) -> str:
    if shard != "auto":
        return shard
    return "keys" if w.num_splits > 1 else "queries"


# Workloads timed in the same run beside the headline one, one entry each in `configs`.
CONFIG_SWEEP = ("tiny", "unmasked", "unmasked_8v", "unmasked_32v", "ragged", "splitkv")
MUFU_EX2_PER_CLK_SM = 16      # ex2.approx.f32 results per clock per SM (measured on B200: 8 cycles per warp-instruction per sub-partition)
NUM_SMS = 148


def mufu_bound_tflops(D: int, sm_mhz: float) -> float:
    """Valid-key TFLOP/s at which every SM's MUFU runs one ex2 per score without pause:
    4*D flops per score, 16 ex2 per clock per SM."""
    return 4.0 * D * MUFU_EX2_PER_CLK_SM * NUM_SMS * sm_mhz * 1e6 / 1e12


def kernel_names(w, splits):
    if w.D in (128, 256):
        tag = "attn_fwd_pair" if w.D == 256 else f"attn_fwd_pair_d{w.D}"
        return tag, f"attn_fwd_pair_kernel<{w.D},{int(bool(splits))}>"
    return f"attn_fwd_d{w.D}", f"attn_fwd_kernel<{w.D},{int(bool(splits))}>"


def roofline_entry(w, workload_name, achieved, clocks, splits):
    """The dominant kernel against its bound.  Head dims 128 and 256: the tensor pipe,
    `frac` against the measured burst cuBLAS bf16 figure (the kernel is timed as its own
    launch), `frac_sustained` against the seconds-long cuBLAS loop under the same 1 kW
    power cap a back-to-back run of this kernel draws, `frac_nominal` against 2250.
    Head dims 32 and 64: the MUFU's ex2 rate (bound "alu", peak from 16 ex2 per clock
    per SM at the maximum SM clock), the tensor figures beside it."""
    peaks, src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    tag, kname = kernel_names(w, splits)
    tensor = {"frac_tensor_burst": round(achieved / burst, 4), "frac_tensor_sustained": round(achieved / sus, 4),
              "frac_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4)}
    traffic = traffic_from_profile(workload_name, tag)
    if w.D <= 64:
        max_mhz = float(clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz", 1965.0))
        peak = mufu_bound_tflops(w.D, max_mhz)
        return {"bound": "alu", "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_rule": f"MUFU ex2 bound: {MUFU_EX2_PER_CLK_SM} ex2/clk/SM x {NUM_SMS} SMs x {max_mhz:.0f} MHz "
                             f"x 4*D flops per score (one exponential per score)",
                **tensor, "traffic": traffic, "kernel": kname}
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": burst, "unit": "TFLOP/s",
            "frac": round(achieved / burst, 4), "frac_sustained": round(achieved / sus, 4),
            "frac_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4),
            "peak_rule": f"frac: {src} burst cuBLAS bf16 ({burst}); frac_sustained: {src} seconds-long cuBLAS "
                         f"loop under the 1 kW cap ({sus}), the cap this back-to-back run also draws",
            "traffic": traffic, "kernel": kname}


class Problem:
    """One workload's inputs on this rank's GPU, sharded for `shard` across `world` ranks,
    and the step that runs the hot path over them."""

    def __init__(self, kp, w, args, rank, world, shard, dev):
        from key_prefix_masked_b200 import sharded
        self.kp, self.w, self.world, self.shard = kp, w, world, shard
        case = synth.make_inputs(w, device=dev, seed=args.seed)
        self.case = case
        self.scale = case["scale"]
        self.flops_total = workload_flops(w, case["kv_len_list"])
        self.splits = w.num_splits if w.num_splits > 1 else 0
        self.segs = w.segments is not None
        self.fused = bool(self.splits) and args.split_mode == "fused"
        q, k, v, kv = case["q"], case["k"], case["v"], case["kv_len"]
        self.r0, self.r1, self.k0, self.k1 = 0, w.Tq, 0, w.Tk
        self.kv_list = list(case["kv_len_list"])
        if world > 1 and shard == "queries":
            self.r0, self.r1 = sharded.query_rows(w.Tq, rank, world)
            q = q[:, :, self.r0:self.r1].contiguous()
        elif world > 1 and shard == "keys":
            if self.segs:
                raise SystemExit("key sharding is not defined for the multi-range workload")
            self.k0, self.k1 = sharded.key_bounds(w.Tk, rank, world)
            k = k[:, :, self.k0:self.k1].contiguous()
            v = v[:, :, self.k0:self.k1].contiguous()
            self.kv_list = sharded.shard_kv_len(case["kv_len_list"], self.k0, self.k1)
            kv = torch.tensor(self.kv_list, dtype=torch.int32, device=dev)
        self.q, self.k, self.v, self.kv = q, k, v, kv
        # work done by this rank (the whole job's work is flops_total in the sharded modes)
        rows = self.r1 - self.r0
        self.flops_rank = float(sum(4.0 * w.H * rows * n * w.D for n in self.kv_list))
        self.flops_job = job_flops(w, case["kv_len_list"], world, shard)
        B, H, D = w.B, w.H, w.D
        Tq_l = self.q.shape[2]
        self.out = torch.empty((B, H, Tq_l, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, H, Tq_l), dtype=torch.float32, device=dev)
        self.seg_ws = (torch.empty(int(kp.lib().attn_segments_workspace_bytes(B, H, w.Tk, D)), dtype=torch.uint8,
                                   device=dev) if self.segs else None)
        self.ws = kp.fused_workspace(self.splits, B, H, Tq_l, D, dev) if self.fused else None
        # key sharding: each rank cuts its shard into num_splits / world chunks
        self.c_local = max(1, self.splits // world) if (shard == "keys" and world > 1) else self.splits
        self.parts = ((torch.empty((self.c_local, B, H, Tq_l, D), dtype=torch.float32, device=dev),
                       torch.empty((self.c_local, B, H, Tq_l), dtype=torch.float32, device=dev))
                      if self.splits and not self.fused else None)
        self.kernel_events = []    # split step: events around the split launch (the dominant kernel)
        self.launches_per_step = 2 if ((self.splits and not self.fused) or self.segs) else 1

    def step(self, timed=False):
        kp = self.kp
        if self.segs:
            kp.attn_prefix_fwd_segments(self.q, self.k, self.v, self.case["seg_start"], self.case["seg_len"],
                                        self.scale, workspace=self.seg_ws, out=self.out, lse=self.lse)
        elif self.fused:
            kp.attn_prefix_fwd_split_fused(self.q, self.k, self.v, self.kv, self.splits, self.scale,
                                           workspace=self.ws, out=self.out, lse=self.lse)
        elif self.splits:
            if timed:
                stream = torch.cuda.current_stream()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            kp.attn_prefix_fwd_split(self.q, self.k, self.v, self.kv, self.c_local, self.scale, *self.parts)
            if timed:
                b_.record(stream)
                self.kernel_events.append((a, b_))
            po, pl = self.parts
            if self.shard == "keys" and self.world > 1:
                from key_prefix_masked_b200 import sharded
                po, pl = sharded.gather_partials(po, pl)
            kp.attn_lse_combine(po, pl, out=self.out, lse=self.lse)
        else:
            kp.attn_prefix_fwd(self.q, self.k, self.v, self.kv, self.scale, out=self.out, lse=self.lse)

    def verify(self):
        """The step's output on a few query rows against the oracle (outside every timed
        region).  Query sharding: rows of this rank's block."""
        rows_l = sorted({0, 1, min(127, self.r1 - self.r0 - 1), min(128, self.r1 - self.r0 - 1),
                         (self.r1 - self.r0) // 2, self.r1 - self.r0 - 1})
        if self.w.name == "tiny":
            rows_l = list(range(self.r1 - self.r0))   # the whole output
        rows_g = [self.r0 + r for r in rows_l]
        return verify_rows(self.case, self.out, self.lse, rows_g, rows_l)


def device_timed(prob, steps, world, flush, clocks_gpu, min_ms=0.0):
    """Time `steps` steps (more when the first measurement says they end under `min_ms`)
    with CUDA events on the launching stream, between barriers; nvidia-smi clocks are
    sampled meanwhile.  Returns (per-step ms, total ms for the max-over-ranks value,
    clock summary, steps)."""
    stream = torch.cuda.current_stream()
    if min_ms > 0:
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        prob.step()
        b_.record(stream)
        torch.cuda.synchronize()
        one = max(a.elapsed_time(b_), 1e-3) + (0.05 if flush is not None else 0.0)
        steps = max(steps, min(5000, int(math.ceil(min_ms / one))))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    prob.kernel_events.clear()
    with ClockMonitor(clocks_gpu) as mon:
        barrier(world)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            if flush is not None:
                flush.zero_()   # evict the inputs from L2 (outside the step's events)
            ev[i][0].record(stream)
            prob.step(timed=True)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    step_ms = [a.elapsed_time(b_) for a, b_ in ev]
    total_ms = sum(step_ms) if flush is not None else t0.elapsed_time(t1)
    return step_ms, total_ms, mon.summary(), steps


def l2_note(flushed: bool):
    return ("inputs larger than the 126 MB L2; no flush" if not flushed else
            "inputs smaller than 2x L2: a 252 MB buffer written before each step, outside the step "
            "events; value from per-step events")


def input_bytes(w, rank, world, shard) -> int:
    """Bytes of q, k and v that one rank holds (its shard)."""
    from key_prefix_masked_b200 import sharded
    rows, keys = w.Tq, w.Tk
    if world > 1 and shard == "queries":
        r0, r1 = sharded.query_rows(w.Tq, rank, world)
        rows = r1 - r0
    elif world > 1 and shard == "keys":
        k0, k1 = sharded.key_bounds(w.Tk, rank, world)
        keys = k1 - k0
    return 2 * w.B * w.H * w.D * (rows + 2 * keys)


def needs_flush(w, rank, world, shard) -> bool:
    return input_bytes(w, rank, world, shard) < 2 * L2_BYTES


def job_flops(w, kv_len_list, world, shard) -> float:
    total = workload_flops(w, kv_len_list)
    return total if (shard in ("queries", "keys") and world > 1) else total * world


SCALING = {"queries": "strong", "keys": "strong", "replicas": "weak", "single": "weak"}
PARALLELISM = {"queries": "query rows sharded x{n} (no exchange)",
               "keys": "key slots sharded x{n} (all-gather of partials, exact combine)",
               "replicas": "replicas x{n}", "single": "single GPU"}


def workload_config(w, case, args, world, shard, flushed):
    """The `config` object of a line; both arms build it here, so they name the same work."""
    return {**w.describe(),
            "kv_len": case["kv_len_list"] if len(case["kv_len_list"]) <= 8 else "ragged",
            "scale": case["scale"], "flops_per_step": job_flops(w, case["kv_len_list"], world, shard),
            "l2": l2_note(flushed),
            **({"split_mode": args.split_mode} if w.num_splits > 1 else {})}


def measure(kp, name, args, rank, world, shard, steps, min_ms=0.0):
    """Device-timed measurement of one workload: (record fields, problem)."""
    w = synth.WORKLOADS[name]
    dev = torch.device("cuda", torch.cuda.current_device())
    prob = Problem(kp, w, args, rank, world, shard, dev)
    for _ in range(args.warmup):
        prob.step()
    torch.cuda.synchronize()
    st = kp.device_status()
    if st != kp.ATTN_OK:
        raise RuntimeError(f"{name}: device status after warm-up: {kp.status_string(st)}")
    in_bytes = sum(t.numel() * t.element_size() for t in (prob.q, prob.k, prob.v))
    assert in_bytes == input_bytes(w, rank, world, shard), "shard shapes"
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if needs_flush(w, rank, world, shard) else None
    step_ms, total_ms, clocks, steps = device_timed(prob, steps, world, flush, torch.cuda.current_device(), min_ms)
    st = kp.device_status()
    if st != kp.ATTN_OK:
        raise RuntimeError(f"{name}: device status after timing: {kp.status_string(st)}")
    flush = flush is not None
    kern_ms = ([a.elapsed_time(b_) for a, b_ in prob.kernel_events] if prob.kernel_events else step_ms)
    seg_info = None
    if prob.segs:
        kern_ms, seg_info = segments_split_time(kp, prob, step_ms, steps)
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / steps
    value = prob.flops_job / (ms_per_step * 1e-3) / 1e12
    # the dominant kernel's own rate: its work on this rank over its average launch time
    kern_flops = prob.flops_rank
    achieved = kern_flops / (statistics.mean(kern_ms) * 1e-3) / 1e12
    rec = {
        "value": round(value, 2), "ms_per_step": round(ms_per_step, 4), "steps": steps,
        "config": workload_config(w, prob.case, args, world, shard, flush),
        "roofline": roofline_entry(w, name, achieved, clocks, prob.splits),
        "gpu_launches": prob.launches_per_step * steps,
        "clocks": clocks,
        "step_ms": {"min": round(min(step_ms), 4), "median": round(statistics.median(step_ms), 4),
                    "max": round(max(step_ms), 4)},
        **({"segments": seg_info} if seg_info else {}),
    }
    if args.verify and rank == 0:
        rec["verified_rows"] = prob.verify()
    return rec, prob


def segments_split_time(kp, prob, step_ms, steps):
    """Multi-range workload: the prefix kernel alone on the rows the gather left in the
    workspace (the same launch as inside the step); the rest of the step is the gather."""
    w = prob.w
    stream = torch.cuda.current_stream()
    kvb = (w.B * w.H * w.Tk * w.D * 2 + 255) // 256 * 256
    kg = prob.seg_ws[:w.B * w.H * w.Tk * w.D * 2].view(torch.bfloat16).view(w.B, w.H, w.Tk, w.D)
    vg = prob.seg_ws[kvb:kvb + w.B * w.H * w.Tk * w.D * 2].view(torch.bfloat16).view(w.B, w.H, w.Tk, w.D)
    kvg = prob.seg_ws[2 * kvb:2 * kvb + 4 * w.B].view(torch.int32)
    a_ev = []
    for _ in range(steps):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kp.attn_prefix_fwd(prob.q, kg, vg, kvg, prob.scale, out=prob.out, lse=prob.lse)
        b_.record(stream)
        a_ev.append((a, b_))
    torch.cuda.synchronize()
    kern_ms = [a.elapsed_time(b_) for a, b_ in a_ev]
    gather_ms = max(statistics.mean(step_ms) - statistics.mean(kern_ms), 1e-6)
    gather_bytes = 2 * 2 * sum(prob.case["kv_len_list"]) * w.H * w.D * 2   # K and V rows, read + write
    return kern_ms, {"gather_ms": round(gather_ms, 4), "gather_bytes": gather_bytes,
                     "gather_gbs": round(gather_bytes / gather_ms / 1e6, 1),
                     "attention_ms": round(statistics.mean(kern_ms), 4),
                     "note": "gather = step time minus the prefix kernel timed alone on the gathered rows"}


def config_entry(kp, name, args):
    """One `configs` entry: the workload timed on this GPU, verified against the oracle,
    with the oracle's time for the whole problem (run in full for the tiny and the
    13622-token workloads, extrapolated from the verified rows otherwise)."""
    rec, prob = measure(kp, name, args, 0, 1, "replicas", args.steps, min_ms=500.0)
    w = prob.w
    if name in ("tiny", "unmasked") and not args.no_cpu_baseline:
        rec["cpu_oracle"] = oracle_full(prob.case, w)
    elif not args.no_cpu_baseline:
        rec["cpu_oracle"] = oracle_extrapolated(prob.case, w)
    rec["scaling"] = "single GPU"
    del prob
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world):
    from key_prefix_masked_b200 import build as kbuild
    if rank == 0 or not os.path.exists(kbuild.LIB_PATH):
        kbuild.build()
    barrier(world)
    import key_prefix_masked_b200 as kp

    w = synth.WORKLOADS[args.workload]
    shard = resolve_shard(args.shard, w) if world > 1 else "single"
    head, prob = measure(kp, args.workload, args, rank, world, shard, args.steps)
    e2e = run_e2e(kp, prob, args, world)
    scaling = SCALING[shard]
    parallelism = PARALLELISM[shard].format(n=world)
    rec = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": scaling, "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,std^2) bf16 q/k/v, NaN in padded key slots)",
        "config": {**head["config"], "parallelism": parallelism},
        "impl": "ours",
        "e2e": e2e,
        "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "step_ms": head["step_ms"],
        "verified_rows": head.get("verified_rows"),
        **({"segments": head["segments"]} if "segments" in head else {}),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(w, prob.case, args.cpu_seconds)
    del prob
    torch.cuda.empty_cache()
    if world == 1 and not args.no_configs:
        rec["configs"] = {}
        for name in CONFIG_SWEEP:
            if name == args.workload:
                continue
            rec["configs"][name] = config_entry(kp, name, args)
    return rec


def run_e2e_pipelined(kp, prob, args, world):
    """Single-pass steps: the public HostPipeline, whose step i+1 copies its inputs in
    while step i computes and step i-1's result is read back (two device buffer sets,
    three streams).  Every step still moves its own inputs and result (this rank's
    shard of them)."""
    from key_prefix_masked_b200.pipeline import HostPipeline
    w = prob.w
    dev = prob.q.device
    hq, hk, hv = (t.cpu().pin_memory() for t in (prob.q, prob.k, prob.v))
    hkv = prob.kv.cpu().pin_memory()
    hout = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hlse = torch.empty(hq.shape[:3], dtype=torch.float32).pin_memory()
    pipe = HostPipeline((w.B, w.H, hq.shape[2], hk.shape[2], w.D), device=dev, scale=prob.scale)
    for _ in range(2):
        pipe.submit(hq, hk, hv, hkv, hout, hlse)
    pipe.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    steps = args.steps
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(pipe.s_h2d)
    for _ in range(steps):
        pipe.submit(hq, hk, hv, hkv, hout, hlse)
    b_.record(pipe.s_d2h)
    pipe.synchronize()
    ms = max_over_ranks(a.elapsed_time(b_), world) / steps
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hkv))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    return {"value": round(prob.flops_job / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "mode": "pipelined: copies of neighbouring steps overlap the kernel (HostPipeline)"}


def run_e2e(kp, prob, args, world):
    """Same metric through the public call with host buffers: every step copies that
    step's inputs (this rank's shard) host->device from pinned memory, runs the step
    (collective included when keys are sharded) and reads the result back."""
    if not prob.splits and not prob.segs:
        return run_e2e_pipelined(kp, prob, args, world)
    names = ("q", "k", "v", "kv")
    host = {n: getattr(prob, n).cpu().pin_memory() for n in names}
    segs = prob.segs
    hseg = (prob.case["seg_start"].cpu().pin_memory(), prob.case["seg_len"].cpu().pin_memory()) if segs else ()
    dseg = (prob.case["seg_start"], prob.case["seg_len"]) if segs else ()
    hout = torch.empty(tuple(prob.out.shape), dtype=torch.bfloat16).pin_memory()
    hlse = torch.empty(tuple(prob.lse.shape), dtype=torch.float32).pin_memory()
    stream = torch.cuda.current_stream()

    def one():
        for n in names:
            getattr(prob, n).copy_(host[n], non_blocking=True)
        for d_, h_ in zip(dseg, hseg):
            d_.copy_(h_, non_blocking=True)
        prob.step()
        hout.copy_(prob.out, non_blocking=True)
        hlse.copy_(prob.lse, non_blocking=True)

    steps = args.steps
    for _ in range(2):
        one()
    torch.cuda.synchronize()
    barrier(world)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b_.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b_), world) / steps
    h2d = sum(t.numel() * t.element_size() for t in list(host.values()) + list(hseg))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    return {"value": round(prob.flops_job / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "mode": "sequential: copy in, compute, copy out per step"}


def _oracle_rows(case, q_rows):
    """The oracle on some query rows (already selected into q_rows) of a workload case."""
    import oracle
    k, v = case["k"].cpu(), case["v"].cpu()
    if "segments" in case:
        return oracle.attn_segments(q_rows, k, v, case["seg_start"].cpu(), case["seg_len"].cpu(), case["scale"])
    return oracle.attn_prefix(q_rows, k, v, case["kv_len_list"], case["scale"])


def verify_rows(case, out, lse, rows_g, rows_l):
    """GPU rows rows_l of (out, lse) against the oracle on query rows rows_g of the case,
    with the parity tolerances (|out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3,
    -inf exactly)."""
    import numpy as np
    q = case["q"][:, :, rows_g].cpu().contiguous()
    t = time.perf_counter()
    ro, rl = _oracle_rows(case, q)
    dt = time.perf_counter() - t
    go = out[:, :, rows_l].float().cpu().double().numpy()
    gl = lse[:, :, rows_l].cpu().double().numpy()
    ok_out = bool((np.abs(go - ro) <= 1e-2 + 1e-2 * np.abs(ro)).all())
    fin = np.isfinite(rl)
    ok_lse = bool(np.array_equal(np.isneginf(gl), np.isneginf(rl)) and
                  (np.abs(gl[fin] - rl[fin]) <= 1e-3).all())
    rows_shown = rows_g if len(rows_g) <= 8 else f"all {len(rows_g)} rows"
    return {"rows": rows_shown, "out_ok": ok_out, "lse_ok": ok_lse,
            "max_abs_err_out": float(np.abs(go - ro).max()),
            "max_abs_err_lse": float(np.abs(gl[fin] - rl[fin]).max()) if fin.any() else 0.0,
            "oracle_s": round(dt, 3)}


def traffic_from_profile(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and workload."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    # null once the kernel has changed since the counters were taken
    return rec.get("dram_bytes_per_launch") if rec.get("current", True) else None


# ------------------------------------------------------------------ CPU baseline / reference arm
def _oracle_sample(w, case, n_rows, seed=0):
    g = torch.Generator().manual_seed(1234 + seed)
    rows = sorted(set(torch.randint(0, w.Tq, (n_rows,), generator=g).tolist()))
    q = case["q"][:, :, rows].cpu().contiguous()
    t = time.perf_counter()
    _oracle_rows(case, q)
    dt = time.perf_counter() - t
    flops = float(sum(4.0 * w.H * len(rows) * n * w.D for n in case["kv_len_list"]))
    return rows, dt, flops


def _rows_for(w, case, seconds: float) -> int:
    """Number of query rows whose oracle sample takes about `seconds` on the host cores.
    Small samples run below the cores' parallel efficiency, so the estimate is grown
    geometrically before it is scaled."""
    _oracle_sample(w, case, 1, seed=7)          # first call: thread pool start-up, page faults
    n = 4
    _, dt, _ = _oracle_sample(w, case, n, seed=8)
    while dt < 0.25 * seconds and n < w.Tq:
        n = min(w.Tq, n * 4)
        _, dt, _ = _oracle_sample(w, case, n, seed=9)
    return max(1, min(w.Tq, int(n * seconds / max(dt, 1e-4))))


def host_oracle():
    """The oracle module, set to run on every host core this process may use.  (torchrun
    starts each rank with OMP_NUM_THREADS=1; the oracle is timed on rank 0 alone, so it
    takes the cores back.)"""
    import oracle
    oracle.set_num_threads(len(os.sched_getaffinity(0)))
    return oracle


def oracle_full(case, w):
    """The oracle over the whole problem (every query row), timed on the host cores."""
    oracle = host_oracle()
    t = time.perf_counter()
    _oracle_rows(case, case["q"].cpu())
    dt = time.perf_counter() - t
    flops = workload_flops(w, case["kv_len_list"])
    return {"kind": "oracle, full problem", "seconds": round(dt, 3), "cores": oracle.num_threads(),
            "value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s"}


def oracle_extrapolated(case, w, n_rows=32):
    """The oracle on n_rows random query rows (all their valid keys), and the whole
    problem's time extrapolated linearly in rows x kv_len."""
    oracle = host_oracle()
    rows, dt, flops = _oracle_sample(w, case, n_rows, seed=3)
    full = workload_flops(w, case["kv_len_list"])
    return {"kind": "oracle, sampled rows", "sample": f"{len(rows)} random query rows x {w.H} heads",
            "seconds": round(dt, 3), "cores": oracle.num_threads(), "value": round(flops / dt / 1e12, 6),
            "unit": "TFLOP/s", "extrapolated_full_s": round(dt * full / flops, 1)}


def cpu_baseline(w, case, target_s: float):
    oracle = host_oracle()
    cores = oracle.num_threads()
    rows, dt, flops = _oracle_sample(w, case, _rows_for(w, case, target_s), seed=1)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(rows)} random query rows x {w.H} heads of the {w.name} workload "
                      f"(all their valid keys), fp64, {dt:.1f} s; throughput extrapolates "
                      f"linearly in rows x kv_len",
            "seconds": round(dt, 2),
            "extrapolated_full_s": round(dt * workload_flops(w, case["kv_len_list"]) / flops, 1)}


def run_reference(args, rank, world):
    """The oracle timed on the host cores: each step evaluates a bounded sample of query
    rows of the same workload."""
    oracle = host_oracle()
    w = synth.WORKLOADS[args.workload]
    shard = resolve_shard(args.shard, w) if world > 1 else "single"
    case = synth.make_inputs(w, device="cpu", seed=args.seed)
    cores = oracle.num_threads()
    per_step_rows = _rows_for(w, case, args.cpu_seconds / max(args.steps + args.warmup, 1))
    for i in range(args.warmup):
        _oracle_sample(w, case, per_step_rows, seed=100 + i)
    times, flops_total = [], 0.0
    for i in range(args.steps):
        _, dt, fl = _oracle_sample(w, case, per_step_rows, seed=200 + i)
        times.append(dt)
        flops_total += fl
    tot = sum(times)
    value = flops_total / tot / 1e12
    return {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": SCALING[shard], "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**workload_config(w, case, args, world, shard, needs_flush(w, 0, world, shard)),
                   "parallelism": PARALLELISM[shard].format(n=world)},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{per_step_rows} random query rows x {w.H} heads per step, "
                                   f"all valid keys, fp64 on host cores"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="icl", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-verify", dest="verify", action="store_false")
    ap.add_argument("--split-mode", default="separate", choices=["separate", "fused"],
                    help="split-KV workloads: the LSE combine as a second launch (faster on B200), "
                         "or fused into the split launch")
    ap.add_argument("--shard", default="auto", choices=["auto", "queries", "keys", "replicas"],
                    help="several GPUs: shard the workload's query rows (no exchange), its key slots "
                         "(all-gather of partials + exact combine), or run replicas; auto = keys for "
                         "split-KV workloads, queries otherwise")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the headline workload (skip the per-config sweep)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        # The oracle runs on rank 0's host cores only; other ranks exit without work.
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args, 0, int(os.environ.get("WORLD_SIZE", "1")))), flush=True)
        return 0
    rank, world, _ = dist_setup(args.gpus)
    try:
        rec = run_ours(args, rank, world)
        if rank == 0:
            print(json.dumps(rec), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
