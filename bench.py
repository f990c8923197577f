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

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of the
workload (weak scaling, no collective on the data path); the step time is the max over
ranks and the value counts the work of all ranks.

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


def whole_job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Throughput of the whole job: every rank's work over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


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
def run_ours(args, rank, world):
    from key_prefix_masked_b200 import build as kbuild
    if rank == 0 or not os.path.exists(kbuild.LIB_PATH):
        kbuild.build()
    barrier(world)
    import key_prefix_masked_b200 as kp

    w = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    case = synth.make_inputs(w, device=dev, seed=args.seed)
    q, k, v, kv = case["q"], case["k"], case["v"], case["kv_len"]
    scale = case["scale"]
    flops = workload_flops(w, case["kv_len_list"])
    splits = w.num_splits if w.num_splits > 1 else 0
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Tq), dtype=torch.float32, device=dev)
    segs = w.segments is not None
    seg_ws = (torch.empty(int(kp.lib().attn_segments_workspace_bytes(w.B, w.H, w.Tk, w.D)), dtype=torch.uint8,
                          device=dev) if segs else None)
    fused = bool(splits) and args.split_mode == "fused"
    ws = kp.fused_workspace(splits, w.B, w.H, w.Tq, w.D, dev) if fused else None
    parts = ((torch.empty((splits, w.B, w.H, w.Tq, w.D), dtype=torch.float32, device=dev),
              torch.empty((splits, w.B, w.H, w.Tq), dtype=torch.float32, device=dev))
             if splits and not fused else None)
    stream = torch.cuda.current_stream(dev)
    k_ev = []   # separate split mode: events around the split launch (the dominant kernel)

    def step(qq, kk, vv, kvl, timed=False):
        if segs:
            kp.attn_prefix_fwd_segments(qq, kk, vv, case["seg_start"], case["seg_len"], scale,
                                        workspace=seg_ws, out=out, lse=lse)
        elif fused:
            kp.attn_prefix_fwd_split_fused(qq, kk, vv, kvl, splits, scale, workspace=ws, out=out, lse=lse)
        elif splits:
            if timed:
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            kp.attn_prefix_fwd_split(qq, kk, vv, kvl, splits, scale, *parts)
            if timed:
                b_.record(stream)
                k_ev.append((a, b_))
            kp.attn_lse_combine(parts[0], parts[1], out=out, lse=lse)
        else:
            kp.attn_prefix_fwd(qq, kk, vv, kvl, scale, out=out, lse=lse)

    launches_per_step = 2 if ((splits and not fused) or segs) else 1
    for _ in range(args.warmup):
        step(q, k, v, kv)
    torch.cuda.synchronize()
    st = kp.device_status()
    if st != kp.ATTN_OK:
        raise RuntimeError(f"device status after warm-up: {kp.status_string(st)}")

    # ---- device-timed region: inputs resident in HBM
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES else None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockMonitor(torch.cuda.current_device()) as mon:
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()   # evict the inputs from L2 (outside the step's events)
            ev[i][0].record(stream)
            step(q, k, v, kv, timed=True)
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    clocks = mon.summary()
    st = kp.device_status()
    if st != kp.ATTN_OK:
        raise RuntimeError(f"device status after timing: {kp.status_string(st)}")
    step_ms = [a.elapsed_time(b_) for a, b_ in ev]
    total_ms = sum(step_ms) if flush is not None else t0.elapsed_time(t1)
    kern_ms = [a.elapsed_time(b_) for a, b_ in k_ev] if k_ev else step_ms
    seg_info = None
    if segs:
        # the dominant kernel alone: the prefix kernel on the rows the gather left in the
        # workspace (same launch as inside the step); the rest of the step is the gather
        kvb = (w.B * w.H * w.Tk * w.D * 2 + 255) // 256 * 256
        kg = seg_ws[:w.B * w.H * w.Tk * w.D * 2].view(torch.bfloat16).view(w.B, w.H, w.Tk, w.D)
        vg = seg_ws[kvb:kvb + w.B * w.H * w.Tk * w.D * 2].view(torch.bfloat16).view(w.B, w.H, w.Tk, w.D)
        kvg = seg_ws[2 * kvb:2 * kvb + 4 * w.B].view(torch.int32)
        a_ev = []
        for _ in range(args.steps):
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            kp.attn_prefix_fwd(q, kg, vg, kvg, scale, out=out, lse=lse)
            b_.record(stream)
            a_ev.append((a, b_))
        torch.cuda.synchronize()
        kern_ms = [a.elapsed_time(b_) for a, b_ in a_ev]
        gather_ms = max(statistics.mean(step_ms) - statistics.mean(kern_ms), 1e-6)
        gather_bytes = 2 * 2 * sum(case["kv_len_list"]) * w.H * w.D * 2   # K and V rows, read + write
        seg_info = {"gather_ms": round(gather_ms, 4), "gather_bytes": gather_bytes,
                    "gather_gbs": round(gather_bytes / gather_ms / 1e6, 1),
                    "attention_ms": round(statistics.mean(kern_ms), 4),
                    "note": "gather = step time minus the prefix kernel timed alone on the gathered rows"}
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(flops, world, ms_per_step)

    # ---- end-to-end: pinned host buffers, copies inside the timed region
    e2e = run_e2e(kp, w, case, scale, splits, fused, args, world)

    # ---- quick correctness check on a few sampled rows (outside every timed region)
    verified = None
    if args.verify and rank == 0:
        verified = verify_rows(case, out, lse, w)

    peaks, peaks_src = load_peaks()
    kern_avg_ms = statistics.mean(kern_ms)
    achieved = flops / (kern_avg_ms * 1e-3) / 1e12
    # the dominant kernel: head dims 128 and 256 run on CTA pairs, 32 and 64 on single CTAs
    pair = w.D in (128, 256)
    kernel_tag = "attn_fwd_pair" if w.D == 256 else (f"attn_fwd_pair_d{w.D}" if pair else f"attn_fwd_d{w.D}")
    kernel_name = (f"attn_fwd_pair_kernel<{w.D},{int(bool(splits))}>" if pair
                   else f"attn_fwd_kernel<{w.D},{int(bool(splits))}>")
    # A kernel that runs long enough to draw the power cap is compared with the sustained
    # cuBLAS figure; a short one (the D=64 shapes, ~1 ms steps) with the burst figure.
    long_run = total_ms >= 1000.0 or "sw_power_cap" in (clocks.get("reasons") or [])
    peak_key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    roofline = {
        "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
        "frac": round(achieved / peak, 4),
        "peak_source": f"{peaks_src} {peak_key} " + ("(kernel under the power cap in a long back-to-back loop)"
                                                      if long_run else "(short kernel, no power cap: burst figure)"),
        "frac_of_nominal_2250": round(achieved / NOMINAL_BF16_TFLOPS, 4),
        "traffic": traffic_from_profile(args.workload, kernel_tag),
        "kernel": kernel_name,
    }
    rec = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,std^2) bf16 q/k/v, NaN in padded key slots)",
        "config": {**w.describe(), "kv_len": case["kv_len_list"] if len(case["kv_len_list"]) <= 8
                   else "ragged", "scale": scale, "flops_per_step": flops,
                   "l2": ("inputs larger than the 126 MB L2; no flush" if flush is None else
                          "inputs smaller than 2x L2: a 252 MB buffer written before each step, "
                          "outside the step events; value from per-step events"),
                   "parallelism": f"replicas x{world}",
                   **({"split_mode": args.split_mode} if splits else {})},
        "impl": "ours",
        "e2e": e2e,
        "roofline": roofline,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "step_ms": {"min": round(min(step_ms), 4), "median": round(statistics.median(step_ms), 4),
                    "max": round(max(step_ms), 4)},
        "verified_rows": verified,
        **({"segments": seg_info} if seg_info else {}),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(w, case, args.cpu_seconds)
    return rec


def run_e2e_pipelined(kp, w, case, scale, args, world):
    """Single-pass workloads: the public HostPipeline, whose step i+1 copies its inputs
    in while step i computes and step i-1's result is read back (two device buffer
    sets, three streams).  Every step still moves its own inputs and result."""
    from key_prefix_masked_b200.pipeline import HostPipeline
    dev = case["q"].device
    hq = case["q"].cpu().pin_memory()
    hk = case["k"].cpu().pin_memory()
    hv = case["v"].cpu().pin_memory()
    hkv = case["kv_len"].cpu().pin_memory()
    hout = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hlse = torch.empty((w.B, w.H, w.Tq), dtype=torch.float32).pin_memory()
    pipe = HostPipeline((w.B, w.H, w.Tq, w.Tk, w.D), device=dev, scale=scale)
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
    flops = workload_flops(w, case["kv_len_list"])
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hkv))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "mode": "pipelined: copies of neighbouring steps overlap the kernel (HostPipeline)"}


def run_e2e(kp, w, case, scale, splits, fused, args, world):
    """Same metric through the public call with host buffers: every step copies that
    step's inputs host->device from pinned memory and reads the result back."""
    if not splits and "segments" not in case:
        return run_e2e_pipelined(kp, w, case, scale, args, world)
    dev = case["q"].device
    hq = case["q"].cpu().pin_memory()
    hk = case["k"].cpu().pin_memory()
    hv = case["v"].cpu().pin_memory()
    hkv = case["kv_len"].cpu().pin_memory()
    segs = "segments" in case
    hseg = (case["seg_start"].cpu().pin_memory(), case["seg_len"].cpu().pin_memory()) if segs else ()
    dseg = tuple(torch.empty_like(case[n]) for n in ("seg_start", "seg_len")) if segs else ()
    seg_ws = (torch.empty(int(kp.lib().attn_segments_workspace_bytes(w.B, w.H, w.Tk, w.D)), dtype=torch.uint8,
                          device=dev) if segs else None)
    hout = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hlse = torch.empty((w.B, w.H, w.Tq), dtype=torch.float32).pin_memory()
    dq, dk, dv, dkv = (torch.empty_like(case[n]) for n in ("q", "k", "v", "kv_len"))
    dout = torch.empty_like(case["q"])
    dlse = torch.empty((w.B, w.H, w.Tq), dtype=torch.float32, device=dev)
    ws = kp.fused_workspace(splits, w.B, w.H, w.Tq, w.D, dev) if fused else None
    parts = ((torch.empty((splits, w.B, w.H, w.Tq, w.D), dtype=torch.float32, device=dev),
              torch.empty((splits, w.B, w.H, w.Tq), dtype=torch.float32, device=dev))
             if splits and not fused else None)
    stream = torch.cuda.current_stream(dev)

    def one():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dkv.copy_(hkv, non_blocking=True)
        for d_, h_ in zip(dseg, hseg):
            d_.copy_(h_, non_blocking=True)
        if segs:
            kp.attn_prefix_fwd_segments(dq, dk, dv, dseg[0], dseg[1], scale, workspace=seg_ws, out=dout, lse=dlse)
        elif fused:
            kp.attn_prefix_fwd_split_fused(dq, dk, dv, dkv, splits, scale, workspace=ws, out=dout, lse=dlse)
        elif splits:
            kp.attn_prefix_fwd_split(dq, dk, dv, dkv, splits, scale, *parts)
            kp.attn_lse_combine(parts[0], parts[1], out=dout, lse=dlse)
        else:
            kp.attn_prefix_fwd(dq, dk, dv, dkv, scale, out=dout, lse=dlse)
        hout.copy_(dout, non_blocking=True)
        hlse.copy_(dlse, non_blocking=True)

    steps = max(1, min(args.steps, 5))
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
    flops = workload_flops(w, case["kv_len_list"])
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hkv) + tuple(hseg))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
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


def verify_rows(case, out, lse, w):
    import numpy as np
    rows = sorted({0, 1, min(127, w.Tq - 1), min(128, w.Tq - 1), w.Tq // 2, w.Tq - 1})
    q = case["q"][:, :, rows].cpu().contiguous()
    ro, rl = _oracle_rows(case, q)
    go = out[:, :, rows].float().cpu().double().numpy()
    gl = lse[:, :, rows].cpu().double().numpy()
    ok_out = bool((np.abs(go - ro) <= 1e-2 + 1e-2 * np.abs(ro)).all())
    fin = np.isfinite(rl)
    ok_lse = bool(np.array_equal(np.isneginf(gl), np.isneginf(rl)) and
                  (np.abs(gl[fin] - rl[fin]) <= 1e-3).all())
    return {"rows": rows, "out_ok": ok_out, "lse_ok": ok_lse,
            "max_abs_err_out": float(np.abs(go - ro).max())}


def traffic_from_profile(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and workload."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}_traffic.json")
    try:
        with open(path) as f:
            return json.load(f).get("dram_bytes_per_launch")
    except (OSError, ValueError):
        return None


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


def cpu_baseline(w, case, target_s: float):
    import oracle
    cores = oracle.num_threads()
    rows, dt, flops = _oracle_sample(w, case, _rows_for(w, case, target_s), seed=1)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{len(rows)} random query rows x {w.H} heads of the {w.name} workload "
                      f"(all their valid keys), fp64, {dt:.1f} s; throughput extrapolates "
                      f"linearly in rows x kv_len",
            "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    """The oracle timed on the host cores: each step evaluates a bounded sample of query
    rows of the same workload."""
    import oracle
    w = synth.WORKLOADS[args.workload]
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
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {**w.describe(), "kv_len": case["kv_len_list"]
                                        if len(case["kv_len_list"]) <= 8 else "ragged"},
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
