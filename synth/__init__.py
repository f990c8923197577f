"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no attention arithmetic: it only draws tensors.  Both the CUDA path
(tests, benchmark) and the fp64 oracle consume what it produces, so it is the one
piece the two sides share.

Workloads (the shapes the pages talk about; no dataset is read):
  tiny      B=2 H=2 D=32 Tq=64 Tk=96, kv_len={40,96}, N(0,1), padded K/V slots NaN
  unmasked  B=1 H=12 D=64 N=13622 (14 views x 973 tokens), kv_len=N, N(0,1)
            ("Broadcast SDPA attn_mask ...", section "Why", multi-view token counts)
  icl       B=1 H=8 D=256, 100000 valid context keys in a 100352-row buffer, Tq=110000
            (context + test rows), N(0,0.5^2), padded slots NaN
            ("Rewrite prefix key-padding masks ...", section "Measured";
             "Add sequence-parallel ...", ICL self-attention and head dim 256)
  ragged    B=8 H=8 D=256 Tq=Tk=32768, kv_len[0..6] uniform in [1,32768], kv_len[7]=0,
            N(0,1), padded slots NaN ("Rewrite prefix ...", ragged packed batches)
  splitkv   B=1 H=8 D=256 Tk=1000000 keys, Tq=1024, N(0,0.5^2), 64 key chunks
            ("Add sequence-parallel ...", inducing attention over a huge context)
  gathered  the icl shape with its 100000 context keys gathered from 4 shards, each
            padded to 25216 slots (Tk = 100864); valid keys are one range per shard,
            padded slots NaN ("Add sequence-parallel ...", ICL self-attention over
            gathered K/V with padded key slots masked)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    Tq: int
    Tk: int
    kv_len: Optional[tuple]      # None -> drawn (ragged) or full
    std: float
    pad_nan: bool
    num_splits: int = 1
    ragged_seed_draw: bool = False
    segments: Optional[tuple] = None   # per batch element, ((start, len), ...): multi-range keys

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "D": self.D,
                "Tq": self.Tq, "Tk": self.Tk, "num_splits": self.num_splits}


WORKLOADS = {
    "tiny": Workload("tiny", 2, 2, 32, 64, 96, (40, 96), 1.0, True),
    "unmasked": Workload("unmasked", 1, 12, 64, 13622, 13622, (13622,), 1.0, False),
    "unmasked_8v": Workload("unmasked_8v", 1, 12, 64, 7784, 7784, (7784,), 1.0, False),
    "unmasked_32v": Workload("unmasked_32v", 1, 12, 64, 31136, 31136, (31136,), 1.0, False),
    "icl": Workload("icl", 1, 8, 256, 110000, 100352, (100000,), 0.5, True),
    "ragged": Workload("ragged", 8, 8, 256, 32768, 32768, None, 1.0, True,
                       ragged_seed_draw=True),
    "splitkv": Workload("splitkv", 1, 8, 256, 1024, 1000000, (1000000,), 0.5, False,
                        num_splits=64),
    # a reduced icl shape for profiler captures: same head dim, padding and value
    # distribution, inputs (161 MB) still larger than the L2
    "icl_profile": Workload("icl_profile", 1, 8, 256, 8192, 16512, (16384,), 0.5, True),
    # head dim 128 (beyond the pages' 64 and 256): the unmasked shape with D=128, and a
    # prefix-masked one with NaN padding
    "gathered": Workload("gathered", 1, 8, 256, 110000, 4 * 25216, (100000,), 0.5, True,
                         segments=(((0, 25000), (25216, 24800), (50432, 25200), (75648, 25000)),)),
    "unmasked_d128": Workload("unmasked_d128", 1, 12, 128, 13622, 13622, (13622,), 1.0, False),
    "prefix_d128": Workload("prefix_d128", 2, 16, 128, 16384, 16512, (16384, 9001), 1.0, True),
}


def ragged_kv_len(B: int, Tk: int, seed: int = 0) -> list:
    """kv_len[0..B-2] uniform in [1, Tk] from a CPU generator seeded with `seed`;
    the last element is empty (kv_len = 0)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    lens = torch.randint(1, Tk + 1, (B - 1,), generator=g).tolist()
    return [int(x) for x in lens] + [0]


def kv_len_for(w: Workload, seed: int = 0) -> list:
    if w.ragged_seed_draw:
        return ragged_kv_len(w.B, w.Tk, seed)
    assert w.kv_len is not None
    return list(w.kv_len)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def normal_bf16(shape: Sequence[int], std: float, gen: torch.Generator,
                device) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from `gen`, rounded to bf16."""
    x = torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def fill_padding(k: torch.Tensor, v: torch.Tensor, kv_len: Sequence[int],
                 value: float = float("nan")) -> None:
    """Write `value` into every K/V slot at or beyond kv_len[b] (in place)."""
    for b, n in enumerate(kv_len):
        if n < k.shape[2]:
            k[b, :, n:, :] = value
            v[b, :, n:, :] = value


def segment_mask(segments, B: int, Tk: int) -> torch.Tensor:
    """[B, Tk] bool: key slot inside one of the batch element's (start, len) ranges."""
    m = torch.zeros((B, Tk), dtype=torch.bool)
    for b in range(B):
        for st, ln in segments[b]:
            lo, hi = max(int(st), 0), min(int(st) + max(int(ln), 0), Tk)
            if hi > lo:
                m[b, lo:hi] = True
    return m


def fill_holes(k: torch.Tensor, v: torch.Tensor, segments, value: float = float("nan")) -> None:
    """Write `value` into every K/V slot outside the segments (in place)."""
    holes = ~segment_mask(segments, k.shape[0], k.shape[2]).to(k.device)
    for b in range(k.shape[0]):
        k[b][:, holes[b]] = value
        v[b][:, holes[b]] = value


def segment_tensors(segments, device) -> tuple:
    """seg_start, seg_len as int32 [B, S] tensors on `device`."""
    st = torch.tensor([[int(a) for a, _ in segs] for segs in segments], dtype=torch.int32, device=device)
    ln = torch.tensor([[int(n) for _, n in segs] for segs in segments], dtype=torch.int32, device=device)
    return st, ln


def random_segments_case(B: int, H: int, Tq: int, Tk: int, D: int, segments, seed: int = 0,
                         std: float = 1.0, device="cpu", hole=float("nan")) -> dict:
    """Seeded q/k/v with key slots outside the segments set to `hole`, plus the
    segment tensors (int32 [B, S]) and lists."""
    w = Workload("custom_segments", B, H, D, Tq, Tk, (Tk,) * B, std, False)
    c = make_inputs(w, device=device, seed=seed)
    fill_holes(c["k"], c["v"], segments, hole)
    st, ln = segment_tensors(segments, device)
    c.update({"seg_start": st, "seg_len": ln, "segments": segments})
    return c


def make_inputs(w: Workload, device="cpu", seed: int = 0, pad_value=None) -> dict:
    """Seeded q, k, v (bf16, [B,H,T,D]) and kv_len (int32 [B]) for a workload.

    The generator lives on `device`, so CPU and CUDA draws differ; each call's tensors
    are what both sides of a comparison consume.  pad_value overrides the NaN padding.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    lens = kv_len_for(w, seed)
    q = normal_bf16((w.B, w.H, w.Tq, w.D), w.std, gen, dev)
    k = normal_bf16((w.B, w.H, w.Tk, w.D), w.std, gen, dev)
    v = normal_bf16((w.B, w.H, w.Tk, w.D), w.std, gen, dev)
    pv = pad_value if pad_value is not None else (float("nan") if w.pad_nan else None)
    extra = {}
    if w.segments is not None:
        # multi-range keys: kv_len is the count of valid keys per element; the holes
        # between the ranges are the padding
        if pv is not None:
            fill_holes(k, v, w.segments, pv)
        st, ln = segment_tensors(w.segments, dev)
        extra = {"seg_start": st, "seg_len": ln, "segments": w.segments}
    elif pv is not None:
        fill_padding(k, v, lens, pv)
    kv = torch.tensor(lens, dtype=torch.int32, device=dev)
    return {"q": q, "k": k, "v": v, "kv_len": kv, "kv_len_list": lens,
            "scale": default_scale(w.D), "workload": w, **extra}


def random_case(B: int, H: int, Tq: int, Tk: int, D: int, kv_len: Sequence[int],
                seed: int = 0, std: float = 1.0, device="cpu", pad_value=float("nan")):
    """Ad-hoc seeded case for parity sweeps (same recipe as the named workloads)."""
    w = Workload("custom", B, H, D, Tq, Tk, tuple(kv_len), std, pad_value is not None)
    return make_inputs(w, device=device, seed=seed,
                       pad_value=pad_value)


def sample_rows(Tq: int, n_random: int = 48, seed: int = 0) -> list:
    """Query rows checked on big workloads: 0-7, 127/128/129, the last 8 and n_random
    seeded random rows (sorted, unique, all < Tq)."""
    g = torch.Generator(device="cpu").manual_seed(seed + 7919)
    rows = set(range(min(8, Tq)))
    rows.update(r for r in (127, 128, 129) if r < Tq)
    rows.update(range(max(0, Tq - 8), Tq))
    if n_random > 0:
        rows.update(torch.randint(0, Tq, (n_random,), generator=g).tolist())
    return sorted(int(r) for r in rows)
