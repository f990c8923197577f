"""GPU parity of the multi-range key mask (attn_prefix_fwd_segments).

Each batch element attends to the keys of its segments: the gathered-shards K/V of
"Add sequence-parallel multi-GPU inference ...", section "Sequence-parallel inference".
Three checks. The output is compared with the fp64 oracle. It is compared bit for bit
with attn_prefix_fwd on the same rows gathered by torch indexing. It must not change
with the content of the holes between the segments. The clamping rules and their
device flag are checked against the oracle, which applies the same rules.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import assert_lse_close, assert_out_close, bits_equal

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kp():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    torch.cuda.init()
    assert kp.device_status() == kp.ATTN_OK
    return kp


def _gathered_prefix(kp, c):
    """attn_prefix_fwd on the segments' rows gathered by torch indexing."""
    B, Tk = c["k"].shape[0], c["k"].shape[2]
    kg, vg = torch.zeros_like(c["k"]), torch.zeros_like(c["v"])
    lens = []
    for b, segs in enumerate(c["segments"]):
        idx = [j for st, ln in segs for j in range(max(st, 0), min(st + max(ln, 0), Tk))][:Tk]
        if idx:
            it = torch.tensor(idx, device=c["k"].device)
            kg[b, :, :len(idx)] = c["k"][b][:, it]
            vg[b, :, :len(idx)] = c["v"][b][:, it]
        lens.append(len(idx))
    kv = torch.tensor(lens, dtype=torch.int32, device=c["k"].device)
    return kp.attn_prefix_fwd(c["q"], kg, vg, kv, c["scale"])


SEGS = [
    # B = 2: shard-like ranges with holes, a single-key segment, an empty one, a range
    # ending at the buffer end, segments shorter than one 128-key tile
    [[(0, 300), (384, 129), (700, 1)], [(5, 0), (100, 127), (811, 189)]],
    [[(999, 1), (0, 64), (200, 600)], [(0, 0), (0, 0), (0, 0)]],
]


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("segs", SEGS, ids=["shards", "reversed_and_empty"])
def test_segments_against_oracle_and_gathered_prefix(kp, D, segs):
    B, H, Tq, Tk = 2, 2, 260, 1000
    c = synth.random_segments_case(B, H, Tq, Tk, D, segs, seed=80 + D, device="cuda")
    out, lse = kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"], c["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    ref_out, ref_lse = _gathered_prefix(kp, c)
    assert bits_equal(out, ref_out) and bits_equal(lse, ref_lse), "differs from the prefix kernel on gathered rows"
    host = {n: c[n].cpu() for n in ("q", "k", "v", "seg_start", "seg_len")}
    o_ref, l_ref = oracle.attn_segments(host["q"], host["k"], host["v"], host["seg_start"], host["seg_len"],
                                        c["scale"])
    assert_out_close(out, o_ref)
    assert_lse_close(lse, l_ref)


@pytest.mark.parametrize("D", [64, 256])
def test_hole_content_never_matters(kp, D):
    segs = [[(10, 200), (400, 90), (600, 37)]]
    ref = None
    for hole in (float("nan"), float("inf"), 0.0, -3.0e38):
        c = synth.random_segments_case(1, 2, 140, 700, D, segs, seed=90, device="cuda", hole=hole)
        out, lse = kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"])
        torch.cuda.synchronize()
        if ref is None:
            ref = (out, lse)
            assert torch.isfinite(out.float()).all()
        assert bits_equal(out, ref[0]) and bits_equal(lse, ref[1])


def test_clamped_segments_are_flagged_and_follow_the_oracle(kp):
    B, H, Tq, Tk, D = 1, 2, 130, 300, 64
    segs = [[(-20, 50), (280, 100), (100, -5), (0, 300)]]   # before 0, past Tk, negative, cut
    c = synth.random_segments_case(B, H, Tq, Tk, D, segs, seed=91, device="cuda")
    out, lse = kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_ERR_KVLEN_RANGE
    assert kp.device_status() == kp.ATTN_OK   # the flag is cleared by the read
    host = {n: c[n].cpu() for n in ("q", "k", "v", "seg_start", "seg_len")}
    o_ref, l_ref = oracle.attn_segments(host["q"], host["k"], host["v"], host["seg_start"], host["seg_len"],
                                        c["scale"])
    assert_out_close(out, o_ref)
    assert_lse_close(lse, l_ref)


def test_in_range_segments_raise_no_flag(kp):
    segs = [[(0, 0), (300, 0), (299, 1), (0, 299)]]   # empty segments anywhere are fine
    c = synth.random_segments_case(1, 1, 64, 300, 32, segs, seed=92, device="cuda")
    kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK


def test_many_segments(kp):
    """1000 segments of mixed lengths per element (the block-wide scan over many runs)."""
    g = torch.Generator().manual_seed(93)
    B, H, Tq, Tk, D = 2, 1, 200, 20000, 64
    segs = []
    for b in range(B):
        starts = torch.randint(0, Tk, (1000,), generator=g).tolist()
        lens = torch.randint(0, 12, (1000,), generator=g).tolist()
        segs.append([(s, min(n, Tk - s)) for s, n in zip(starts, lens)])
    c = synth.random_segments_case(B, H, Tq, Tk, D, segs, seed=94, device="cuda")
    out, lse = kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    ref_out, ref_lse = _gathered_prefix(kp, c)
    assert bits_equal(out, ref_out) and bits_equal(lse, ref_lse)
    rows = list(range(0, Tq, 7))
    host = {n: c[n].cpu() for n in ("q", "k", "v", "seg_start", "seg_len")}
    o_ref, l_ref = oracle.attn_segments(host["q"], host["k"], host["v"], host["seg_start"], host["seg_len"],
                                        c["scale"], rows=rows)
    assert_out_close(out[:, :, rows], o_ref)
    assert_lse_close(lse[:, :, rows], l_ref)


def test_workload_gathered(kp):
    """The icl shape over 4 gathered shards (100000 valid keys in 100864 slots, NaN
    holes): sampled rows against the oracle, and bit-exact against the prefix kernel
    on the contiguous icl-like buffer of the same keys."""
    w = synth.WORKLOADS["gathered"]
    c = synth.make_inputs(w, device="cuda", seed=0)
    out, lse = kp.attn_prefix_fwd_segments(c["q"], c["k"], c["v"], c["seg_start"], c["seg_len"], c["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    ref_out, ref_lse = _gathered_prefix(kp, c)
    assert bits_equal(out, ref_out) and bits_equal(lse, ref_lse)
    del ref_out, ref_lse
    rows = synth.sample_rows(w.Tq, n_random=8, seed=0)
    host = {n: c[n].cpu() for n in ("q", "k", "v", "seg_start", "seg_len")}
    o_ref, l_ref = oracle.attn_segments(host["q"], host["k"], host["v"], host["seg_start"], host["seg_len"],
                                        c["scale"], rows=rows)
    assert_out_close(out[:, :, rows], o_ref)
    assert_lse_close(lse[:, :, rows], l_ref)
