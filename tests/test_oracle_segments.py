"""Pins of the oracle's multi-range key mask (oracle.attn_segments), on the CPU.

The segments case is the gathered-shards K/V of "Add sequence-parallel multi-GPU
inference ...", section "Sequence-parallel inference": each shard's keys are gathered
with padded slots, so each batch element's valid keys are one range per shard. The
pins do not retype the oracle's formula. They use torch SDPA with the equivalent
boolean key mask, the prefix oracle on a buffer compacted with numpy, invariants
(segment order, hole contents) and the clamping rules stated in the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _holey_case(B, H, Tq, Tk, D, segs, seed, hole=float("nan")):
    """Random q/k/v with every key row outside the segments set to `hole`."""
    c = synth.random_case(B, H, Tq, Tk, D, (Tk,) * B, seed=seed)
    k, v = c["k"].clone(), c["v"].clone()
    for b in range(B):
        valid = np.zeros(Tk, dtype=bool)
        for st, ln in segs[b]:
            lo, hi = max(st, 0), min(st + max(ln, 0), Tk)
            valid[lo:hi] = True
        holes = torch.from_numpy(~valid)
        k[b][:, holes] = hole
        v[b][:, holes] = hole
    starts = [[s for s, _ in segs[b]] for b in range(B)]
    lens = [[n for _, n in segs[b]] for b in range(B)]
    return c["q"], k, v, starts, lens


def _sdpa_reference(q, k, v, valid_mask, scale):
    """torch SDPA (CPU, float64) with a [B,1,1,Tk] boolean key mask; torch.logsumexp."""
    qd, kd, vd = (t.to(torch.float64) for t in (q, k, v))
    m4 = torch.from_numpy(valid_mask)[:, None, None, :]
    # masked slots may hold NaN: give SDPA finite values there (they are masked anyway)
    kd = torch.where(m4.transpose(-1, -2), kd, torch.zeros_like(kd))
    vd = torch.where(m4.transpose(-1, -2), vd, torch.zeros_like(vd))
    out = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=m4, scale=scale)
    scores = torch.einsum("bhid,bhjd->bhij", qd, kd) * scale
    lse = torch.logsumexp(scores.masked_fill(~m4, float("-inf")), dim=-1)
    return out.numpy(), lse.numpy()


SEGS = [
    [[(0, 30), (64, 20), (128, 50)], [(10, 1), (40, 60), (150, 28)]],
    [[(5, 120), (130, 7), (170, 0)], [(0, 0), (0, 0), (100, 78)]],
]


@pytest.mark.parametrize("segs", SEGS)
def test_segments_match_library_sdpa(segs):
    B, H, Tq, Tk, D = 2, 2, 11, 178, 32
    q, k, v, st, ln = _holey_case(B, H, Tq, Tk, D, segs, seed=70)
    scale = 1.0 / math.sqrt(D)
    valid = np.zeros((B, Tk), dtype=bool)
    for b in range(B):
        for s, n in segs[b]:
            valid[b, s:s + n] = True
    out, lse = oracle.attn_segments(q, k, v, st, ln, scale)
    ref_out, ref_lse = _sdpa_reference(q, k, v, valid, scale)
    np.testing.assert_allclose(out, ref_out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    assert np.isfinite(out).all()


def test_pin_detects_plausible_mistakes():
    """The SDPA pin moves far beyond its tolerance for a segment one key too long or
    shifted by one, or a segment dropped."""
    B, H, Tq, Tk, D = 1, 2, 7, 90, 16
    segs = [[(3, 20), (40, 30)]]
    q, k, v, st, ln = _holey_case(B, H, Tq, Tk, D, segs, seed=71, hole=0.5)
    valid = np.zeros((B, Tk), dtype=bool)
    valid[0, 3:23] = valid[0, 40:70] = True
    ref_out, ref_lse = _sdpa_reference(q, k, v, valid, 0.3)
    for bad_st, bad_ln in (([[3, 40]], [[21, 30]]), ([[4, 40]], [[20, 30]]), ([[3, 40]], [[20, 0]])):
        out, lse = oracle.attn_segments(q, k, v, bad_st, bad_ln, 0.3)
        assert np.abs(out - ref_out).max() > 1e-6 or np.abs(lse - ref_lse).max() > 1e-6


def test_one_prefix_segment_equals_prefix_oracle():
    B, H, Tq, Tk, D = 3, 2, 9, 70, 32
    lens = (70, 1, 0)
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=72)
    out, lse = oracle.attn_segments(c["q"], c["k"], c["v"], [[0]] * B, [[n] for n in lens], 0.2)
    ref_out, ref_lse = oracle.attn_prefix(c["q"], c["k"], c["v"], lens, 0.2)
    np.testing.assert_allclose(out, ref_out, rtol=1e-13, atol=1e-14)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_lse))
    fin = np.isfinite(ref_lse)
    np.testing.assert_allclose(lse[fin], ref_lse[fin], rtol=1e-13, atol=1e-14)


def test_scattered_segments_equal_prefix_of_compacted_buffer():
    B, H, Tq, Tk, D = 2, 2, 6, 200, 16
    segs = [[(150, 40), (2, 9), (60, 33)], [(199, 1), (0, 1), (100, 50)]]
    q, k, v, st, ln = _holey_case(B, H, Tq, Tk, D, segs, seed=73)
    out, lse = oracle.attn_segments(q, k, v, st, ln, 0.25)
    for b in range(B):
        idx = np.concatenate([np.arange(s, s + n) for s, n in segs[b]])
        kc = torch.zeros_like(k[b:b + 1])
        vc = torch.zeros_like(v[b:b + 1])
        kc[0, :, :idx.size] = k[b][:, torch.from_numpy(idx)]
        vc[0, :, :idx.size] = v[b][:, torch.from_numpy(idx)]
        ref_out, ref_lse = oracle.attn_prefix(q[b:b + 1], kc, vc, [int(idx.size)], 0.25)
        np.testing.assert_allclose(out[b], ref_out[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[b], ref_lse[0], rtol=1e-12, atol=1e-13)


def test_hole_content_never_matters():
    B, H, Tq, Tk, D = 1, 2, 5, 120, 16
    segs = [[(0, 10), (50, 20), (100, 5)]]
    ref = None
    for hole in (float("nan"), float("inf"), 0.0, -1e30):
        q, k, v, st, ln = _holey_case(B, H, Tq, Tk, D, segs, seed=74, hole=hole)
        got = oracle.attn_segments(q, k, v, st, ln, 0.3)
        if ref is None:
            ref = got
            assert np.isfinite(got[0]).all()
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_segment_order_does_not_matter():
    B, H, Tq, Tk, D = 1, 3, 7, 160, 32
    segs = [[(0, 40), (60, 30), (120, 40)]]
    q, k, v, st, ln = _holey_case(B, H, Tq, Tk, D, segs, seed=75)
    out, lse = oracle.attn_segments(q, k, v, st, ln, 0.2)
    out_r, lse_r = oracle.attn_segments(q, k, v, [st[0][::-1]], [ln[0][::-1]], 0.2)
    np.testing.assert_allclose(out, out_r, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lse_r, rtol=1e-13, atol=1e-13)


def test_overlapping_key_takes_part_twice():
    B, H, Tq, Tk, D = 1, 1, 4, 40, 16
    c = synth.random_case(B, H, Tq, Tk, D, (Tk,), seed=76)
    out, lse = oracle.attn_segments(c["q"], c["k"], c["v"], [[0, 9]], [[10, 3]], 0.3)
    # keys 0..9 then 9..11: key 9 twice; the same as a prefix of 13 explicit rows
    idx = torch.tensor(list(range(10)) + [9, 10, 11])
    kc = torch.zeros_like(c["k"])
    vc = torch.zeros_like(c["v"])
    kc[0, :, :13] = c["k"][0][:, idx]
    vc[0, :, :13] = c["v"][0][:, idx]
    ref_out, ref_lse = oracle.attn_prefix(c["q"], kc, vc, [13], 0.3)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13, atol=1e-13)


def test_clamping_rules():
    B, H, Tq, Tk, D = 1, 1, 3, 50, 8
    c = synth.random_case(B, H, Tq, Tk, D, (Tk,), seed=77)
    q, k, v = c["q"], c["k"], c["v"]
    # start < 0 is cut at 0; a range past Tk is cut at Tk; a negative length is empty
    out, lse = oracle.attn_segments(q, k, v, [[-5, 45, 10]], [[10, 100, -3]], 0.4)
    ref = oracle.attn_segments(q, k, v, [[0, 45]], [[5, 5]], 0.4)
    assert np.array_equal(out, ref[0]) and np.array_equal(lse, ref[1])
    # the concatenation is cut after Tk keys: [0,50) then [0,50) again keeps only the first
    out2, lse2 = oracle.attn_segments(q, k, v, [[0, 0]], [[50, 50]], 0.4)
    ref2 = oracle.attn_prefix(q, k, v, [50], 0.4)
    np.testing.assert_allclose(out2, ref2[0], rtol=1e-13, atol=1e-14)


def test_no_valid_key_gives_zero_and_minus_inf():
    B, H, Tq, Tk, D = 2, 1, 3, 20, 8
    c = synth.random_case(B, H, Tq, Tk, D, (Tk, Tk), seed=78)
    out, lse = oracle.attn_segments(c["q"], c["k"], c["v"], [[0, 5], [25, 30]], [[0, -1], [4, 2]], 0.5)
    assert np.array_equal(out, np.zeros_like(out)) and np.isneginf(lse).all()
