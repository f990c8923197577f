"""Pins for the fp64 oracle: values and identities fixed by the pages and by mathematics,
none of them computed by the oracle itself.

- hand-derived cases (tests/golden/hand_cases.json, each with its citation);
- a library routine that computes the pages' own operation: torch's CPU
  scaled_dot_product_attention in float64 with a [B,1,1,Tk] boolean key mask, and
  torch.logsumexp of the masked scores;
- closed forms (uniform values, single key, zero scale, equal keys, empty prefix);
- the identities the pages state: prefix mask == k/v truncation, ragged prefix ==
  per-element truncation, shard-wise LSE combination == unsplit result.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _num(x):
    if isinstance(x, str):
        env = {"log": math.log, "exp": math.exp, "sqrt": math.sqrt,
               "inf": math.inf, "nan": math.nan, "__builtins__": {}}
        return float(eval(x, env))  # noqa: S307 - fixture expressions only
    return float(x)


def _bf16(rows, B=1, H=1):
    t = torch.tensor([[_num(x) for x in r] for r in rows], dtype=torch.float64)
    assert torch.equal(t.to(torch.bfloat16).to(torch.float64).nan_to_num(7.0),
                       t.nan_to_num(7.0)), "fixture value not representable in bf16"
    return t.to(torch.bfloat16).reshape(B, H, t.shape[0], t.shape[1])


def _load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _load_golden()["cases"], ids=lambda c: c["name"])
def test_hand_derived_case(case):
    q, k, v = _bf16(case["q"]), _bf16(case["k"]), _bf16(case["v"])
    out, lse = oracle.attn_prefix(q, k, v, [case["kv_len"]], _num(case["scale"]))
    want_out = np.array([[_num(x) for x in r] for r in case["out"]])
    want_lse = np.array([_num(x) for x in case["lse"]])
    np.testing.assert_allclose(out[0, 0], want_out, rtol=1e-14, atol=1e-14)
    if np.isinf(want_lse).any():
        assert np.array_equal(lse[0, 0], want_lse)
    else:
        np.testing.assert_allclose(lse[0, 0], want_lse, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("case", _load_golden()["combine_cases"], ids=lambda c: c["name"])
def test_hand_derived_combine(case):
    po = np.array([[_num(x) for x in r] for r in case["part_out"]])[:, None, :]
    pl = np.array([_num(x) for x in case["part_lse"]])[:, None]
    out, lse = oracle.lse_combine(po, pl)
    np.testing.assert_allclose(out[0], [_num(x) for x in case["out"]], rtol=1e-14,
                               atol=1e-14)
    want = _num(case["lse"])
    if math.isinf(want):
        assert lse[0] == want
    else:
        assert abs(lse[0] - want) < 1e-14
    assert np.isfinite(out).all()


def _sdpa_reference(q, k, v, kv_len, scale):
    """torch SDPA (CPU, float64) with a [B,1,1,Tk] boolean prefix mask, and the
    log-sum-exp of the masked scaled scores from torch.logsumexp."""
    B, H, Tq, D = q.shape
    Tk = k.shape[2]
    qd, kd, vd = (t.to(torch.float64) for t in (q, k, v))
    mask = torch.arange(Tk)[None, :] < torch.tensor(kv_len)[:, None]     # [B, Tk]
    m4 = mask[:, None, None, :]                                          # [B,1,1,Tk]
    out = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=m4,
                                                           scale=scale)
    scores = torch.einsum("bhid,bhjd->bhij", qd, kd) * scale
    scores = scores.masked_fill(~m4, float("-inf"))
    lse = torch.logsumexp(scores, dim=-1)
    return out.numpy(), lse.numpy()


@pytest.mark.parametrize("B,H,Tq,Tk,D,lens,seed", [
    (2, 2, 64, 96, 32, (40, 96), 0),          # the tiny workload's shape
    (1, 3, 17, 33, 64, (33,), 1),
    (3, 1, 5, 129, 16, (1, 128, 129), 2),
    (2, 2, 9, 7, 8, (7, 3), 3),
    (1, 1, 300, 260, 32, (257,), 4),
])
def test_oracle_matches_library_sdpa(B, H, Tq, Tk, D, lens, seed):
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=seed, pad_value=0.25)
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle.attn_prefix(c["q"], c["k"], c["v"], lens, scale)
    ref_out, ref_lse = _sdpa_reference(c["q"], c["k"], c["v"], list(lens), scale)
    np.testing.assert_allclose(out, ref_out, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_library_pin_detects_transposed_and_unscaled_variants():
    """The library pin is sensitive to the plausible mistakes it must catch: a missing
    scale, k and v swapped, or keys beyond the prefix taking part all move the result
    far beyond the comparison tolerance."""
    B, H, Tq, Tk, D = 1, 2, 8, 12, 16
    lens = [9]
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=5, pad_value=0.5)
    scale = 0.25
    ref_out, ref_lse = _sdpa_reference(c["q"], c["k"], c["v"], lens, scale)
    bad = [
        oracle.attn_prefix(c["q"], c["k"], c["v"], lens, 1.0),            # dropped scale
        oracle.attn_prefix(c["q"], c["v"], c["k"], lens, scale),          # k/v swapped
        oracle.attn_prefix(c["q"], c["k"], c["v"], [Tk], scale),          # mask ignored
        oracle.attn_prefix(c["q"], c["k"], c["v"], [8], scale),           # off by one
    ]
    for out, lse in bad:
        assert (np.abs(out - ref_out).max() > 1e-6) or (np.abs(lse - ref_lse).max() > 1e-6)


def test_uniform_values_return_the_value():
    B, H, Tq, Tk, D = 2, 2, 7, 50, 32
    lens = [1, 37]
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=11)
    v = torch.full_like(c["v"], 0.375)
    out, _ = oracle.attn_prefix(c["q"], c["k"], v, lens, 0.3)
    np.testing.assert_allclose(out, 0.375, rtol=0, atol=1e-15)


def test_single_key_closed_form():
    B, H, Tq, Tk, D = 1, 2, 6, 10, 8
    c = synth.random_case(B, H, Tq, Tk, D, [1], seed=12)
    scale = 0.7
    out, lse = oracle.attn_prefix(c["q"], c["k"], c["v"], [1], scale)
    q = c["q"].to(torch.float64)
    k0 = c["k"].to(torch.float64)[:, :, 0, :]
    v0 = c["v"].to(torch.float64)[:, :, 0, :]
    want_lse = scale * (q * k0[:, :, None, :]).sum(-1)
    np.testing.assert_allclose(out, v0[:, :, None, :].expand_as(q).numpy(), rtol=0, atol=0)
    np.testing.assert_allclose(lse, want_lse.numpy(), rtol=1e-14, atol=1e-14)


def test_zero_scale_is_the_mean():
    B, H, Tq, Tk, D = 1, 1, 4, 20, 8
    n = 13
    c = synth.random_case(B, H, Tq, Tk, D, [n], seed=13)
    out, lse = oracle.attn_prefix(c["q"], c["k"], c["v"], [n], 0.0)
    mean = c["v"].to(torch.float64)[0, 0, :n, :].mean(0).numpy()
    np.testing.assert_allclose(out[0, 0], np.broadcast_to(mean, (Tq, D)), rtol=1e-14,
                               atol=1e-14)
    np.testing.assert_allclose(lse, math.log(n), rtol=1e-15, atol=1e-15)


def test_equal_keys_closed_form():
    B, H, Tq, Tk, D = 1, 1, 3, 9, 4
    n = 6
    c = synth.random_case(B, H, Tq, Tk, D, [n], seed=14)
    k = c["k"].clone()
    k[0, 0, :n, :] = k[0, 0, 0, :]
    scale = 0.5
    out, lse = oracle.attn_prefix(c["q"], k, c["v"], [n], scale)
    q = c["q"].to(torch.float64)[0, 0]
    s = scale * (q @ k.to(torch.float64)[0, 0, 0])
    mean = c["v"].to(torch.float64)[0, 0, :n].mean(0)
    np.testing.assert_allclose(out[0, 0], mean.expand(Tq, D).numpy(), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], (s + math.log(n)).numpy(), rtol=1e-14, atol=1e-14)


def test_empty_prefix():
    c = synth.random_case(2, 2, 5, 8, 16, [0, 3], seed=15)
    out, lse = oracle.attn_prefix(c["q"], c["k"], c["v"], [0, 3], 0.25)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isneginf(lse[0]))
    assert np.isfinite(out[1]).all() and np.isfinite(lse[1]).all()


def test_prefix_mask_equals_truncation():
    """Dense boolean-mask attention over the padded buffer equals the truncated
    computation (finite padding), as the prefix-mask rewrite states."""
    B, H, Tq, Tk, D = 2, 2, 11, 40, 32
    lens = [17, 40]
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=16, pad_value=3.0)
    mask = (torch.arange(Tk)[None, :] < torch.tensor(lens)[:, None]).numpy()
    out_m, lse_m = oracle.attn_masked(c["q"], c["k"], c["v"], mask, 0.2)
    out_t, lse_t = oracle.attn_prefix(c["q"], c["k"], c["v"], lens, 0.2)
    np.testing.assert_allclose(out_m, out_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse_m, lse_t, rtol=1e-12, atol=1e-12)
    # and the truncated buffer itself (k/v cut to n rows, no mask) gives the same rows
    for b, n in enumerate(lens):
        qb, kb, vb = c["q"][b:b + 1], c["k"][b:b + 1, :, :n], c["v"][b:b + 1, :, :n]
        o1, l1 = oracle.attn_prefix(qb, kb.contiguous(), vb.contiguous(), [n], 0.2)
        np.testing.assert_allclose(o1[0], out_t[b], rtol=0, atol=0)
        np.testing.assert_allclose(l1[0], lse_t[b], rtol=0, atol=0)


def test_padding_content_never_matters():
    B, H, Tq, Tk, D = 2, 1, 6, 30, 16
    lens = [10, 29]
    base = synth.random_case(B, H, Tq, Tk, D, lens, seed=17, pad_value=float("nan"))
    ref = oracle.attn_prefix(base["q"], base["k"], base["v"], lens, 0.25)
    for pad in (float("inf"), float("-inf"), 0.0, 1e30):
        k, v = base["k"].clone(), base["v"].clone()
        synth.fill_padding(k, v, lens, pad)
        got = oracle.attn_prefix(base["q"], k, v, lens, 0.25)
        assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
    assert np.isfinite(ref[0]).all()


def test_ragged_equals_per_element_truncation():
    B, H, Tq, Tk, D = 4, 2, 9, 64, 32
    lens = [64, 1, 33, 0]
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=18)
    out, lse = oracle.attn_prefix(c["q"], c["k"], c["v"], lens, 0.17)
    for b, n in enumerate(lens):
        o1, l1 = oracle.attn_prefix(c["q"][b:b + 1], c["k"][b:b + 1], c["v"][b:b + 1], [n],
                                    0.17)
        assert np.array_equal(o1[0], out[b]) and np.array_equal(l1[0], lse[b])


@pytest.mark.parametrize("bounds", [
    [0, 16, 32, 48, 64],           # equal chunks
    [0, 5, 40, 41, 64],            # unequal, one single-key chunk
    [0, 30, 64, 100, 200],         # chunks past every prefix are empty
])
def test_lse_combination_equals_unsplit(bounds):
    B, H, Tq, Tk, D = 3, 2, 7, 64, 32
    lens = [64, 29, 0]
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=19)
    full_o, full_l = oracle.attn_prefix(c["q"], c["k"], c["v"], lens, 0.2)
    parts = [oracle.attn_chunk(c["q"], c["k"], c["v"], lens, 0.2, a, b)
             for a, b in zip(bounds[:-1], bounds[1:])]
    po = np.stack([p[0] for p in parts])
    pl = np.stack([p[1] for p in parts])
    out, lse = oracle.lse_combine(po, pl)
    np.testing.assert_allclose(out, full_o, rtol=1e-12, atol=1e-12)
    fin = np.isfinite(full_l)
    np.testing.assert_allclose(lse[fin], full_l[fin], rtol=1e-12, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(full_l))


def test_row_sampling_matches_full():
    c = synth.random_case(1, 2, 40, 50, 16, [45], seed=20)
    rows = [0, 3, 39, 17]
    full_o, full_l = oracle.attn_prefix(c["q"], c["k"], c["v"], [45], 0.3)
    o, l = oracle.attn_prefix(c["q"], c["k"], c["v"], [45], 0.3, rows=rows)
    assert np.array_equal(o, full_o[:, :, rows]) and np.array_equal(l, full_l[:, :, rows])


def test_oracle_rejects_bad_arguments():
    c = synth.random_case(1, 1, 4, 8, 8, [8], seed=21)
    with pytest.raises(ValueError):
        oracle.attn_prefix(c["q"], c["k"], c["v"], [9], 1.0)       # kv_len > Tk
    with pytest.raises(ValueError):
        oracle.attn_prefix(c["q"], c["k"], c["v"], [-1], 1.0)
    with pytest.raises(ValueError):
        oracle.attn_prefix(c["q"], c["k"], c["v"], [8], 1.0, rows=[4])
