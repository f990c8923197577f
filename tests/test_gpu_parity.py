"""GPU parity: the sm_100a kernels, called through the C ABI, against the fp64 oracle on
the same seeded inputs, plus the bit-exact key-selection properties.

Sizes span several 128-row query tiles and 128-key tiles with ragged tails; the full
workloads are checked on sampled query rows (the oracle evaluates them one by one).
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


def _cuda(case):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}


def _run_and_compare(kp, case, rows=None):
    g = _cuda(case)
    out, lse = kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"], g["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], case["kv_len_list"],
                                          case["scale"], rows=rows)
    if rows is not None:
        out, lse = out[:, :, rows], lse[:, :, rows]
    assert_out_close(out, ref_out)
    assert_lse_close(lse, ref_lse)
    return out, lse


def test_tiny_workload(kp):
    case = synth.make_inputs(synth.WORKLOADS["tiny"], device="cpu", seed=0)
    _run_and_compare(kp, case)


SWEEP = [
    # B, H, Tq, Tk, kv_len per element
    (2, 2, 200, 300, (0, 1)),
    (1, 2, 129, 257, (257,)),
    (3, 1, 300, 384, (127, 128, 129)),
    (2, 1, 64, 1000, (999, 500)),
    (1, 1, 1, 17, (16,)),
    (2, 1, 256, 640, (15, 17)),
    (1, 1, 383, 130, (130,)),
    (1, 1, 1, 1, (1,)),                       # one query, one key
    (1, 2, 1, 1000, (1000,)),                 # one query row against a long prefix
    (4, 16, 33, 65, (65, 1, 64, 0)),          # many (b, h) slices of short sequences
    (1, 1, 513, 1024, (1024,)),               # a CTA pair whose second tile holds one row
]


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("shape", SWEEP, ids=lambda s: "B{}H{}Tq{}Tk{}kv{}".format(
    s[0], s[1], s[2], s[3], "-".join(map(str, s[4]))))
def test_sweep_against_oracle(kp, D, shape):
    B, H, Tq, Tk, lens = shape
    case = synth.random_case(B, H, Tq, Tk, D, lens, seed=D + Tq, std=1.0)
    _run_and_compare(kp, case)


@pytest.mark.parametrize("D", [64, 256])
def test_scale_variants(kp, D):
    for scale, std in ((0.0, 1.0), (0.5, 1.0), (1.0 / math.sqrt(D), 3.0), (-0.2, 1.0)):
        case = synth.random_case(1, 2, 150, 270, D, (261,), seed=7, std=std)
        case["scale"] = scale
        _run_and_compare(kp, case)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_padding_content_is_never_read(kp, D):
    lens = (77, 200, 129)
    base = synth.random_case(3, 2, 140, 256, D, lens, seed=3)
    outs = []
    for pad in (float("nan"), float("inf"), float("-inf"), 0.0, 3.0e38):
        k, v = base["k"].clone(), base["v"].clone()
        synth.fill_padding(k, v, lens, pad)
        out, lse = kp.attn_prefix_fwd(base["q"].cuda(), k.cuda(), v.cuda(), base["kv_len"].cuda())
        outs.append((out, lse))
    torch.cuda.synchronize()
    for out, lse in outs[1:]:
        assert bits_equal(out, outs[0][0]) and bits_equal(lse, outs[0][1])
    assert torch.isfinite(outs[0][0].float()).all()


@pytest.mark.parametrize("D", [64, 256])
def test_ragged_equals_per_element_calls(kp, D):
    lens = (300, 1, 0, 129, 512)
    case = _cuda(synth.random_case(len(lens), 2, 190, 512, D, lens, seed=4))
    out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    for b in range(len(lens)):
        o1, l1 = kp.attn_prefix_fwd(case["q"][b:b + 1].contiguous(), case["k"][b:b + 1].contiguous(),
                                    case["v"][b:b + 1].contiguous(), case["kv_len"][b:b + 1].contiguous())
        assert bits_equal(o1[0], out[b]) and bits_equal(l1[0], lse[b]), b


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_padded_buffer_equals_truncated_buffer(kp, D):
    for n in (1, 100, 128, 129, 255):
        case = _cuda(synth.random_case(1, 2, 130, 300, D, (n,), seed=n))
        out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
        kt = case["k"][:, :, :n].contiguous()
        vt = case["v"][:, :, :n].contiguous()
        o2, l2 = kp.attn_prefix_fwd(case["q"], kt, vt, case["kv_len"])
        assert bits_equal(out, o2) and bits_equal(lse, l2), n


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_closed_forms(kp, D):
    case = _cuda(synth.random_case(2, 2, 140, 300, D, (1, 290), seed=9))
    v = torch.full_like(case["v"], 0.3125)
    out, _ = kp.attn_prefix_fwd(case["q"], case["k"], v, case["kv_len"])
    assert_out_close(out, np.full(tuple(out.shape), 0.3125), what="uniform v")
    # kv_len = 1: out = v_0 exactly, lse = scale q.k_0
    out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    v0 = case["v"][0, :, 0:1, :].expand(-1, out.shape[2], -1)
    assert torch.equal(out[0], v0)
    s = (case["q"][0].double() * case["k"][0, :, 0:1, :].double()).sum(-1) * case["scale"]
    assert (lse[0].double() - s).abs().max().item() < 1e-3


def test_empty_element_exact(kp):
    for D in (32, 64, 128, 256):
        case = _cuda(synth.random_case(2, 3, 200, 256, D, (0, 256), seed=10))
        out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
        assert torch.equal(out[0], torch.zeros_like(out[0]))
        assert torch.isneginf(lse[0]).all() and torch.isfinite(lse[1]).all()


def test_kv_len_out_of_range_is_clamped_and_flagged(kp):
    case = _cuda(synth.random_case(2, 1, 100, 160, 64, (160, 5), seed=11, pad_value=0.5))
    ref_out, ref_lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    assert kp.device_status() == kp.ATTN_OK
    bad = torch.tensor([165, -3], dtype=torch.int32, device="cuda")
    out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], bad)
    assert kp.device_status() == kp.ATTN_ERR_KVLEN_RANGE
    assert kp.device_status() == kp.ATTN_OK           # the flag is cleared once read
    assert bits_equal(out[0], ref_out[0]) and bits_equal(lse[0], ref_lse[0])
    assert torch.equal(out[1], torch.zeros_like(out[1])) and torch.isneginf(lse[1]).all()


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("C", [1, 3, 7])
def test_split_partials_against_oracle_chunks(kp, D, C):
    lens = (700, 129, 0)
    case = synth.random_case(3, 2, 150, 700, D, lens, seed=12 + C)
    g = _cuda(case)
    part_out, part_lse = kp.attn_prefix_fwd_split(g["q"], g["k"], g["v"], g["kv_len"], C)
    L = kp.split_chunk_len(700, C)
    for c in range(C):
        ro, rl = oracle.attn_chunk(case["q"], case["k"], case["v"], lens, case["scale"], c * L, (c + 1) * L)
        assert_out_close(part_out[c], ro, what=f"part_out[{c}]")
        assert_lse_close(part_lse[c], rl, what=f"part_lse[{c}]")
    out, lse = kp.attn_lse_combine(part_out, part_lse)
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], lens, case["scale"])
    assert_out_close(out, ref_out)
    assert_lse_close(lse, ref_lse)


def test_split_equals_single_pass_within_tolerance(kp):
    case = _cuda(synth.random_case(1, 4, 256, 4096, 256, (4000,), seed=13, std=0.5))
    o1, l1 = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    o2, l2 = kp.attn_prefix_fwd_splitkv(case["q"], case["k"], case["v"], case["kv_len"], 8)
    assert_out_close(o2, o1.double().cpu().numpy(), what="split vs single")
    assert_lse_close(l2, l1.double().cpu().numpy(), what="split lse vs single")


def test_lse_is_optional_and_streams_are_honoured(kp):
    case = _cuda(synth.random_case(1, 2, 130, 200, 64, (199,), seed=14))
    o_ref, _ = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"], need_lse=False)
    s.synchronize()
    assert l2 is None and bits_equal(o_ref, o2)


# ---------------------------------------------------------------- full-size workloads
def _workload_check(kp, name, n_random, splits=None):
    w = synth.WORKLOADS[name]
    case = synth.make_inputs(w, device="cuda", seed=0)
    rows = synth.sample_rows(w.Tq, n_random=n_random, seed=0)
    if splits:
        out, lse = kp.attn_prefix_fwd_splitkv(case["q"], case["k"], case["v"], case["kv_len"], splits)
    else:
        out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    # properties at every row: finite output where the prefix is non-empty, -inf lse otherwise
    for b, n in enumerate(case["kv_len_list"]):
        if n > 0:
            assert torch.isfinite(out[b].float()).all() and torch.isfinite(lse[b]).all()
        else:
            assert torch.equal(out[b], torch.zeros_like(out[b])) and torch.isneginf(lse[b]).all()
    host = {k: case[k].cpu() for k in ("q", "k", "v")}
    del case["q"], case["k"], case["v"]
    ref_out, ref_lse = oracle.attn_prefix(host["q"], host["k"], host["v"], case["kv_len_list"],
                                          case["scale"], rows=rows)
    assert_out_close(out[:, :, rows], ref_out)
    assert_lse_close(lse[:, :, rows], ref_lse)


def test_workload_unmasked(kp):
    _workload_check(kp, "unmasked", n_random=40)


def test_workload_icl(kp):
    _workload_check(kp, "icl", n_random=16)


def test_workload_ragged(kp):
    _workload_check(kp, "ragged", n_random=16)


def test_workload_splitkv(kp):
    _workload_check(kp, "splitkv", n_random=0, splits=64)


def test_workload_unmasked_8v(kp):
    _workload_check(kp, "unmasked_8v", n_random=24)


def test_workload_unmasked_32v(kp):
    _workload_check(kp, "unmasked_32v", n_random=24)


def test_workload_unmasked_d128(kp):
    _workload_check(kp, "unmasked_d128", n_random=24)


def test_workload_prefix_d128(kp):
    _workload_check(kp, "prefix_d128", n_random=16)


@pytest.mark.parametrize("D", [64, 256])
def test_grid_beyond_65535_slices(kp, D):
    """131072 (b, h) slices of short sequences: a 1-D grid of more than 2^16 CTAs (and
    CTA pairs at D=256), ragged kv_len drawn per element including 0."""
    B, H, Tq, Tk = 512, 256, 8, 8
    g = torch.Generator().manual_seed(170 + D)
    lens = torch.randint(0, Tk + 1, (B,), generator=g).tolist()
    case = synth.random_case(B, H, Tq, Tk, D, tuple(lens), seed=171 + D, device="cuda")
    out, lse = kp.attn_prefix_fwd(case["q"], case["k"], case["v"], case["kv_len"], case["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    bsel = [0, 1, 255, 256, 511]
    q = case["q"][bsel].cpu()
    k, v = case["k"][bsel].cpu(), case["v"][bsel].cpu()
    ref_out, ref_lse = oracle.attn_prefix(q, k, v, [lens[b] for b in bsel], case["scale"])
    assert_out_close(out[bsel], ref_out)
    assert_lse_close(lse[bsel], ref_lse)


@pytest.mark.parametrize("D", [64, 256])
def test_cuda_graph_capture_and_replay(kp, D):
    """The forward captured into a CUDA graph (after one eager call) replays bit for bit;
    new inputs copied into the captured buffers give the new result."""
    c1 = synth.random_case(2, 2, 300, 700, D, (700, 129), seed=180 + D, device="cuda")
    c2 = synth.random_case(2, 2, 300, 700, D, (64, 700), seed=181 + D, device="cuda")
    q, k, v, kv = (c1[n].clone() for n in ("q", "k", "v", "kv_len"))
    out = torch.empty_like(q)
    lse = torch.empty(2, 2, 300, dtype=torch.float32, device="cuda")
    kp.attn_prefix_fwd(q, k, v, kv, out=out, lse=lse)      # eager warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kp.attn_prefix_fwd(q, k, v, kv, out=out, lse=lse)
    for c in (c1, c2):
        for dst, n in ((q, "q"), (k, "k"), (v, "v"), (kv, "kv_len")):
            dst.copy_(c[n])
        g.replay()
        torch.cuda.synchronize()
        ref_out, ref_lse = kp.attn_prefix_fwd(c["q"], c["k"], c["v"], c["kv_len"])
        torch.cuda.synchronize()
        assert bits_equal(out, ref_out) and bits_equal(lse, ref_lse)
    assert kp.device_status() == kp.ATTN_OK
