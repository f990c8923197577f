"""GPU parity of split-KV with the combine fused into the launch (attn_prefix_fwd_split_fused).

The fused path must give, bit for bit, what the two-launch path gives (split partials,
then attn_lse_combine): both run the same per-row combination arithmetic. It is also
compared with the fp64 oracle. The kernel must leave its tile counters at zero so
that a workspace can be reused. Shapes cover query counts that leave a CTA pair's
second tile empty, chunks past kv_len, an empty batch element and one split.
"""
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


def _counters(kp, ws, C, B, H, Tq, D):
    lib = kp.lib()
    off = int(lib.attn_split_counter_offset(C, B, H, Tq, D))
    n = B * H * ((Tq + 127) // 128)
    return ws[off:off + 4 * n].view(torch.int32)


SHAPES = [
    # B, H, Tq, Tk, kv_len
    (3, 2, 150, 700, (700, 129, 0)),
    (2, 3, 300, 1000, (1000, 1)),       # Tq=300: the last CTA pair's second tile has no rows
    (1, 2, 513, 2048, (1999,)),
]


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("C", [1, 3, 7])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B{}H{}Tq{}Tk{}".format(*s[:4]))
def test_fused_equals_two_launch_and_oracle(kp, D, C, shape):
    B, H, Tq, Tk, lens = shape
    case = synth.random_case(B, H, Tq, Tk, D, lens, seed=40 + C + D)
    g = _cuda(case)
    part_out, part_lse = kp.attn_prefix_fwd_split(g["q"], g["k"], g["v"], g["kv_len"], C)
    o2, l2 = kp.attn_lse_combine(part_out, part_lse)
    ws = kp.fused_workspace(C, B, H, Tq, D, g["q"].device)
    o1, l1 = kp.attn_prefix_fwd_split_fused(g["q"], g["k"], g["v"], g["kv_len"], C, workspace=ws)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert bits_equal(o1, o2) and bits_equal(l1, l2), "fused and two-launch combine differ"
    assert int(_counters(kp, ws, C, B, H, Tq, D).abs().sum()) == 0, "tile counters not left at zero"
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], lens, case["scale"])
    assert_out_close(o1, ref_out)
    assert_lse_close(l1, ref_lse)
    # the same workspace again, with its counters back at zero: same result
    o3, l3 = kp.attn_prefix_fwd_split_fused(g["q"], g["k"], g["v"], g["kv_len"], C, workspace=ws)
    torch.cuda.synchronize()
    assert bits_equal(o1, o3) and bits_equal(l1, l3)


def test_fused_without_lse(kp):
    case = _cuda(synth.random_case(1, 2, 200, 900, 64, (850,), seed=47))
    o1, l1 = kp.attn_prefix_fwd_split_fused(case["q"], case["k"], case["v"], case["kv_len"], 4)
    o2, l2 = kp.attn_prefix_fwd_split_fused(case["q"], case["k"], case["v"], case["kv_len"], 4,
                                            need_lse=False)
    torch.cuda.synchronize()
    assert l2 is None and bits_equal(o1, o2)


def test_fused_rejects_small_workspace(kp):
    case = _cuda(synth.random_case(1, 1, 64, 256, 64, (256,), seed=48))
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        kp.attn_prefix_fwd_split_fused(case["q"], case["k"], case["v"], case["kv_len"], 2, workspace=ws)


def test_workload_splitkv_fused(kp):
    """The split-KV workload (1e6 keys, 64 chunks): fused == two-launch bit for bit, and
    sampled rows against the oracle."""
    w = synth.WORKLOADS["splitkv"]
    case = synth.make_inputs(w, device="cuda", seed=0)
    o1, l1 = kp.attn_prefix_fwd_split_fused(case["q"], case["k"], case["v"], case["kv_len"], w.num_splits)
    o2, l2 = kp.attn_prefix_fwd_splitkv(case["q"], case["k"], case["v"], case["kv_len"], w.num_splits)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert bits_equal(o1, o2) and bits_equal(l1, l2)
    rows = synth.sample_rows(w.Tq, n_random=0, seed=0)
    host = {k: case[k].cpu() for k in ("q", "k", "v")}
    ref_out, ref_lse = oracle.attn_prefix(host["q"], host["k"], host["v"], case["kv_len_list"],
                                          case["scale"], rows=rows)
    assert_out_close(o1[:, :, rows], ref_out)
    assert_lse_close(l1[:, :, rows], ref_lse)
