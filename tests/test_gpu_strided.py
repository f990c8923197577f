"""GPU parity of strided operand layouts (attn_prefix_fwd_strided and friends).

JAX's [B, T, H, D] layout ("Add sequence-parallel multi-GPU inference ...", section
"cuDNN flash attention", where the boolean mask becomes key_value_seq_lengths) and q,
k, v sliced out of one packed [B, T, 3, H, D] tensor reach the kernels as [B,H,T,D]
views. The TMA maps carry the caller's strides, so the arithmetic is the one of the
contiguous path. The results must match contiguous copies bit for bit, and the oracle
within tolerance.
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


def _bthd(x):
    """The same values as x [B,H,T,D], stored as [B,T,H,D], viewed as [B,H,T,D]."""
    return x.transpose(1, 2).contiguous().transpose(1, 2)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_bthd_equals_contiguous(kp, D):
    lens = (700, 129, 0)
    c = synth.random_case(3, 2, 300, 700, D, lens, seed=100 + D, device="cuda")
    q, k, v = (_bthd(c[n]) for n in ("q", "k", "v"))
    assert not q.is_contiguous() and q.stride(3) == 1
    out, lse = kp.attn_prefix_fwd(q, k, v, c["kv_len"], c["scale"])
    ref_out, ref_lse = kp.attn_prefix_fwd(c["q"], c["k"], c["v"], c["kv_len"], c["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert out.stride() == q.stride(), "out takes q's layout"
    assert bits_equal(out.contiguous(), ref_out) and bits_equal(lse, ref_lse)


@pytest.mark.parametrize("D", [64, 256])
def test_packed_qkv_and_strided_out(kp, D):
    B, H, T = 2, 3, 520
    g = torch.Generator(device="cuda").manual_seed(7 + D)
    x = torch.randn(B, T, 3, H, D, generator=g, device="cuda").to(torch.bfloat16)
    q, k, v = (x[:, :, i].transpose(1, 2) for i in range(3))      # [B,H,T,D] views, strides (3THD, D, 3HD)
    kv = torch.tensor([T, 333], dtype=torch.int32, device="cuda")
    out_store = torch.empty(B, T, H, D, dtype=torch.bfloat16, device="cuda")
    out = out_store.transpose(1, 2)
    o, l = kp.attn_prefix_fwd(q, k, v, kv, out=out)
    ref_out, ref_lse = kp.attn_prefix_fwd(q.contiguous(), k.contiguous(), v.contiguous(), kv)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert o.data_ptr() == out_store.data_ptr()
    assert bits_equal(out.contiguous(), ref_out) and bits_equal(l, ref_lse)
    ro, rl = oracle.attn_prefix(q.contiguous().cpu(), k.contiguous().cpu(), v.contiguous().cpu(), [T, 333],
                                1.0 / D ** 0.5)
    assert_out_close(out.contiguous(), ro)
    assert_lse_close(l, rl)


@pytest.mark.parametrize("D", [64, 256])
def test_split_and_combine_strided(kp, D):
    lens = (900, 1)
    c = synth.random_case(2, 2, 260, 1000, D, lens, seed=120 + D, device="cuda")
    q, k, v = (_bthd(c[n]) for n in ("q", "k", "v"))
    po, pl = kp.attn_prefix_fwd_split(q, k, v, c["kv_len"], 5)
    ref_po, ref_pl = kp.attn_prefix_fwd_split(c["q"], c["k"], c["v"], c["kv_len"], 5)
    out = torch.empty(2, 260, 2, D, dtype=torch.bfloat16, device="cuda").transpose(1, 2)
    o, l = kp.attn_lse_combine(po, pl, out=out)
    ref_o, ref_l = kp.attn_lse_combine(ref_po, ref_pl)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert bits_equal(po, ref_po) and bits_equal(pl, ref_pl)
    assert bits_equal(out.contiguous(), ref_o) and bits_equal(l, ref_l)


def test_bad_strides_are_rejected(kp):
    c = synth.random_case(1, 2, 64, 128, 64, (128,), seed=130, device="cuda")
    # a [B,H,T,D] view whose row stride is not a multiple of 8 elements
    wide = torch.zeros(1, 2, 64, 68, dtype=torch.bfloat16, device="cuda")[..., :64]
    with pytest.raises(ValueError):
        kp.attn_prefix_fwd(wide, c["k"], c["v"], c["kv_len"])
