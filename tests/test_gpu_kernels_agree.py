"""Head dims 128 and 256 have two implementations: CTA pairs (default) and a single-CTA
kernel (selected by the ATTN_DEBUG_SINGLE_CTA test hook).  Both must match the oracle
and each other, single pass and split."""
import numpy as np
import pytest
import torch

import synth
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kp():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    yield kp
    kp.set_debug_flags(0)


SINGLE_CTA = 2


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("shape", [
    (2, 2, 300, 700, (700, 129)),
    (1, 3, 513, 1000, (999,)),
    (3, 1, 130, 256, (0, 1, 255)),
])
def test_pair_and_single_cta_agree(kp, D, shape):
    B, H, Tq, Tk, lens = shape
    c = synth.random_case(B, H, Tq, Tk, D, lens, seed=Tq + D)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in c.items()}
    kp.set_debug_flags(0)
    o_pair, l_pair = kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"])
    po_pair, pl_pair = kp.attn_prefix_fwd_split(g["q"], g["k"], g["v"], g["kv_len"], 3)
    kp.set_debug_flags(SINGLE_CTA)
    o_one, l_one = kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"])
    po_one, pl_one = kp.attn_prefix_fwd_split(g["q"], g["k"], g["v"], g["kv_len"], 3)
    kp.set_debug_flags(0)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert_out_close(o_pair, o_one.double().cpu().numpy(), what="pair vs single out")
    assert_lse_close(l_pair, l_one.double().cpu().numpy(), what="pair vs single lse")
    assert_out_close(po_pair, po_one.double().cpu().numpy(), what="pair vs single partials")
    assert_lse_close(pl_pair, pl_one.double().cpu().numpy(), what="pair vs single partial lse")
