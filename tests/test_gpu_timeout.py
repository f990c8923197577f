"""The bounded waits: a copy that is announced but never issued (test hook
ATTN_DEBUG_DROP_COPY) makes the consumer's wait run out; the kernel must end, report
ATTN_ERR_TIMEOUT through attn_get_device_status, and leave the context usable."""
import pytest
import torch

import synth
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

DROP_COPY = 1
SINGLE_CTA = 2


@pytest.fixture(scope="module")
def kp():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    yield kp
    kp.set_debug_flags(0)
    kp.set_wait_limit_ns(1_000_000_000)


@pytest.mark.parametrize("D,flags", [(256, 0), (256, SINGLE_CTA), (64, 0), (128, 0), (128, SINGLE_CTA)])
def test_dropped_copy_times_out_and_context_survives(kp, D, flags):
    import oracle
    c = synth.random_case(1, 2, 200, 500, D, (480,), seed=D + flags)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in c.items()}
    assert kp.device_status() == kp.ATTN_OK
    kp.set_wait_limit_ns(20_000_000)
    kp.set_debug_flags(DROP_COPY | flags)
    try:
        kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"])
        assert kp.device_status() == kp.ATTN_ERR_TIMEOUT
    finally:
        kp.set_debug_flags(0)
        kp.set_wait_limit_ns(1_000_000_000)
    # the next launch on the same context is unaffected
    out, lse = kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"])
    assert kp.device_status() == kp.ATTN_OK
    ro, rl = oracle.attn_prefix(c["q"], c["k"], c["v"], c["kv_len_list"], c["scale"])
    assert_out_close(out, ro)
    assert_lse_close(lse, rl)
