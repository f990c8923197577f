"""GPU check of the host-memory pipeline (key_prefix_masked_b200.pipeline.HostPipeline).

Steps with different inputs go through the double-buffered pipeline back to back.
Every step's host output must equal the direct device-memory call bit for bit. That
holds only if no step reads a buffer set that the next step is still copying into, or
that the read-out of the step before has not yet emptied.
"""
import pytest
import torch

import synth
from parity import bits_equal

pytestmark = pytest.mark.gpu


def test_pipeline_steps_equal_direct_calls():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    from key_prefix_masked_b200.pipeline import HostPipeline
    B, H, Tq, Tk, D = 2, 2, 300, 900, 64
    cases = [synth.random_case(B, H, Tq, Tk, D, (900 - 100 * i, 1 + 50 * i), seed=160 + i) for i in range(5)]
    pipe = HostPipeline((B, H, Tq, Tk, D))
    outs, lses = [], []
    for c in cases:
        o = torch.empty((B, H, Tq, D), dtype=torch.bfloat16).pin_memory()
        l = torch.empty((B, H, Tq), dtype=torch.float32).pin_memory()
        pipe.submit(*(c[n].pin_memory() for n in ("q", "k", "v", "kv_len")), o, l)
        outs.append(o)
        lses.append(l)
    pipe.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    for c, o, l in zip(cases, outs, lses):
        ro, rl = kp.attn_prefix_fwd(*(c[n].cuda() for n in ("q", "k", "v", "kv_len")))
        torch.cuda.synchronize()
        assert bits_equal(o, ro.cpu()) and bits_equal(l, rl.cpu())
