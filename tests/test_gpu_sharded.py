"""GPU parity of key-sharded attention (key_prefix_masked_b200.sharded) on one GPU.

The per-shard partial and the combine are the product kernels. Shards are emulated on
one device by stacking the partials the all-gather would deliver, in rank order. A
world-size-1 NCCL group runs the whole call. The multi-rank exchange itself is covered
by tests/test_sharded_cpu.py on gloo ranks.
"""
import socket

import pytest
import torch

import oracle
import synth
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kp():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    torch.cuda.init()
    assert kp.device_status() == kp.ATTN_OK
    return kp


@pytest.mark.parametrize("D", [64, 256])
def test_emulated_shards_equal_unsharded(kp, D):
    from key_prefix_masked_b200 import sharded
    kv_full = [3000, 700]
    c = synth.random_case(2, 2, 300, 3000, D, tuple(kv_full), seed=140 + D, device="cuda")
    bounds = [(0, 1000), (1000, 1900), (1900, 3000)]      # three unequal shards
    parts = []
    for lo, hi in bounds:
        kv = torch.tensor([max(0, min(n - lo, hi - lo)) for n in kv_full], dtype=torch.int32, device="cuda")
        parts.append(sharded.local_partial(c["q"], c["k"][:, :, lo:hi].contiguous(),
                                           c["v"][:, :, lo:hi].contiguous(), kv, c["scale"]))
    po = torch.cat([p[0] for p in parts], dim=0)
    pl = torch.cat([p[1] for p in parts], dim=0)
    out, lse = sharded.combine(po, pl)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    assert torch.isneginf(pl[2, 1]).all()                 # element 1 has no key in shard 2
    ref_out, ref_lse = oracle.attn_prefix(c["q"].cpu(), c["k"].cpu(), c["v"].cpu(), kv_full, c["scale"])
    assert_out_close(out, ref_out)
    assert_lse_close(lse, ref_lse)
    single_out, _ = kp.attn_prefix_fwd(c["q"], c["k"], c["v"], c["kv_len"], c["scale"])
    assert_out_close(out, single_out.double().cpu().numpy(), what="sharded vs single pass")


def test_world_size_one_nccl_group(kp):
    import torch.distributed as dist
    from key_prefix_masked_b200 import sharded
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    c = synth.random_case(1, 2, 130, 500, 64, (480,), seed=150, device="cuda")
    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{port}")
    try:
        out, lse = sharded.key_sharded_fwd(c["q"], c["k"], c["v"], c["kv_len"], c["scale"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref_out, ref_lse = oracle.attn_prefix(c["q"].cpu(), c["k"].cpu(), c["v"].cpu(), [480], c["scale"])
    assert_out_close(out, ref_out)
    assert_lse_close(lse, ref_lse)
