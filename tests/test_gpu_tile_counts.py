"""GPU parity at every small key-tile count, against the fp64 oracle.

Both kernels issue S_0 and S_1 up front, then PV_j and S_{j+2} per tile (the single-CTA
kernel's two-group mode at head dims 32 and 64: S_2 before PV_0, then S_{j+3}, with P in
buffers of its own). Two softmax warpgroups take alternate key tiles at head dims 32, 64
and 128 (group 1 gets no tile at all when there is one) and merge their partial results
at the end; the masked last tile belongs to either group. With fewer tiles than S buffers
the MMA warp issues fewer S tiles up front. This sweeps 1 to 5 key tiles (all-full and
partial last tiles, a last tile of one valid key, a prefix ending one key into a tile),
positive, zero and negative scales (the sign of the scale selects a separate
specialisation), at every head dim, single pass and split-KV, with K/V padding set to
NaN so any read of it would show.
"""
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


# kv_len values: full 1..5 tiles, ragged 1..5 tiles, one key into a tile, one key short of a tile
KV_LENS = (128, 256, 384, 512, 640, 1, 129, 300, 385, 600, 513, 639)
SCALES = (None, 0.0, -0.04)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("scale", SCALES)
def test_tile_counts_single_pass(kp, D, scale):
    B = len(KV_LENS)
    case = synth.random_case(B, 2, 300, 640, D, KV_LENS, seed=D + 7, std=0.7)
    sc = case["scale"] if scale is None else scale
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    out, lse = kp.attn_prefix_fwd(g["q"], g["k"], g["v"], g["kv_len"], sc)
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], case["kv_len_list"], sc)
    assert_out_close(out, ref_out, what=f"out D={D} scale={sc}")
    assert_lse_close(lse, ref_lse, what=f"lse D={D} scale={sc}")


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_tile_counts_split(kp, D):
    # chunks of 256 keys (2 tiles): chunk-local tile counts of 0, 1 and 2, ragged ends
    B = len(KV_LENS)
    case = synth.random_case(B, 2, 150, 640, D, KV_LENS, seed=D + 11, std=0.7)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
    out, lse = kp.attn_prefix_fwd_splitkv(g["q"], g["k"], g["v"], g["kv_len"], 3, g["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], case["kv_len_list"], case["scale"])
    assert_out_close(out, ref_out, what=f"split out D={D}")
    assert_lse_close(lse, ref_lse, what=f"split lse D={D}")
