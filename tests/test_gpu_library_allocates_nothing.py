"""The C library allocates no device memory: every buffer is the caller's.

After one warm-up call per entry point (which may load the kernels' code onto the
device), further calls through the C ABI with caller-owned buffers must leave the
device's free memory exactly where it was, at every head dim and for the single-pass,
split + combine, fused-split, multi-range and no-allocation split-KV entries.
"""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


@pytest.fixture(scope="module")
def lib():
    from key_prefix_masked_b200 import build
    build.build()
    from key_prefix_masked_b200 import _binding
    return _binding.lib()


def _free_bytes():
    torch.cuda.synchronize()
    return torch.cuda.mem_get_info()[0]


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_entry_points_allocate_nothing(lib, D):
    B, H, Tq, Tk, C = 2, 2, 300, 700, 3
    case = synth.random_case(B, H, Tq, Tk, D, (700, 129), seed=D)
    q, k, v, kv = (case[n].cuda() for n in ("q", "k", "v", "kv_len"))
    out = torch.empty_like(q)
    lse = torch.empty(B, H, Tq, dtype=torch.float32, device="cuda")
    po = torch.empty(C, B, H, Tq, D, dtype=torch.float32, device="cuda")
    pl = torch.empty(C, B, H, Tq, dtype=torch.float32, device="cuda")
    ws = torch.zeros(lib.attn_split_fused_workspace_bytes(C, B, H, Tq, D), dtype=torch.uint8, device="cuda")
    seg_start = torch.tensor([[0, 400], [10, 600]], dtype=torch.int32, device="cuda")
    seg_len = torch.tensor([[200, 300], [50, 79]], dtype=torch.int32, device="cuda")
    seg_ws = torch.zeros(lib.attn_segments_workspace_bytes(B, H, Tk, D), dtype=torch.uint8, device="cuda")
    stream = P(torch.cuda.current_stream().cuda_stream)
    scale = ctypes.c_float(case["scale"])

    def calls():
        assert lib.attn_prefix_fwd(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(kv.data_ptr()),
                                   P(out.data_ptr()), P(lse.data_ptr()), B, H, Tq, Tk, D, scale, stream) == 0
        assert lib.attn_prefix_fwd_split(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(kv.data_ptr()), C,
                                         P(po.data_ptr()), P(pl.data_ptr()), B, H, Tq, Tk, D, scale, stream) == 0
        assert lib.attn_lse_combine(P(po.data_ptr()), P(pl.data_ptr()), C, P(out.data_ptr()), P(lse.data_ptr()),
                                    B, H, Tq, D, stream) == 0
        assert lib.attn_prefix_fwd_split_fused(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(kv.data_ptr()),
                                               C, P(ws.data_ptr()), P(out.data_ptr()), P(lse.data_ptr()),
                                               B, H, Tq, Tk, D, scale, stream) == 0
        assert lib.attn_prefix_fwd_segments(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()),
                                            P(seg_start.data_ptr()), P(seg_len.data_ptr()), 2, P(seg_ws.data_ptr()),
                                            P(out.data_ptr()), P(lse.data_ptr()), B, H, Tq, Tk, D, scale,
                                            stream) == 0
        assert lib.attn_split_workspace_bytes(C, B, H, Tq, D) <= 64 * 1024 * 1024
        assert lib.attn_prefix_fwd_splitkv_noalloc(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()),
                                                   P(kv.data_ptr()), C, P(out.data_ptr()), P(lse.data_ptr()),
                                                   B, H, Tq, Tk, D, scale, stream) == 0

    calls()                      # warm-up: module and kernel loading
    before = _free_bytes()
    for _ in range(3):
        calls()
    after = _free_bytes()
    assert after == before, f"device free memory changed by {before - after} bytes"
    assert lib.attn_get_device_status(stream) == 0
