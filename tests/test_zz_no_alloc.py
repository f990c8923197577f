"""The split-KV entry point that allocates nothing (attn_prefix_fwd_splitkv_noalloc).

It serves callers that cannot call cudaMalloc themselves -- code that only receives its
inputs and outputs from a framework allocator or a fixed memory plan.  Its partials live
in the library's own device array, so the test checks, through the C ABI, that two calls
in a row (the second reusing whatever the first left in that array) give what the
existing allocate-your-own-workspace split-KV path gives, and what the fp64 oracle
gives, within the parity tolerance.  Empty and one-key prefixes are among the rows.

The file name sorts after every other test file, so a run that stops at its first
failure has run all the other tests before this one.  Nothing here depends on that
order: the test passes alone in a fresh process and after the others.
"""
import ctypes

import pytest
import torch

import oracle
import synth
from parity import assert_lse_close, assert_out_close

SCRATCH_BYTES = 64 * 1024 * 1024


@pytest.fixture(scope="module")
def lib():
    from key_prefix_masked_b200 import build
    build.build()
    from key_prefix_masked_b200 import _binding
    return _binding.lib()


def _call(lib, g, C, out, lse):
    B, H, Tq, D = g["q"].shape
    Tk = g["k"].shape[2]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.attn_prefix_fwd_splitkv_noalloc(
        ctypes.c_void_p(g["q"].data_ptr()), ctypes.c_void_p(g["k"].data_ptr()),
        ctypes.c_void_p(g["v"].data_ptr()), ctypes.c_void_p(g["kv_len"].data_ptr()), C,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(0 if lse is None else lse.data_ptr()),
        B, H, Tq, Tk, D, g["scale"], stream)


def test_oversized_workspace_is_rejected_before_any_cuda_call(lib):
    A = ctypes.c_void_p(0x10000)
    # 64 splits x 8 heads x 1024 rows x (256 + 1) floats is ~539 MB > 64 MiB
    st = lib.attn_prefix_fwd_splitkv_noalloc(A, A, A, A, 64, A, A, 1, 8, 1024, 1000000, 256,
                                             0.0625, ctypes.c_void_p(0))
    assert st == 1
    need = lib.attn_split_workspace_bytes(64, 1, 8, 1024, 256)
    assert need > SCRATCH_BYTES


@pytest.mark.gpu
def test_noalloc_matches_split_kv_path_on_two_calls(lib):
    import key_prefix_masked_b200 as kp
    cases = [
        # first call: larger footprint; the next ones are smaller and reuse the array
        (synth.random_case(2, 4, 300, 3000, 256, (3000, 1111), seed=31, std=0.5), 6),
        (synth.random_case(3, 2, 130, 900, 64, (0, 1, 899), seed=32), 3),
        (synth.random_case(2, 3, 77, 500, 128, (129, 0), seed=33), 4),
        (synth.random_case(2, 2, 64, 96, 32, (40, 1), seed=34), 2),
    ]
    for case, C in cases:
        g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in case.items()}
        B, H, Tq, D = g["q"].shape
        assert lib.attn_split_workspace_bytes(C, B, H, Tq, D) <= SCRATCH_BYTES
        out = torch.full_like(g["q"], float("nan"))
        lse = torch.full((B, H, Tq), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(lib, g, C, out, lse) == 0
        ref_out, ref_lse = kp.attn_prefix_fwd_splitkv(g["q"], g["k"], g["v"], g["kv_len"], C,
                                                      g["scale"])
        torch.cuda.synchronize()
        assert kp.device_status() == kp.ATTN_OK
        assert_out_close(out, ref_out.double().cpu().numpy(), what="noalloc out vs split path")
        assert_lse_close(lse, ref_lse.double().cpu().numpy(), what="noalloc lse vs split path")
        o_out, o_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], case["kv_len_list"], case["scale"])
        assert_out_close(out, o_out, what="noalloc out vs oracle")
        assert_lse_close(lse, o_lse, what="noalloc lse vs oracle")
