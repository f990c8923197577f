"""Comparison helpers shared by the GPU parity tests.

Tolerances: |out - ref| <= 1e-2 + 1e-2 |ref| per bf16 output element and
|lse - ref| <= 1e-3 absolute for the fp32 log-sum-exp; -inf must match exactly.
Split partials (fp32 outputs) use the same element bound.
"""
import numpy as np
import torch

OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_ATOL = 1e-3


def to_f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().float().cpu().double().numpy()


def assert_out_close(got, ref, what="out"):
    g = to_f64(got)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values at {np.argwhere(~np.isfinite(g))[:5]}"
    err = np.abs(g - r)
    bound = OUT_ATOL + OUT_RTOL * np.abs(r)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; first {idx.tolist()}; "
            f"worst at {worst}: got {g[worst]!r} ref {r[worst]!r}")


def assert_lse_close(got, ref, what="lse"):
    g = to_f64(got)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    ninf = np.isneginf(r)
    assert np.array_equal(np.isneginf(g), ninf), f"{what}: -inf pattern differs"
    fin = ~ninf
    assert np.isfinite(g[fin]).all(), f"{what}: non-finite where the oracle is finite"
    err = np.abs(g[fin] - r[fin])
    if err.size and err.max() > LSE_ATOL:
        raise AssertionError(f"{what}: max |diff| {err.max():.3e} > {LSE_ATOL} "
                             f"({int((err > LSE_ATOL).sum())} rows)")


def bits_equal(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bit-for-bit equality (NaN patterns included)."""
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)
