"""GPU parity on seeded random problems: shape, head dim, key lengths, value spread,
scale, call (single pass, split + combine, fused split, [B,T,H,D] views) all drawn from
one generator per case, each compared with the fp64 oracle.

The fixed sweeps cover the edges one at a time; this one mixes them, so that a
combination nobody listed (a ragged tail inside a split chunk of a two-group kernel with
a negative scale, say) is exercised too.  Every case is small enough for the oracle to
finish in well under a second.
"""
import math

import pytest
import torch

import oracle
import synth
from parity import assert_lse_close, assert_out_close

pytestmark = pytest.mark.gpu

N_CASES = 160


@pytest.fixture(scope="module")
def kp():
    from key_prefix_masked_b200 import build
    build.build()
    import key_prefix_masked_b200 as kp
    torch.cuda.init()
    assert kp.device_status() == kp.ATTN_OK
    return kp


def draw(seed):
    g = torch.Generator().manual_seed(90001 + seed)
    ri = lambda lo, hi: int(torch.randint(lo, hi + 1, (1,), generator=g))  # noqa: E731
    D = (32, 64, 128, 256)[ri(0, 3)]
    B, H = ri(1, 3), ri(1, 2)
    Tq, Tk = ri(1, 400), ri(1, 1500)
    lens = []
    for _ in range(B):
        kind = ri(0, 5)
        lens.append(0 if kind == 0 else Tk if kind == 1 else ri(1, Tk))
    std = (0.5, 1.0, 2.0)[ri(0, 2)]
    scale_kind = ri(0, 5)
    scale = (1.0 / math.sqrt(D)) if scale_kind < 4 else (-0.1 if scale_kind == 4 else 0.0)
    mode = ("single", "split", "fused", "view")[ri(0, 3)]
    splits = ri(2, 9)
    return dict(D=D, B=B, H=H, Tq=Tq, Tk=Tk, lens=tuple(lens), std=std, scale=scale, mode=mode, splits=splits)


@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_problem(kp, seed):
    p = draw(seed)
    case = synth.random_case(p["B"], p["H"], p["Tq"], p["Tk"], p["D"], p["lens"], seed=seed, std=p["std"])
    case["scale"] = p["scale"]
    q, k, v = (case[n].cuda() for n in ("q", "k", "v"))
    kv = case["kv_len"].cuda()
    if p["mode"] == "single":
        out, lse = kp.attn_prefix_fwd(q, k, v, kv, p["scale"])
    elif p["mode"] == "split":
        po, pl = kp.attn_prefix_fwd_split(q, k, v, kv, p["splits"], p["scale"])
        out, lse = kp.attn_lse_combine(po, pl)
    elif p["mode"] == "fused":
        out, lse = kp.attn_prefix_fwd_split_fused(q, k, v, kv, p["splits"], p["scale"])
    else:
        # [B, T, H, D] storage seen as [B, H, T, D] views (strided entry points)
        qv, kv_, vv = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))
        assert not qv.is_contiguous() or p["H"] == 1 or p["Tq"] == 1
        out, lse = kp.attn_prefix_fwd(qv, kv_, vv, kv, p["scale"])
    torch.cuda.synchronize()
    assert kp.device_status() == kp.ATTN_OK, p
    ref_out, ref_lse = oracle.attn_prefix(case["q"], case["k"], case["v"], case["kv_len_list"], p["scale"])
    assert_out_close(out, ref_out, what=str(p))
    assert_lse_close(lse, ref_lse, what=str(p))
