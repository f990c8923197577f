"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/attn_prefix.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_prefix.h")


@pytest.fixture(scope="module")
def lib():
    from key_prefix_masked_b200 import build
    build.build()
    from key_prefix_masked_b200 import _binding
    return _binding.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("attn_prefix_fwd", "attn_prefix_fwd_split", "attn_lse_combine",
                     "attn_split_workspace_bytes", "attn_get_device_status",
                     "attn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"{name} declared in the header but not exported"


def test_binding_covers_every_declared_symbol():
    from key_prefix_masked_b200 import _binding
    assert set(_declared_functions()) == set(_binding._SIGNATURES)


# Fake but well-aligned device addresses: every call below must fail a host check
# before any CUDA call could dereference them.
A = ctypes.c_void_p(0x10000)
NULL = ctypes.c_void_p(0)


def _fwd(lib, q=A, k=A, v=A, kv=A, out=A, lse=NULL, B=1, H=1, Tq=8, Tk=8, D=64, scale=0.125):
    return lib.attn_prefix_fwd(q, k, v, kv, out, lse, B, H, Tq, Tk, D, scale, NULL)


@pytest.mark.parametrize("kw,want", [
    (dict(q=NULL), 1), (dict(k=NULL), 1), (dict(v=NULL), 1), (dict(kv=NULL), 1),
    (dict(out=NULL), 1),
    (dict(q=ctypes.c_void_p(0x10008)), 1),          # not 16-byte aligned
    (dict(kv=ctypes.c_void_p(0x10002)), 1),         # kv_len not 4-byte aligned
    (dict(B=0), 1), (dict(H=-1), 1), (dict(Tq=0), 1), (dict(Tk=0), 1),
    (dict(B=65536, H=65536), 1),                    # B*H overflows int32
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1),
    (dict(D=96), 2), (dict(D=48), 2), (dict(D=0), 2),
])
def test_fwd_rejects_bad_arguments(lib, kw, want):
    assert _fwd(lib, **kw) == want


def test_split_and_combine_reject_bad_arguments(lib):
    f = lib.attn_prefix_fwd_split
    assert f(A, A, A, A, 0, A, A, 1, 1, 8, 8, 64, 0.1, NULL) == 1        # num_splits 0
    assert f(A, A, A, A, 1025, A, A, 1, 1, 8, 8, 64, 0.1, NULL) == 1     # > 1024
    assert f(A, A, A, A, 4, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1     # no part_lse
    assert f(A, A, A, A, 4, A, A, 1, 1, 8, 8, 96, 0.1, NULL) == 2        # head dim
    c = lib.attn_lse_combine
    assert c(NULL, A, 4, A, NULL, 1, 1, 8, 64, NULL) == 1
    assert c(A, A, 0, A, NULL, 1, 1, 8, 64, NULL) == 1
    assert c(A, A, 4, A, NULL, 1, 1, 8, 100, NULL) == 2
    assert c(A, A, 4, ctypes.c_void_p(0x10004), NULL, 1, 1, 8, 64, NULL) == 1


def test_split_geometry(lib):
    # ceil(Tk / C) rounded up to the 128-key tile
    assert lib.attn_split_chunk_len(1000000, 64) == 15744
    assert lib.attn_split_chunk_len(128, 1) == 128
    assert lib.attn_split_chunk_len(129, 1) == 256
    assert lib.attn_split_chunk_len(100, 7) == 128
    assert lib.attn_split_chunk_len(0, 4) == 0
    assert lib.attn_split_chunk_len(10, 0) == 0
    C, B, H, Tq, D = 64, 1, 8, 1024, 256
    off = lib.attn_split_lse_offset(C, B, H, Tq, D)
    assert off == C * B * H * Tq * D * 4 and off % 256 == 0
    assert lib.attn_split_workspace_bytes(C, B, H, Tq, D) == off + C * B * H * Tq * 4
    assert lib.attn_split_lse_offset(3, 1, 1, 5, 32) == ((3 * 5 * 32 * 4 + 255) // 256) * 256


def test_status_strings(lib):
    names = [lib.attn_status_string(i).decode() for i in range(6)]
    assert names == ["ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA",
                     "ATTN_ERR_TIMEOUT", "ATTN_ERR_KVLEN_RANGE"]
    assert lib.attn_status_string(99).decode() == "ATTN_ERR_UNKNOWN"
    assert lib.attn_version() >= 100


def test_product_fails_loudly_without_library(tmp_path, monkeypatch):
    from key_prefix_masked_b200 import _binding
    monkeypatch.setattr(_binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_binding, "_lib", None)
    with pytest.raises(ImportError):
        _binding.lib()


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "key_prefix_masked_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"\b(import|from)\s+oracle\b|attn_oracle|liboracle", text), fn


def test_fused_split_geometry_and_argument_checks(lib):
    C, B, H, Tq, D = 64, 1, 8, 1024, 256
    ws = lib.attn_split_workspace_bytes(C, B, H, Tq, D)
    off = lib.attn_split_counter_offset(C, B, H, Tq, D)
    assert off >= ws and off % 256 == 0 and off - ws < 256
    # one int32 counter per 128-row query tile of every (b, h)
    assert lib.attn_split_fused_workspace_bytes(C, B, H, Tq, D) == off + B * H * 8 * 4
    assert lib.attn_split_fused_workspace_bytes(3, 2, 3, 300, 64) == \
        lib.attn_split_counter_offset(3, 2, 3, 300, 64) + 2 * 3 * 3 * 4
    assert lib.attn_split_fused_workspace_bytes(0, 1, 1, 8, 64) == 0
    f = lib.attn_prefix_fwd_split_fused
    assert f(A, A, A, A, 4, NULL, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1        # no workspace
    assert f(A, A, A, A, 4, ctypes.c_void_p(0x10008), A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1  # misaligned
    assert f(A, A, A, A, 0, A, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1           # num_splits 0
    assert f(A, A, A, A, 4, A, NULL, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1        # no out
    assert f(A, A, A, A, 4, A, A, NULL, 1, 1, 8, 8, 96, 0.1, NULL) == 2           # head dim


def test_segments_geometry_and_argument_checks(lib):
    B, H, Tk, D = 2, 3, 1000, 64
    kv = ((B * H * Tk * D * 2 + 255) // 256) * 256
    assert lib.attn_segments_workspace_bytes(B, H, Tk, D) == 2 * kv + 256
    assert lib.attn_segments_workspace_bytes(0, H, Tk, D) == 0
    f = lib.attn_prefix_fwd_segments
    #          q  k  v  st len S  ws   out  lse   B  H  Tq Tk  D  scale stream
    assert f(A, A, A, A, A, 0, A, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1       # no segments
    assert f(A, A, A, A, A, 4097, A, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1    # too many
    assert f(A, A, A, A, NULL, 2, A, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1    # no seg_len
    assert f(A, A, A, NULL, A, 2, A, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1    # no seg_start
    assert f(A, A, A, A, A, 2, NULL, A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1    # no workspace
    assert f(A, A, A, A, A, 2, ctypes.c_void_p(0x10004), A, NULL, 1, 1, 8, 8, 64, 0.1, NULL) == 1
    assert f(A, A, A, A, A, 2, A, A, NULL, 1, 1, 8, 8, 96, 0.1, NULL) == 2       # head dim


class _Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("t", ctypes.c_int64)]


def test_strided_entries_check_strides(lib):
    f = lib.attn_prefix_fwd_strided
    ok = _Strides(8 * 64 * 64, 64, 8 * 64)          # a [B,T,H,D] layout with H=8, D=64
    bad_align = _Strides(8 * 64 * 64, 60, 8 * 64)   # h stride not a multiple of 8
    bad_row = _Strides(8 * 64 * 64, 64, 32)         # t stride shorter than a row
    neg = _Strides(-8, 64, 8 * 64)
    for s in (bad_align, bad_row, neg):
        for pos in range(4):
            args = [NULL] * 4
            args[pos] = ctypes.c_void_p(ctypes.addressof(s))
            assert f(A, A, A, A, A, NULL, 1, 8, 8, 8, 64, 0.1, *args, NULL) == 1
    del ok
    g = lib.attn_prefix_fwd_split_strided
    assert g(A, A, A, A, 4, A, A, 1, 8, 8, 8, 64, 0.1, ctypes.c_void_p(ctypes.addressof(bad_row)),
             NULL, NULL, NULL) == 1
    c = lib.attn_lse_combine_strided
    assert c(A, A, 4, A, NULL, 1, 8, 8, 64, ctypes.c_void_p(ctypes.addressof(bad_align)), NULL) == 1
