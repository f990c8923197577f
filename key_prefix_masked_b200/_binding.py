"""ctypes binding of the C ABI declared in include/attn_prefix.h.

Argument marshalling only: torch provides device memory and the current stream; every
step of the computation runs in the library's sm_100a kernels.  If the compiled library
is missing, importing the functions raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libattn_prefix.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4
ATTN_ERR_KVLEN_RANGE = 5
ATTN_DEBUG_DROP_COPY = 1

SUPPORTED_HEAD_DIMS = (32, 64, 128, 256)

# Every symbol the header exports, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SIGNATURES = {
    "attn_prefix_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_prefix_fwd_strided": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P, _P]),
    "attn_prefix_fwd_split_strided": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "attn_lse_combine_strided": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P, _P]),
    "attn_split_chunk_len": (_I, [_I, _I]),
    "attn_split_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_split_lse_offset": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_prefix_fwd_split": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_lse_combine": (_I, [_P, _P, _I, _P, _P, _I, _I, _I, _I, _P]),
    "attn_split_counter_offset": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_split_fused_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I, _I]),
    "attn_prefix_fwd_split_fused": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_segments_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "attn_prefix_fwd_segments": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_prefix_fwd_splitkv_noalloc": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _F, _P]),
    "attn_get_device_status": (_I, [_P]),
    "attn_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "attn_set_debug_flags": (None, [ctypes.c_uint]),
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_version": (_I, []),
}

_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"CUDA library not built: {LIB_PATH} is missing "
                    "(run `python -m key_prefix_masked_b200.build` or __graft_entry__.build())")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, where)


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


class _Strides(ctypes.Structure):
    """attn_strides: element strides along b, h, t of a [B,H,T,D] operand (d contiguous)."""
    _fields_ = [("b", ctypes.c_int64), ("h", ctypes.c_int64), ("t", ctypes.c_int64)]


def _strides_of(t):
    """The attn_strides of a [B,H,T,D] view whose last dim is contiguous."""
    sb, sh, st, sd = t.stride()
    if sd != 1:
        raise ValueError("the head dim must be contiguous (stride 1)")
    return _Strides(sb, sh, st)


def _strided_ok(t):
    return t.dim() == 4 and t.stride(3) == 1 and all(x % 8 == 0 for x in t.stride()[:3])


def _check_qkv(q, k, v, kv_len, strided=False):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4:
            raise ValueError(f"{name} must be a bf16 CUDA tensor [B,H,T,D]")
        if not (t.is_contiguous() or (strided and _strided_ok(t))):
            raise ValueError(f"{name} must be contiguous, or a [B,H,T,D] view with a contiguous head dim "
                             "and strides that are multiples of 8 elements")
    B, H, Tq, D = q.shape
    if k.shape[:2] != (B, H) or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("k and v must be [B,H,Tk,D] matching q's B, H, D")
    if kv_len is not None and (not kv_len.is_cuda or kv_len.dtype != torch.int32 or kv_len.numel() != B
                               or not kv_len.is_contiguous()):
        raise ValueError("kv_len must be a contiguous int32 CUDA tensor of B entries")
    if len({q.device, k.device, v.device} | ({kv_len.device} if kv_len is not None else set())) != 1:
        raise ValueError("all tensors must be on one device")
    return int(B), int(H), int(Tq), int(k.shape[2]), int(D)


def fwd(q, k, v, kv_len, scale=None, out=None, lse=None, need_lse=True):
    """Prefix-masked attention forward (attn_prefix_fwd): returns (out bf16, lse fp32).

    q, k, v (and out, if given) may be [B,H,T,D] views of other layouts, e.g.
    x.transpose(1, 2) of a [B,T,H,D] tensor: their strides go to attn_prefix_fwd_strided.
    A new out takes q's layout."""
    B, H, Tq, Tk, D = _check_qkv(q, k, v, kv_len, strided=True)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    elif (out.shape != q.shape or out.dtype != torch.bfloat16 or out.device != q.device
          or not (out.is_contiguous() or _strided_ok(out))):
        raise ValueError("out must be a bf16 [B,H,Tq,D] tensor on q's device with a contiguous head dim")
    if lse is None and need_lse:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        if all(t.is_contiguous() for t in (q, k, v, out)):
            st = lib().attn_prefix_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), _ptr(out), _ptr(lse),
                                       B, H, Tq, Tk, D, scale, _stream_ptr(q.device))
        else:
            s4 = [_strides_of(t) for t in (q, k, v, out)]
            st = lib().attn_prefix_fwd_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), _ptr(out), _ptr(lse),
                                               B, H, Tq, Tk, D, scale, *[ctypes.addressof(x) for x in s4],
                                               _stream_ptr(q.device))
    _check(st, "attn_prefix_fwd")
    return out, lse


def split_chunk_len(Tk: int, num_splits: int) -> int:
    return int(lib().attn_split_chunk_len(int(Tk), int(num_splits)))


def fwd_split(q, k, v, kv_len, num_splits, scale=None, part_out=None, part_lse=None):
    """Split-KV partials (attn_prefix_fwd_split): fp32 part_out [C,B,H,Tq,D], part_lse [C,B,H,Tq]."""
    B, H, Tq, Tk, D = _check_qkv(q, k, v, kv_len, strided=True)
    C = int(num_splits)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if part_out is None:
        part_out = torch.empty((C, B, H, Tq, D), dtype=torch.float32, device=q.device)
    if part_lse is None:
        part_lse = torch.empty((C, B, H, Tq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        if all(t.is_contiguous() for t in (q, k, v)):
            st = lib().attn_prefix_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), C, _ptr(part_out),
                                             _ptr(part_lse), B, H, Tq, Tk, D, scale,
                                             _stream_ptr(q.device))
        else:
            s3 = [_strides_of(t) for t in (q, k, v)]
            st = lib().attn_prefix_fwd_split_strided(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), C, _ptr(part_out),
                                                     _ptr(part_lse), B, H, Tq, Tk, D, scale,
                                                     *[ctypes.addressof(x) for x in s3], _stream_ptr(q.device))
    _check(st, "attn_prefix_fwd_split")
    return part_out, part_lse


def lse_combine(part_out, part_lse, out=None, lse=None, need_lse=True):
    """Exact LSE combination of split partials (attn_lse_combine): (out bf16, lse fp32)."""
    if part_out.dtype != torch.float32 or part_lse.dtype != torch.float32:
        raise ValueError("partials must be fp32")
    if not (part_out.is_contiguous() and part_lse.is_contiguous()):
        raise ValueError("partials must be contiguous")
    C, B, H, Tq, D = (int(s) for s in part_out.shape)
    if tuple(part_lse.shape) != (C, B, H, Tq):
        raise ValueError("part_lse must be [C,B,H,Tq]")
    if out is None:
        out = torch.empty((B, H, Tq, D), dtype=torch.bfloat16, device=part_out.device)
    elif (tuple(out.shape) != (B, H, Tq, D) or out.dtype != torch.bfloat16 or out.device != part_out.device
          or not (out.is_contiguous() or _strided_ok(out))):
        raise ValueError("out must be a bf16 [B,H,Tq,D] tensor with a contiguous head dim")
    if lse is None and need_lse:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=part_out.device)
    with torch.cuda.device(part_out.device):
        if out.is_contiguous():
            st = lib().attn_lse_combine(_ptr(part_out), _ptr(part_lse), C, _ptr(out), _ptr(lse),
                                        B, H, Tq, D, _stream_ptr(part_out.device))
        else:
            so = _strides_of(out)
            st = lib().attn_lse_combine_strided(_ptr(part_out), _ptr(part_lse), C, _ptr(out), _ptr(lse),
                                                B, H, Tq, D, ctypes.addressof(so), _stream_ptr(part_out.device))
    _check(st, "attn_lse_combine")
    return out, lse


def fwd_splitkv(q, k, v, kv_len, num_splits, scale=None, workspace=None):
    """Split-KV forward: partials over num_splits key chunks, then the LSE combine."""
    part_out, part_lse = fwd_split(q, k, v, kv_len, num_splits, scale,
                                   *(workspace if workspace is not None else (None, None)))
    return lse_combine(part_out, part_lse)


def fused_workspace(num_splits, B, H, Tq, D, device):
    """A zeroed workspace for fwd_split_fused (partials + tile counters), as uint8."""
    n = int(lib().attn_split_fused_workspace_bytes(int(num_splits), int(B), int(H), int(Tq), int(D)))
    if n == 0:
        raise ValueError("invalid split shape")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def fwd_split_fused(q, k, v, kv_len, num_splits, scale=None, workspace=None, out=None, lse=None,
                    need_lse=True):
    """Split-KV forward with the combine fused into the launch (attn_prefix_fwd_split_fused).

    `workspace` (from fused_workspace, reusable: the kernel leaves its counters zero) is
    allocated and zeroed here when not given.  Returns (out bf16, lse fp32)."""
    B, H, Tq, Tk, D = _check_qkv(q, k, v, kv_len)
    C = int(num_splits)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if workspace is None:
        workspace = fused_workspace(C, B, H, Tq, D, q.device)
    need = int(lib().attn_split_fused_workspace_bytes(C, B, H, Tq, D))
    if (not workspace.is_cuda or workspace.device != q.device or not workspace.is_contiguous()
            or workspace.numel() * workspace.element_size() < need):
        raise ValueError(f"workspace must be a contiguous CUDA buffer of at least {need} bytes")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib().attn_prefix_fwd_split_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), C, _ptr(workspace),
                                               _ptr(out), _ptr(lse), B, H, Tq, Tk, D, scale,
                                               _stream_ptr(q.device))
    _check(st, "attn_prefix_fwd_split_fused")
    return out, lse


def fwd_segments(q, k, v, seg_start, seg_len, scale=None, workspace=None, out=None, lse=None,
                 need_lse=True):
    """Multi-range key mask (attn_prefix_fwd_segments): batch element b attends to the keys
    of its segments [seg_start[b, s], seg_start[b, s] + seg_len[b, s]).

    seg_start, seg_len: contiguous int32 CUDA tensors [B, S].  `workspace` (uint8, at least
    attn_segments_workspace_bytes) is allocated here when not given.  Returns (out, lse)."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, T, D]")
    B = int(q.shape[0])
    for t, name in ((seg_start, "seg_start"), (seg_len, "seg_len")):
        if (not t.is_cuda or t.dtype != torch.int32 or t.dim() != 2 or int(t.shape[0]) != B
                or not t.is_contiguous() or t.device != q.device):
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor [B, S] on q's device")
    if seg_start.shape != seg_len.shape:
        raise ValueError("seg_start and seg_len must have the same shape")
    S = int(seg_start.shape[1])
    B, H, Tq, Tk, D = _check_qkv(q, k, v, None)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    need = int(lib().attn_segments_workspace_bytes(B, H, Tk, D))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if (not workspace.is_cuda or workspace.device != q.device or not workspace.is_contiguous()
            or workspace.numel() * workspace.element_size() < need):
        raise ValueError(f"workspace must be a contiguous CUDA buffer of at least {need} bytes")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and need_lse:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib().attn_prefix_fwd_segments(_ptr(q), _ptr(k), _ptr(v), _ptr(seg_start), _ptr(seg_len), S,
                                            _ptr(workspace), _ptr(out), _ptr(lse), B, H, Tq, Tk, D, scale,
                                            _stream_ptr(q.device))
    _check(st, "attn_prefix_fwd_segments")
    return out, lse


def device_status(device=None) -> int:
    """Synchronizes the current stream and returns (and clears) the sticky device flags."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib().attn_get_device_status(_stream_ptr(dev)))


def set_wait_limit_ns(ns: int) -> None:
    lib().attn_set_wait_limit_ns(int(ns))


def set_debug_flags(flags: int) -> None:
    lib().attn_set_debug_flags(int(flags))


def version() -> int:
    return int(lib().attn_version())
