"""ctypes front end of the fp64 C oracle (attn_oracle.c).

TEST INFRASTRUCTURE ONLY.  Argument marshalling lives here; every number comes from the
C code, which follows the plain definition of scaled-dot-product attention with a
per-batch key prefix ("Rewrite prefix key-padding masks as k/v truncation ...", sections
"Problem" and "Fix") and the exact log-sum-exp combination of key shards ("Add
sequence-parallel multi-GPU inference ...", section "Sequence-parallel inference").

Inputs are bf16 tensors or uint16 arrays of bf16 bit patterns, laid out [B, H, T, D]
row-major.  Outputs are float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile attn_oracle.c with gcc (-O2, OpenMP, no fast-math); returns the .so path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            path = build_oracle()
            lib = ctypes.CDLL(path)
            p = ctypes.c_void_p
            i = ctypes.c_int
            lib.oracle_attn_prefix.argtypes = [p, p, p, p, i, i, i, i, i, ctypes.c_double,
                                               p, i, p, p]
            lib.oracle_attn_prefix.restype = i
            lib.oracle_attn_chunk.argtypes = [p, p, p, p, i, i, i, i, i, ctypes.c_double,
                                              p, i, ctypes.c_long, ctypes.c_long, p, p]
            lib.oracle_attn_chunk.restype = i
            lib.oracle_attn_masked.argtypes = [p, p, p, p, i, i, i, i, i, ctypes.c_double,
                                               p, p]
            lib.oracle_attn_masked.restype = i
            lib.oracle_lse_combine.argtypes = [p, p, i, ctypes.c_long, i, p, p]
            lib.oracle_attn_segments.argtypes = [p, p, p, p, p, i, i, i, i, i, i, ctypes.c_double,
                                                 p, i, p, p]
            lib.oracle_attn_segments.restype = i
            lib.oracle_lse_combine.restype = i
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i
            lib.oracle_set_num_threads.argtypes = [i]
            lib.oracle_set_num_threads.restype = None
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _bits(x) -> np.ndarray:
    """bf16 tensor (any device) or uint16 array -> contiguous uint16 numpy array."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("numpy inputs must be uint16 bf16 bit patterns")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError(f"expected a bf16 tensor, got {x.dtype}")
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _shape4(q, k):
    B, H, Tq, D = (int(s) for s in q.shape)
    Bk, Hk, Tk, Dk = (int(s) for s in k.shape)
    if (Bk, Hk, Dk) != (B, H, D):
        raise ValueError("q and k/v must agree on B, H, D")
    return B, H, Tq, Tk, D


def _rows_arg(rows, Tq):
    if rows is None:
        return None, Tq
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, int(r.size)


def attn_prefix(q, k, v, kv_len, scale: float, rows=None):
    """Truncation mode: out[b,h,r,:], lse[b,h,r] over keys j < kv_len[b].

    rows: optional query-row indices evaluated for every (b, h); default all rows.
    Returns (out float64 [B,H,R,D], lse float64 [B,H,R]).
    """
    lib = _load()
    B, H, Tq, Tk, D = _shape4(q, k)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    kl = np.ascontiguousarray(np.asarray(_to_numpy(kv_len), dtype=np.int32))
    if kl.size != B:
        raise ValueError("kv_len must have B entries")
    r, R = _rows_arg(rows, Tq)
    out = np.empty((B, H, R, D), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    rc = lib.oracle_attn_prefix(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(kl), B, H, Tq, Tk, D,
                                float(scale), None if r is None else _ptr(r), R,
                                _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_prefix rejected its arguments")
    return out, lse


def attn_segments(q, k, v, seg_start, seg_len, scale: float, rows=None):
    """Multi-range key mask: batch element b attends to the concatenation of its segments
    [seg_start[b][s], seg_start[b][s] + seg_len[b][s]) (each cut to [0, Tk), negative
    lengths as 0, the concatenation cut after Tk keys).  seg_start, seg_len: [B, S] ints.
    Returns (out float64 [B,H,R,D], lse float64 [B,H,R])."""
    lib = _load()
    B, H, Tq, Tk, D = _shape4(q, k)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    st = np.ascontiguousarray(np.asarray(_to_numpy(seg_start), dtype=np.int32))
    ln = np.ascontiguousarray(np.asarray(_to_numpy(seg_len), dtype=np.int32))
    if st.ndim != 2 or st.shape[0] != B or st.shape != ln.shape:
        raise ValueError("seg_start and seg_len must both be [B, S]")
    S = int(st.shape[1])
    r, R = _rows_arg(rows, Tq)
    out = np.empty((B, H, R, D), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    rc = lib.oracle_attn_segments(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(st), _ptr(ln), S, B, H, Tq, Tk, D,
                                  float(scale), None if r is None else _ptr(r), R, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_segments rejected its arguments")
    return out, lse


def attn_chunk(q, k, v, kv_len, scale: float, key_begin: int, key_end: int, rows=None):
    """One key chunk [key_begin, key_end) intersected with the prefix: (O_c, lse_c)."""
    lib = _load()
    B, H, Tq, Tk, D = _shape4(q, k)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    kl = np.ascontiguousarray(np.asarray(_to_numpy(kv_len), dtype=np.int32))
    r, R = _rows_arg(rows, Tq)
    out = np.empty((B, H, R, D), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    rc = lib.oracle_attn_chunk(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(kl), B, H, Tq, Tk, D,
                               float(scale), None if r is None else _ptr(r), R,
                               int(key_begin), int(key_end), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_chunk rejected its arguments")
    return out, lse


def attn_masked(q, k, v, mask, scale: float):
    """Dense-mask mode over all Tk keys with a [B, Tk] boolean key mask (finite padding)."""
    lib = _load()
    B, H, Tq, Tk, D = _shape4(q, k)
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    m = np.ascontiguousarray(np.asarray(_to_numpy(mask), dtype=np.uint8).reshape(B, Tk))
    out = np.empty((B, H, Tq, D), dtype=np.float64)
    lse = np.empty((B, H, Tq), dtype=np.float64)
    rc = lib.oracle_attn_masked(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(m), B, H, Tq, Tk, D,
                                float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attn_masked rejected its arguments")
    return out, lse


def lse_combine(part_out, part_lse):
    """Exact LSE combination of C partials: part_out [C, ..., D], part_lse [C, ...]."""
    lib = _load()
    po = np.ascontiguousarray(np.asarray(part_out, dtype=np.float64))
    pl = np.ascontiguousarray(np.asarray(part_lse, dtype=np.float64))
    C = int(po.shape[0])
    D = int(po.shape[-1])
    rows = int(pl.size // C)
    if po.size != C * rows * D:
        raise ValueError("part_out / part_lse shapes disagree")
    out = np.empty(po.shape[1:], dtype=np.float64)
    lse = np.empty(pl.shape[1:], dtype=np.float64)
    rc = lib.oracle_lse_combine(_ptr(po), _ptr(pl), C, rows, D, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_lse_combine rejected its arguments")
    return out, lse


def _to_numpy(x):
    if isinstance(x, np.ndarray):
        return x
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x)
