"""B200-native (sm_100a) prefix-masked attention forward.

    out, lse = attn_prefix_fwd(q, k, v, kv_len)          # single pass
    out, lse = attn_prefix_fwd_splitkv(q, k, v, kv_len, num_splits=64)      # split + combine
    out, lse = attn_prefix_fwd_split_fused(q, k, v, kv_len, num_splits=64)  # one launch
    out, lse = attn_prefix_fwd_segments(q, k, v, seg_start, seg_len)        # multi-range keys

q, k, v: bf16 CUDA tensors [B, H, T, D] with D in {32, 64, 128, 256} and d contiguous (the
single-pass, split and combine calls take other strides as given, so [B, T, H, D] views
and slices of a packed QKV run without copies; the fused-split and multi-range calls want
contiguous tensors); kv_len: int32 CUDA tensor [B] of valid key counts (keys at or beyond
kv_len[b] never take part).
The computation runs in the hand-written kernels of the C library built from csrc/;
this package only marshals arguments.
"""
from . import sharded  # noqa: F401  (key-sharded attention across ranks)
from ._binding import (  # noqa: F401
    AttnError,
    ATTN_OK,
    ATTN_ERR_INVALID_ARG,
    ATTN_ERR_UNSUPPORTED,
    ATTN_ERR_CUDA,
    ATTN_ERR_TIMEOUT,
    ATTN_ERR_KVLEN_RANGE,
    ATTN_DEBUG_DROP_COPY,
    SUPPORTED_HEAD_DIMS,
    LIB_PATH,
    device_status,
    fwd as attn_prefix_fwd,
    fwd_split as attn_prefix_fwd_split,
    fwd_splitkv as attn_prefix_fwd_splitkv,
    fwd_split_fused as attn_prefix_fwd_split_fused,
    fwd_segments as attn_prefix_fwd_segments,
    fused_workspace,
    lib,
    lse_combine as attn_lse_combine,
    set_debug_flags,
    set_wait_limit_ns,
    split_chunk_len,
    status_string,
    version,
)
