"""Key-sharded attention across ranks: each rank holds a shard of the keys.

This is the sequence-parallel scheme of "Add sequence-parallel multi-GPU inference ...",
section "Sequence-parallel inference". Every device runs an fp32 online softmax over
its own key shard. The partial results are then combined exactly by log-sum-exp
weights, so unequal shards need nothing special. Here:

  1. ``local_partial``: on this rank's keys (the first ``kv_len_local[b]`` rows of its
     shard), the normalised partial output O_r (fp32) and its log-sum-exp lse_r. This
     is one split-KV chunk of the prefix kernel (attn_prefix_fwd_split with C = 1).
  2. ``gather_partials``: (O_r, lse_r) of every rank, stacked in rank order
     ([world, B, H, Tq, D] and [world, B, H, Tq]), by an all-gather over the process
     group (NCCL over NVLink between GPUs).
  3. ``combine``: out = sum_r exp(lse_r - lse) O_r with lse = logsumexp_r lse_r
     (attn_lse_combine). An empty shard has lse_r = -inf and weight 0.

``key_sharded_fwd`` runs the three steps; every rank returns the full (out, lse).
Queries are replicated on every rank: the pages shard only the keys here.

Query rows need no exchange at all (each row's softmax is independent of the others):
``query_rows`` gives rank r its contiguous block of rows, and every rank keeps the full
keys.  ``key_bounds`` and ``shard_kv_len`` give rank r its contiguous block of keys and
the valid prefix inside it.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding


def query_rows(Tq: int, rank: int, world: int):
    """Rank `rank`'s contiguous block [r0, r1) of the Tq query rows; blocks differ in
    size by at most one row, and together cover every row once."""
    base, extra = divmod(Tq, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def key_bounds(Tk: int, rank: int, world: int, align: int = 128):
    """Rank `rank`'s contiguous block [k0, k1) of the Tk key slots: blocks of whole
    `align`-key tiles (the last one ragged), possibly empty when Tk is small."""
    tiles = -(-Tk // align)
    t0, t1 = query_rows(tiles, rank, world)
    return min(Tk, t0 * align), min(Tk, t1 * align)


def shard_kv_len(kv_len, k0: int, k1: int):
    """The valid keys of each batch element that fall in the block [k0, k1): a prefix of
    the block, of length clamp(kv_len[b] - k0, 0, k1 - k0)."""
    return [max(0, min(int(n) - k0, k1 - k0)) for n in kv_len]


def local_partial(q, k_local, v_local, kv_len_local, scale=None, num_splits=1):
    """This rank's normalised partial outputs and log-sum-exps over its own keys, in
    `num_splits` chunks of the shard: fp32 [C, B, H, Tq, D] and [C, B, H, Tq]."""
    return _binding.fwd_split(q, k_local, v_local, kv_len_local, num_splits, scale)


def gather_partials(part_out, part_lse, group=None):
    """All ranks' partials stacked in rank order along dim 0 ([world * C, ...]); the
    inputs are this rank's [C, ...] partials (C the same on every rank)."""
    world = dist.get_world_size(group)
    if world == 1:
        return part_out, part_lse
    outs = [torch.empty_like(part_out) for _ in range(world)]
    lses = [torch.empty_like(part_lse) for _ in range(world)]
    dist.all_gather(outs, part_out.contiguous(), group=group)
    dist.all_gather(lses, part_lse.contiguous(), group=group)
    return torch.cat(outs, dim=0), torch.cat(lses, dim=0)


def combine(part_out, part_lse, out=None, lse=None):
    """Exact log-sum-exp combination of stacked partials: (out bf16, lse fp32)."""
    return _binding.lse_combine(part_out, part_lse, out=out, lse=lse)


def key_sharded_fwd(q, k_local, v_local, kv_len_local, scale=None, group=None, num_splits=1, out=None,
                    lse=None):
    """Attention of the replicated queries q over the keys of all ranks' shards.

    k_local, v_local: this rank's [B, H, Tk_r, D] shard; kv_len_local: int32 [B], the
    valid keys at the front of the shard (0 for an empty shard).  All ranks must pass
    the same q, scale, head dim and num_splits (the chunks each rank cuts its shard
    into, so that a short query block still fills the GPU).  Returns (out bf16
    [B,H,Tq,D], lse fp32 [B,H,Tq]).
    """
    po, pl = local_partial(q, k_local, v_local, kv_len_local, scale, num_splits)
    po, pl = gather_partials(po, pl, group)
    return combine(po, pl, out=out, lse=lse)
