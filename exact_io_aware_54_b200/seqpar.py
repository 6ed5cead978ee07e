"""Sequence-parallel attention across the ranks of a process group (one GPU each).

Every rank holds all queries and one contiguous shard of the keys and values, the
shards equal in length and in rank order (the multi-GPU extension the second page
wishes for, "AI Bible 13", section 06).  The forward runs attention over the local
shard (causal shards see the bottom-right boundary of the whole sequence),
exchanges the partial (O, lse) of all shards over the group (NCCL all-gather: the
one exchange step) and merges them with the block-merge rule ("FlashAttention
saves IO, not N^2 work", sections 3 and 7) in the library's merge kernel.  The
backward needs no merge: attention's backward over the local shard with the
merged O and lse gives that shard's dK and dV exactly and a partial dQ; the
partial dQ are summed over the group (NCCL all-reduce, in at least fp32).

The per-shard attention and the merge are parameters (the library's calls by
default), so the exchange logic can be exercised on CPU ranks with other
implementations of the same calls.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fa_bwd, fa_bwd_shard, fa_fwd, fa_fwd_shard, fa_merge_partials


def _shard_extent(k_shard, group):
    """(key_offset, Nk_total) of this rank's shard: equal shards in rank order."""
    n = k_shard.shape[1]
    return dist.get_rank(group) * n, dist.get_world_size(group) * n


def _default_attn(softmax_scale):
    def attn(q, k, v, causal, key_offset, nk_total):
        if causal:
            return fa_fwd_shard(q, k, v, key_offset, nk_total, softmax_scale=softmax_scale)
        return fa_fwd(q, k, v, causal=False, softmax_scale=softmax_scale)
    return attn


def _default_attn_bwd(softmax_scale):
    def attn_bwd(q, k, v, o, dout, lse, causal, key_offset, nk_total):
        if causal:
            return fa_bwd_shard(q, k, v, o, dout, lse, key_offset, nk_total, softmax_scale=softmax_scale)
        return fa_bwd(q, k, v, o, dout, lse, causal=False, softmax_scale=softmax_scale)
    return attn_bwd


def sequence_parallel_fwd(q, k_shard, v_shard, causal: bool = False, group=None, softmax_scale=None, attn=None,
                          merge=None):
    """q [B, Nq, H, d] (the same on every rank), k_shard / v_shard [B, Nk_r, H, d]
    (this rank's keys).  Returns the merged (o [B, Nq, H, d], lse [B, H, Nq]) on
    every rank."""
    attn = attn or _default_attn(softmax_scale)
    merge = merge or fa_merge_partials
    key_offset, nk_total = _shard_extent(k_shard, group)
    o_s, lse_s = attn(q, k_shard, v_shard, causal, key_offset, nk_total)
    world = dist.get_world_size(group)
    # gathered along dim 0 (the form every backend takes), then seen as [world, ...]:
    # for contiguous tensors the two layouts are the same memory
    o_s, lse_s = o_s.contiguous(), lse_s.contiguous()
    o_all = torch.empty((world * o_s.shape[0],) + tuple(o_s.shape[1:]), dtype=o_s.dtype, device=o_s.device)
    lse_all = torch.empty((world * lse_s.shape[0],) + tuple(lse_s.shape[1:]), dtype=lse_s.dtype,
                          device=lse_s.device)
    dist.all_gather_into_tensor(o_all, o_s, group=group)
    dist.all_gather_into_tensor(lse_all, lse_s, group=group)
    return merge(o_all.view((world,) + tuple(o_s.shape)), lse_all.view((world,) + tuple(lse_s.shape)))


def sequence_parallel_bwd(q, k_shard, v_shard, o, dout, lse, causal: bool = False, group=None, softmax_scale=None,
                          attn_bwd=None):
    """Gradients of sum(O * dout) for sequence_parallel_fwd: o and lse are its merged
    results.  Returns (dq [B, Nq, H, d], the same on every rank; dk_shard, dv_shard for
    this rank's keys)."""
    attn_bwd = attn_bwd or _default_attn_bwd(softmax_scale)
    key_offset, nk_total = _shard_extent(k_shard, group)
    dq, dk, dv = attn_bwd(q, k_shard, v_shard, o, dout, lse, causal, key_offset, nk_total)
    # the partial dQ are summed in at least fp32 (bf16 partials are widened first)
    acc = dq.float() if dq.dtype in (torch.bfloat16, torch.float16) else dq.clone()
    dist.all_reduce(acc, group=group)
    return acc.to(dq.dtype), dk, dv
