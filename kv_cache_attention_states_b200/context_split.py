"""Decode with each sequence's context split across ranks (one per GPU).

Rank r holds positions [key_begin_r, key_begin_r + capacity) of every
sequence, the ranks' ranges in rank order.  Each rank computes the
partial-softmax record of its shard (attn_decode_partial), one all-gather
exchanges the records (8 heads x 258 floats per sequence, ~8 KiB), and every
rank merges them in rank order (attn_merge_partials), so all ranks hold the
same output bits.  The exchange is a few KiB per step: latency-bound, one
NCCL call.
"""
import torch
import torch.distributed as dist

from . import attn_decode_partial, attn_merge_partials, partial_floats


def exchange_partials(part, group=None):
    """All-gather of this rank's partial record: returns [world, n] in rank
    order (NCCL: one all_gather_into_tensor; other backends: all_gather)."""
    world = dist.get_world_size(group)
    gathered = torch.empty((world, part.numel()), dtype=part.dtype, device=part.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(gathered, part.reshape(-1), group=group)
    else:
        dist.all_gather(list(gathered.unbind(0)), part.reshape(-1), group=group)
    return gathered


def decode_context_split(q, k_shard, v_shard, ctx_len, key_begin: int, window: int = 0,
                         scale: float = 1.0 / 16.0, group=None, workspace=None, stream=None):
    """attn_decode of the whole context from this rank's shard and the other
    ranks' records; q and ctx_len are the same on every rank."""
    batch = q.shape[0]
    part = attn_decode_partial(q, k_shard, v_shard, ctx_len, key_begin, window, scale,
                               workspace=workspace, stream=stream)
    parts = exchange_partials(part, group)
    assert parts.shape[1] == partial_floats(batch)
    return attn_merge_partials(parts, batch, stream=stream)
