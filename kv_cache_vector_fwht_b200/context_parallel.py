"""Context-parallel decode: one process per GPU, each holding a contiguous slice of every
sequence's context in its own KVCache.

Each rank runs the fused decode over its slice and keeps the softmax partials instead of
normalising (tq_decode_attention_partial: per sequence and query head the base-2 maximum m,
the sum l and the unnormalised o). The records are all-gathered over the process group
(NCCL over NVLink between GPUs) and every rank merges them with tq_merge_partials, so that
each rank ends with the attention output over the whole context. This is the one exchange
that splitting a decode over the context needs: a record is 132 floats per (sequence, query
head), independent of the context length. Splitting by KV head or by sequence needs no
exchange at all; those are independent decodes.
"""
from __future__ import annotations

from . import TQ_PART_FLOATS, tq_decode_attention_partial, tq_merge_partials


def context_slice(n_tokens: int, rank: int, world: int) -> tuple[int, int]:
    """Token range [start, stop) of `rank` when n_tokens are split into `world` contiguous
    slices whose sizes differ by at most one (the first n_tokens mod world slices are
    longer)."""
    if world < 1 or not 0 <= rank < world or n_tokens < 0:
        raise ValueError("need 0 <= rank < world and n_tokens >= 0")
    base, extra = divmod(n_tokens, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_partials(part, group=None):
    """All-gather this rank's records (batch, n_q_heads, TQ_PART_FLOATS) into a contiguous
    (world, batch, n_q_heads, TQ_PART_FLOATS) tensor, rank r's records at index r."""
    import torch
    import torch.distributed as dist
    assert part.is_contiguous() and part.shape[-1] == TQ_PART_FLOATS
    world = dist.get_world_size(group)
    parts = torch.empty((world,) + tuple(part.shape), dtype=part.dtype, device=part.device)
    dist.all_gather(list(parts.unbind(0)), part, group=group)
    return parts


def context_parallel_decode(q, cache, query, out, workspace, group=None, head_map=None,
                            sm_scale: float = 0.0):
    """Attention output over the union of every rank's context slice, written to `out`
    (batch, n_q_heads, d) on every rank. `query` is the same on all ranks; `cache` holds
    this rank's slice (a cache with values); `workspace` as for tq_decode_attention. All
    three steps run on torch's current stream, which the collective is ordered against.
    Returns the gathered records (world, batch, n_q_heads, TQ_PART_FLOATS)."""
    import torch
    part = torch.empty((query.shape[0], query.shape[1], TQ_PART_FLOATS), dtype=torch.float32,
                       device=query.device)
    tq_decode_attention_partial(q, cache, query, part, workspace, head_map=head_map,
                                sm_scale=sm_scale)
    parts = gather_partials(part, group)
    tq_merge_partials(parts, out)
    return parts
