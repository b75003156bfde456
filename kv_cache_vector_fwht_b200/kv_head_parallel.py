"""KV-head-parallel decode: one process per GPU, each holding a contiguous range of every
sequence's KV heads in its own KVCache.

Attention of a query head reads only its own KV head, so a partition by KV head needs no
exchange at all: each rank decodes the query heads whose KV head it holds, through the same
fused decode, with the head map renumbered to its local KV heads. This module holds the host
logic of that partition (which KV heads and which query heads a rank owns, the local head
map) and the rank-local call; assembling the ranks' outputs, if a caller wants them in one
place, is an ordinary gather of (batch, local query heads, d) blocks.
"""
from __future__ import annotations

from . import tq_decode_attention


def kv_head_slice(n_kv_heads: int, rank: int, world: int) -> tuple[int, int]:
    """KV heads [start, stop) of `rank` when n_kv_heads are split into `world` contiguous
    ranges whose sizes differ by at most one (the first n_kv_heads mod world are longer)."""
    if world < 1 or not 0 <= rank < world or n_kv_heads < 0:
        raise ValueError("need 0 <= rank < world and n_kv_heads >= 0")
    base, extra = divmod(n_kv_heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def default_head_map(n_q_heads: int, n_kv_heads: int) -> list[int]:
    """Query head h reads KV head h // (n_q_heads / n_kv_heads) (grouped-query attention)."""
    if n_kv_heads <= 0 or n_q_heads % n_kv_heads:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    g = n_q_heads // n_kv_heads
    return [h // g for h in range(n_q_heads)]


def local_heads(head_map, kv_start: int, kv_stop: int) -> tuple[list[int], list[int]]:
    """The query heads whose KV head lies in [kv_start, kv_stop), in ascending order, and
    their head map over the rank's local KV heads (KV head kv -> kv - kv_start)."""
    qs = [h for h, kv in enumerate(head_map) if kv_start <= int(kv) < kv_stop]
    return qs, [int(head_map[h]) - kv_start for h in qs]


def kv_head_parallel_decode(q, cache, query, out, workspace, kv_start: int, kv_stop: int,
                            head_map=None, sm_scale: float = 0.0, stream=None):
    """Rank-local decode of a KV-head partition. `cache` holds KV heads [kv_start, kv_stop)
    of every sequence (cache.n_kv_heads == kv_stop - kv_start); `query` is the full (batch,
    n_q_heads, d) query, the same on every rank; `head_map` is the global map (None: grouped
    -query default over n_kv_heads = the global count implied by the map). Writes the
    attention output of the rank's query heads to `out` (batch, len(local query heads), d)
    and returns those query heads' global indices."""
    n_q = query.shape[1]
    if head_map is None:
        raise ValueError("pass the global head map (default_head_map(n_q_heads, n_kv_heads))")
    if len(head_map) != n_q:
        raise ValueError("head_map needs one entry per query head")
    if cache.n_kv_heads != kv_stop - kv_start:
        raise ValueError("cache must hold exactly KV heads [kv_start, kv_stop)")
    qs, lmap = local_heads(head_map, kv_start, kv_stop)
    if not qs:
        return qs
    q_local = query[:, qs].contiguous()
    tq_decode_attention(q, cache, q_local, out, workspace, head_map=lmap, sm_scale=sm_scale,
                        stream=stream)
    return qs
