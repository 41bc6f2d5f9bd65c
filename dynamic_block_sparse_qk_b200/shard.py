"""Partition of one prefill over GPUs by KV-head groups.

Every stage of the path (proxy map, routing, selection, attention) reads
only a query head and its KV head, so a problem with H_kv KV heads splits
into N contiguous groups of H_kv / N KV heads, each with its g = H_q / H_kv
query heads, with no exchange between the parts: rank r runs the unchanged
library calls on its slice, and the outputs of the ranks, concatenated
along the head axis, are the outputs of the whole problem.
"""
from __future__ import annotations


def kv_head_range(h_kv: int, world: int, rank: int) -> range:
    """The KV heads rank ``rank`` of ``world`` owns (contiguous, equal parts)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if h_kv % world:
        raise ValueError(f"{h_kv} KV heads do not split evenly over {world} ranks")
    per = h_kv // world
    return range(rank * per, (rank + 1) * per)


def q_head_range(h_q: int, h_kv: int, world: int, rank: int) -> range:
    """The query heads that go with kv_head_range: g per KV head."""
    g = h_q // h_kv
    kv = kv_head_range(h_kv, world, rank)
    return range(kv.start * g, kv.stop * g)
