"""KV-head sharding of one attention layer across ranks (one process per GPU).

The selection, the attention and the rectification of a GQA group read only
that group's keys, values, descriptors and query heads ("Rectified Sparse
Attention", section "What carries the argument": each group pools its own
queries and picks its own blocks), so the groups of a layer can be split
across GPUs with no exchange inside the decode path: rank i holds KV heads
[h0, h1) of every cache and query heads [h0 G, h1 G), calls the library on
those local tensors, and produces those heads' outputs. Gathering the heads
afterwards (or a sharded output projection) belongs to the model around this
path, not to it.
"""
from __future__ import annotations


def kv_head_range(n_kv_heads: int, rank: int, world: int) -> tuple[int, int]:
    """KV heads [h0, h1) owned by `rank`: contiguous ranges whose sizes differ
    by at most one, covering every head once. Needs 1 <= world <= n_kv_heads."""
    if not (1 <= world <= n_kv_heads) or not (0 <= rank < world):
        raise ValueError(f"cannot split {n_kv_heads} KV heads over {world} ranks (rank {rank})")
    base, extra = divmod(n_kv_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def q_head_range(n_q_heads: int, n_kv_heads: int, rank: int, world: int) -> tuple[int, int]:
    """Query heads [h0 G, h1 G) that read the rank's KV heads (G = Hq / Hkv)."""
    G = n_q_heads // n_kv_heads
    h0, h1 = kv_head_range(n_kv_heads, rank, world)
    return h0 * G, h1 * G
