"""Sharing one layer's attention heads out over ranks.

Every (batch, head) pair of the method is independent: selection is per head (one KV head per
query head, no cross-head term in the pooled scores, the selection or the attention), so a layer
splits over GPUs by head with no data exchange (FastVideo API docs, fastvideo.attention.backends
page, ``abstract``: the backend sees ``[B, L, heads, D]`` and the sequence-parallel wrapper hands it
whole heads). Each rank passes its own head range (``head0``, ``heads``) of the same full-width
``[B, L, heads_total, D]`` rows to the library; the ranges of all ranks tile ``0 .. heads_total - 1``
and each rank writes only its heads' columns of the output.
"""
from __future__ import annotations


def head_partition(heads_total: int, world: int, rank: int) -> tuple[int, int]:
    """``(head0, heads)`` of ``rank``: contiguous ranges, the first ``heads_total % world`` ranks one
    head longer, so the per-rank head counts differ by at most one. A rank beyond the head count
    gets an empty range ``(heads_total, 0)``."""
    if world < 1 or not 0 <= rank < world or heads_total < 0:
        raise ValueError(f"bad partition request: {heads_total} heads, world {world}, rank {rank}")
    base, extra = divmod(heads_total, world)
    heads = base + (1 if rank < extra else 0)
    head0 = rank * base + min(rank, extra)
    return (head0, heads) if heads > 0 else (heads_total, 0)
