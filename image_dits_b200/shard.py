"""Splitting one attention call over GPUs by heads.

Every head of a call is an independent problem (the permutation, the mask of
"RainFusion2.0" section 3.2 and the block-sparse attention of section 3.1 are
all per (batch, head)), so a call's heads can be divided among GPUs with no
exchange at all: rank r runs heads [h0, h1) through the same library calls on
a geometry with h1 - h0 heads, and the outputs, concatenated along the head
axis, are those of the whole call.
"""
from __future__ import annotations


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` among `world` ranks: contiguous ranges whose
    sizes differ by at most one, covering 0 .. heads - 1 once.  Every rank
    gets at least one head, so `world` may not exceed `heads`."""
    if not (1 <= world <= heads):
        raise ValueError(f"cannot split {heads} heads over {world} ranks")
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside 0..{world - 1}")
    return heads * rank // world, heads * (rank + 1) // world
