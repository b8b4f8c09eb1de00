"""Head sharding of one attention layer over several GPUs.

Every step of the path (permutation, TripPool, scores, top-k, attention, tile
map, KL, recall) works on each head on its own: a head has its own tiling,
scorer, mask and attention (Veda summary 2.1-2.3). A layer's heads therefore
split over ranks with no exchange at all: rank r runs the unchanged library
on its contiguous block of heads, and the whole layer is the union of the
ranks' outputs. Host logic only; no collective is part of the data path.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def head_ranges(n_heads: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous, balanced [h0, h1) blocks covering heads 0..n_heads-1 once;
    the first n_heads % world ranks take one head more. Ranks beyond the head
    count get empty blocks."""
    if n_heads < 0 or world < 1:
        raise ValueError("n_heads >= 0 and world >= 1 are required")
    base, extra = divmod(n_heads, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def local_heads(global_heads: Sequence[int], h0: int, h1: int) -> List[int]:
    """The rank-local indices of those of `global_heads` that fall in [h0, h1)."""
    return [h - h0 for h in global_heads if h0 <= h < h1]
