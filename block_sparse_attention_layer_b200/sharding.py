"""Splitting one VMoBA layer's heads across GPUs (one process per GPU).

VMoBA notes, key design 2: every head has its own global pool of
(query, block) pairs, its own threshold and its own attention, so a layer's
heads are independent problems.  Head sharding gives each rank a contiguous
range of heads and runs the unchanged layer on them: no collective exists
inside the layer.  (In a DiT the projections around the attention are where
ranks exchange data; that is the caller's model code, not this library.)

Each rank holds its heads' Q, K, V (and dO) contiguous as
[s][local heads][head_dim]: the library's layout with n_heads = the local
count, exactly what a head-parallel QKV projection produces.
"""
from __future__ import annotations

from dataclasses import replace

from ._lib import LayerShape


def head_range(rank: int, world: int, n_heads: int) -> tuple[int, int]:
    """Heads [h0, h1) of ``rank`` among ``world`` ranks: contiguous ranges,
    sizes differing by at most one, lower ranks taking the larger share.
    Ranks beyond n_heads get an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n_heads < 0:
        raise ValueError("n_heads must be >= 0")
    base, extra = divmod(n_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def local_shape(shape: LayerShape, rank: int, world: int) -> LayerShape | None:
    """The layer shape a rank runs: the same latent and boxes with its share of
    the heads, or None if it owns no head."""
    h0, h1 = head_range(rank, world, shape.n_heads)
    if h1 == h0:
        return None
    return replace(shape, n_heads=h1 - h0)


def take_heads(x, rank: int, world: int, n_heads: int):
    """The rank's heads of a [s][n_heads][d] tensor or array, contiguous."""
    h0, h1 = head_range(rank, world, n_heads)
    part = x[:, h0:h1]
    return part.contiguous() if hasattr(part, "contiguous") else part.copy()
