"""Head sharding of one layer over ranks (one process per GPU, no exchange inside the layer).

Every stage of the layer is independent across heads: packing and pooling act per
head, the gate G is shared by all heads and the TripPool projections W_q[h], W_k[h]
are per head, the top-k runs per (head, query tile), and attention never mixes
heads (Veda news page, "Что делает Veda": head-aware tiles and top-k; BSAI
VedaSparse README, "Core Technology: Head-Aware Tiling"). So rank r of n runs the
whole layer on a contiguous block of heads, with the replicated G, its own slice of
W_q / W_k and its heads' k, and no collective on the data path. In a full model the
exchange would sit outside the layer: the all-to-all that turns sequence-sharded
activations into head-sharded ones and back.
"""
from __future__ import annotations


def partition_heads(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [start, stop) of `rank`: contiguous blocks, the first heads % world ranks one larger."""
    if heads < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad partition: {heads} heads, world {world}, rank {rank}")
    if world > heads:
        raise ValueError(f"{world} ranks cannot each hold one of {heads} heads")
    base, extra = divmod(heads, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_config(cfg, start: int, stop: int):
    """The layer config of heads [start, stop): same grid, prefix, scorer and sparsity."""
    return cfg.with_(heads=stop - start, tile_shapes=tuple(cfg.tile_shapes[start:stop]))


def shard_k(k_per_head, start: int, stop: int) -> list:
    return list(k_per_head)[start:stop]


def shard_heads_of(x, start: int, stop: int, axis: int):
    """Heads [start, stop) of a token-major [B, N, heads, d] tensor (axis 2) or of per-head
    projections [heads, 3d, p] (axis 0), as a contiguous copy."""
    idx = [slice(None)] * x.ndim
    idx[axis] = slice(start, stop)
    y = x[tuple(idx)]
    return y.contiguous() if hasattr(y, "contiguous") else y.copy()
