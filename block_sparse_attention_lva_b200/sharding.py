"""Head sharding of one attention layer across ranks (one process per GPU).

Every (batch, head, query block) row of block-sparse attention depends only on its own
head's Q, K and V and on the block mask, so one layer splits into contiguous head ranges
with no exchange on the data path: rank r computes heads [h0, h1) of every batch element
from its own slice of Q, K and V, and the mask is replicated -- the one shared CSR of a
parametric mask is built on every rank, and a per-head static mask or repetitive-head map
contributes its rows h0..h1-1.  The outputs of the ranks are the unsharded layer's outputs
for their heads, bit for bit (the same kernels compute the same rows).
"""
from __future__ import annotations

from .pipeline import VideoBlockSparseAttention


def head_range(H: int, world: int, rank: int):
    """Heads [h0, h1) of ``rank`` among ``world`` ranks: contiguous ranges in rank order whose
    sizes differ by at most one (the first H % world ranks take one more head).  A rank past
    the number of heads gets an empty range."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"need 0 <= rank < world, got rank {rank} of {world}")
    if H < 0:
        raise ValueError("H must be >= 0")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_rows(table, h0: int, h1: int):
    """The rows of a per-head table ([H, ...]) for heads [h0, h1); a table shared by every
    head ([1, ...]) is replicated unchanged."""
    if table is None or table.shape[0] == 1:
        return table
    return table[h0:h1]


class HeadShard:
    """One rank's part of a block-sparse attention layer: heads [h0, h1) of H.

    Constructed from the layer's full description (``static_mask`` and ``query_src`` with
    their rows for all H heads, or one shared row); runs ``VideoBlockSparseAttention`` on the
    rank's heads.  Inputs and outputs are the rank's head slices: Q, K, V raster
    [B, h1 - h0, N, d] -> O raster [B, h1 - h0, N, d] and LSE [B, h1 - h0, n_pad].
    """

    def __init__(self, B, H, d, grid, tile, block_size, mask: dict, world: int, rank: int, static_mask=None,
                 scale=None, device="cuda", query_src=None):
        self.h0, self.h1 = head_range(H, world, rank)
        if self.h1 <= self.h0:
            raise ValueError(f"rank {rank} of {world} has no heads of {H}")
        self.layer = VideoBlockSparseAttention(B, self.h1 - self.h0, d, grid, tile, block_size, mask,
                                               static_mask=shard_rows(static_mask, self.h0, self.h1),
                                               scale=scale, device=device,
                                               query_src=shard_rows(query_src, self.h0, self.h1))

    def __call__(self, q, k, v, step: int = 0):
        return self.layer(q, k, v, step=step)
