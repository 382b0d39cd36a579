"""Split of block-sparse attention work across ranks (one process per GPU).

The (batch, kv head) slices of a block-sparse problem are independent in the forward and the
backward: a slice's queries read only its own keys and values, and its dK and dV sum only over the
slice's own group of query heads (BlockSparseAttentionGrad page, formulas; the GQA rule).  So
ranks take contiguous ranges of slices, balanced by the number of selected tiles each slice holds
(the metadata operator's per-core share of the task list, SparseAttnSharedkvMetadata page), and
no collective is needed on the data path.  This module turns a rank's range into the contiguous
pieces of the BNSD tensors it owns; the cut itself is the C library's bsa_partition."""
from __future__ import annotations

import numpy as np

from . import partition


def slice_weights(block_mask: np.ndarray, N2: int) -> np.ndarray:
    """Selected tiles per (batch, kv head) slice, int64 [B * N2] in (b, g) order: the nonzero
    entries of the BlockSparseMask rows of the slice's N1 / N2 query heads."""
    B, N1 = block_mask.shape[:2]
    return (block_mask.reshape(B, N2, -1) != 0).sum(axis=2, dtype=np.int64).reshape(-1)


def segments(starts: np.ndarray, rank: int, B: int, N2: int) -> list[tuple[int, int, int, int]]:
    """The rank's slices [starts[rank], starts[rank + 1]) as contiguous BNSD pieces
    (b0, b1, g0, g1): batches b0..b1-1 and kv heads g0..g1-1 (query heads g0*G..g1*G-1).  A piece is
    either part of one batch's heads or a run of whole batches, so each is one strided block of a
    BNSD tensor.  An empty range gives no pieces."""
    s0, s1 = int(starts[rank]), int(starts[rank + 1])
    out = []
    while s0 < s1:
        b, g = divmod(s0, N2)
        if g == 0 and s1 - s0 >= N2:  # a run of whole batches
            nb = (s1 - s0) // N2
            out.append((b, b + nb, 0, N2))
            s0 += nb * N2
        else:  # part of batch b
            g1 = min(N2, g + (s1 - s0))
            out.append((b, b + 1, g, g1))
            s0 += g1 - g
    return out


def split(block_mask: np.ndarray, N2: int, world: int, rank: int):
    """partition + segments for one rank: (starts, that rank's pieces)."""
    starts = partition(slice_weights(block_mask, N2), world)
    return starts, segments(starts, rank, block_mask.shape[0], N2)
