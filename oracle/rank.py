"""Shared ranking and precision assignment (oracle).

DraftAttention2 abstract and reading note (Method overview, bullet 2): within
each head all region pairs are ranked by draft score once, and that one
ranking hands out the budget in order — the highest-scoring pairs get 16-bit,
the next INT8, the next the low-bit (NVFP4) format, and the rest are skipped.
A query region may therefore keep a different number of key regions, and a
different precision mix, than its neighbours under the same head budget.

Readings adopted: ranking is descending by the fp32 score; equal scores are
ordered by ascending pair index p = q_block * nb + k_block; -0 counts as +0.
The rank r(p) of a pair is its position in that order, and
r < n16 → 16-bit, r < n16 + n8 → 8-bit, r < n16 + n8 + n4 → 4-bit, else skip.
"""

from __future__ import annotations

import numpy as np

SKIP, BIT4, BIT8, BIT16 = 0, 4, 8, 16


def pair_ranks(D32):
    """int64 ranks [nb, nb] of every pair of one head (full sort)."""
    flat = np.asarray(D32, dtype=np.float32).ravel()
    if not np.all(np.isfinite(flat)):
        raise ValueError("draft scores must be finite")
    flat = flat + np.float32(0.0)  # -0 → +0
    idx = np.arange(flat.size)
    order = np.lexsort((idx, -flat.astype(np.float64)))
    ranks = np.empty(flat.size, dtype=np.int64)
    ranks[order] = idx
    return ranks.reshape(np.shape(D32))


def assign(D32, n16, n8, n4):
    """uint8 precision map [nb, nb] with values 16, 8, 4 or 0 (skip)."""
    r = pair_ranks(D32)
    out = np.zeros(r.shape, dtype=np.uint8)
    out[r < n16 + n8 + n4] = BIT4
    out[r < n16 + n8] = BIT8
    out[r < n16] = BIT16
    return out
