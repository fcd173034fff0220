"""Region packing and budget counts (oracle).

Region packing — DraftAttention2 reading note, Figure 3(a) caption and Method
overview bullet 1: each frame's token grid is cut into compact 2-D spatial
regions, each region becomes one contiguous block, and cells a region does not
cover are padding.  The pages give no order; the reading adopted here:

* region rows nRy = ceil(Hh / rh), region columns nRx = ceil(Ww / rw), so every
  frame is padded up to a multiple of the region size in both y and x;
* block id = (t * nRy + ry) * nRx + rx (frame-major, then region row, then
  region column);
* slot s = i * rw + j inside a block holds token (t, ry * rh + i, rx * rw + j),
  or is a padding slot when that y >= Hh or x >= Ww.

Budget counts — the reading note's Method overview bullet 2 and its experiment
section: each head has one budget given as 0/4/8/16 percentages of its region
pairs.  Reading adopted: the percentages are taken in permille
(q = round(10 * pct)), cumulated in precision order 16 → 8 → 4, and each
cumulative count is rounded half up, c = floor((P * cum + 500) / 1000).  The
skip count is what remains, so a budget summing to 99.9 % (80.7/14.4/4.8/0)
skips 80.8 %.
"""

from __future__ import annotations

import numpy as np


def block_tokens(p) -> np.ndarray:
    """int64 [nb, rh*rw]: original token index of every slot, -1 for padding."""
    table = np.full((p.nb, p.rh * p.rw), -1, dtype=np.int64)
    for t in range(p.T):
        for ry in range(p.nry):
            for rx in range(p.nrx):
                blk = (t * p.nry + ry) * p.nrx + rx
                for i in range(p.rh):
                    for j in range(p.rw):
                        y = ry * p.rh + i
                        x = rx * p.rw + j
                        if y < p.Hh and x < p.Ww:
                            table[blk, i * p.rw + j] = (t * p.Hh + y) * p.Ww + x
    return table


def permille(pct: float) -> int:
    return int(np.rint(10.0 * float(pct)))


def budget_counts(p):
    """(n16, n8, n4, nskip) region pairs per head for P = nb^2 pairs."""
    P = p.nb * p.nb
    _skip, b4, b8, b16 = (permille(x) for x in p.budget)
    cum16 = b16
    cum8 = b16 + b8
    cum4 = b16 + b8 + b4
    if cum4 > 1000 or min(b4, b8, b16) < 0:
        raise ValueError("budget: 4/8/16-bit shares must be >= 0 and sum to <= 100 %")

    def c(cum):
        return (P * cum + 500) // 1000

    c16, c8, c4 = c(cum16), c(cum8), c(cum4)
    return c16, c8 - c16, c4 - c8, P - c4
