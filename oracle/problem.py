"""Problem statement of one attention call, as the oracle reads it.

Q, K, V are [B, H, N, d] with N = T * Hh * Ww tokens of a latent video grid,
token n = (t * Hh + y) * Ww + x.  The grid is cut into rh x rw spatial
regions per frame (DraftAttention2 reading note, Method overview, bullet 1;
Figure 3(a): compact regions, padding cells grey).  ``budget`` is
(skip, 4-bit, 8-bit, 16-bit) in percent, the "Bit" column order of the
reading note's experiment section.  ``lam`` is the weight of the max-pooled
draft map (Method overview, bullet 1).
"""

from __future__ import annotations

import dataclasses
import math


@dataclasses.dataclass(frozen=True)
class Problem:
    B: int
    H: int
    T: int
    Hh: int
    Ww: int
    d: int
    lam: float
    budget: tuple  # (skip, 4-bit, 8-bit, 16-bit) percent
    rh: int = 8
    rw: int = 8

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.Ww

    @property
    def nry(self) -> int:
        return math.ceil(self.Hh / self.rh)

    @property
    def nrx(self) -> int:
        return math.ceil(self.Ww / self.rw)

    @property
    def nb(self) -> int:
        return self.T * self.nry * self.nrx

    @property
    def S(self) -> int:
        """Tokens per region block (64 for 8x8 regions)."""
        return self.rh * self.rw

    @classmethod
    def from_workload(cls, wl, **kw) -> "Problem":
        p = cls(wl.B, wl.H, wl.T, wl.Hh, wl.Ww, wl.d, wl.lam, tuple(wl.budget),
                wl.rh, wl.rw)
        return dataclasses.replace(p, **kw) if kw else p


def _load_configs():
    from mixed_precision_block_b200.synth import WORKLOADS
    return {k: Problem.from_workload(w) for k, w in WORKLOADS.items()}


CONFIGS = _load_configs()
