"""The whole hot path, stage by stage, on the CPU (oracle).

prep (reorder + pool + quantise) → draft map → shared ranking and assignment →
mixed-precision attention → restore to token order: the pipeline of the
DraftAttention2 reading note's Figure 2 and Method overview.
"""

from __future__ import annotations

import numpy as np

from . import attention, draft, prep, rank
from .geometry import block_tokens, budget_counts


def to_f64(t):
    """bf16 torch tensor (any device) → fp64 numpy (exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_head(p, qh, kh, vh, mode="emulate", prec_map=None, scores=None,
             qblocks=None, table=None):
    """One (batch, head).  ``prec_map`` / ``scores`` override the oracle's own
    assignment / fp32 scores (stage-wise parity).  Returns a dict."""
    if table is None:
        table = block_tokens(p)
    pr = prep.prepare_head(p, qh, kh, vh, table)
    D = draft.draft_scores(pr["q_avg"], pr["k_avg"], pr["q_max"], pr["k_max"], p.lam, p.d)
    n16, n8, n4, _ = budget_counts(p)
    if prec_map is None:
        prec_map = rank.assign(D if scores is None else scores, n16, n8, n4)
    blk = attention.head_attention(pr, prec_map, p.d, mode, qblocks)
    out = attention.scatter(blk, table, p.N) if qblocks is None else None
    return {"prep": pr, "scores": D, "map": prec_map, "block_out": blk, "out": out}


def run(p, q, k, v, mode="emulate"):
    """Full output [B, H, N, d] (fp64) and the per-head intermediates."""
    table = block_tokens(p)
    out = np.zeros((p.B, p.H, p.N, p.d))
    heads = {}
    for b in range(p.B):
        for h in range(p.H):
            r = run_head(p, q[b, h], k[b, h], v[b, h], mode, table=table)
            out[b, h] = r["out"]
            heads[(b, h)] = r
    return out, heads
