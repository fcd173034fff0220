"""Mixed-precision block-sparse attention (oracle).

DraftAttention2 abstract and reading note (Method overview, bullet 4): one
attention pass per query block runs a phase per precision; the phases share
the softmax statistics (running max and sum) and one output accumulator, and
quantisation scales are folded in at the phase boundaries, so no partial
outputs are written back and merged.  Skipped pairs contribute nothing.

This module follows that structure per query block, in fp64: phase 16, then
phase 8, then phase 4.  Every retained key block contributes a partial
(reference m_blk, sum l_blk, numerator x_blk) that is merged into one
online-softmax state (m, l, O); a low-bit phase gathers its blocks' numerators
in the units of its quantised operands and applies the V channel scale once,
at the phase boundary.  The result depends only on the query block's own
precision row: no block's contribution depends on another block's, so the
order in which blocks are visited (and any grouping a kernel uses) does not
change it beyond rounding.

Readings adopted (the pages leave these open):

* scores: 16-bit phase from the bf16 values; 8-bit phase from the exact
  integer product of the INT8 codes times both block scales; 4-bit phase from
  the dequantised NVFP4 values; all times 1/sqrt(d).  Padding keys score -inf.
* low-bit P is quantised per (query row, key block), relative to that block's
  own row maximum rounded up to a power of two: with x = s log2 e, the
  reference is r_blk = ceil(max x) and p = 2^(x - r_blk) in (0, 1].  Every
  retained block so keeps the full resolution of its format whatever its rank
  in the row (the reading note, Method overview bullet 3: low-bit precision
  recovers the mid-importance interactions), and since its scale 2^r_blk is a
  power of two, its weights enter the shared accumulator exactly, with no
  separate merge per block (bullet 4: the phases rescale at their boundaries
  and avoid repeated write-backs and merges):
  - 8-bit: code = round(255 p) as an unsigned byte; weights code/255 times
    2^r_blk;
  - 4-bit: NVFP4 of 2688 p over 16 consecutive keys of the row (2688 = 6 x 448
    puts the largest possible p at the top of the e2m1 x e4m3 range),
    dequantised and divided by 2688; weights that times 2^r_blk.  A power of
    two passes through the e4m3 scale exactly, so the same codes come out
    against any larger power-of-two reference while the microblock scale
    stays normal (>= 2^-6).
* the softmax denominator sums, per phase, the weights the numerator uses:
  unquantised p in the 16-bit phase, the quantised weights above in the
  low-bit phases (so each low-bit block enters numerator and denominator with
  the same weights and the output stays a weighted mean of V).
* 16-bit phase, ``emulate`` mode: P is rounded to bf16 relative to a power of
  two, 2^ceil(max x) over the block; bf16 rounding commutes with scaling by
  powers of two, so this is the rounding against any integer-exponent
  reference a kernel keeps (parity unpinned beyond that: the GPU's
  exponential).  ``math`` mode keeps P exact.
* ``emulate`` mode rounds the output to bf16; a query block with no retained
  key block outputs zeros.
"""

from __future__ import annotations

import numpy as np

from . import formats as F
from .rank import BIT4, BIT8, BIT16

LOG2E = 1.4426950408889634
LN2 = 0.6931471805599453
P4_RANGE = 2688.0  # 6 (largest e2m1) x 448 (largest e4m3)


def bf16_round(x):
    """fp64 → fp32 (RN) → bf16 (RN, ties to even), returned as fp64."""
    f = np.asarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


class _State:
    """Online-softmax state shared by every phase: per row a reference m, the
    sum l and the numerator O, both relative to exp(m)."""

    def __init__(self, rows, d):
        self.m = np.full(rows, -np.inf)
        self.l = np.zeros(rows)
        self.o = np.zeros((rows, d))

    def merge(self, m_blk, l_blk, x_blk):
        """Merge a partial whose weights were taken relative to exp(m_blk)."""
        m_new = np.maximum(self.m, m_blk)
        ok = np.isfinite(m_new)
        a_old = np.where(ok & np.isfinite(self.m), np.exp(self.m - np.where(ok, m_new, 0)), 0.0)
        a_blk = np.where(ok & np.isfinite(m_blk), np.exp(m_blk - np.where(ok, m_new, 0)), 0.0)
        self.l = self.l * a_old + l_blk * a_blk
        self.o = self.o * a_old[:, None] + x_blk * a_blk[:, None]
        self.m = m_new


def _row_max(s):
    return s.max(axis=1)


def _exp_rel(s, m):
    """exp(s - m) per row, 0 where s is -inf or the row has no finite score."""
    ok = np.isfinite(m)[:, None] & np.isfinite(s)
    return np.where(ok, np.exp(np.where(ok, s - np.where(np.isfinite(m), m, 0)[:, None], 0)), 0.0)


def _pow2_reference(x):
    """Per row: r = ceil(max x) (-inf for a row without a finite score) and
    p = 2^(x - r), 0 where x is -inf."""
    xm = _row_max(x)
    live = np.isfinite(xm)
    r_blk = np.where(live, np.ceil(np.where(live, xm, 0.0)), -np.inf)
    ok = np.isfinite(x) & live[:, None]
    p = np.where(ok, np.exp2(np.where(ok, x - np.where(live, r_blk, 0.0)[:, None], 0.0)), 0.0)
    return r_blk, p


def p8_weights(x):
    """8-bit phase weights of one key block (rows x keys, log2-unit scores,
    -inf for unused keys): returns (r_blk, w) with r_blk = ceil(row max) and
    w = round(255 * 2^(x - r_blk)) / 255 relative to 2^r_blk."""
    r_blk, p = _pow2_reference(x)
    return r_blk, np.rint(255.0 * p) / 255.0


def p4_weights(x):
    """4-bit phase weights of one key block (rows x keys, log2-unit scores,
    -inf for unused keys): returns (r_blk, w) with r_blk = ceil(row max) and
    w = NVFP4(2688 * 2^(x - r_blk)) / 2688 relative to 2^r_blk."""
    r_blk, p = _pow2_reference(x)
    t = F.f32(P4_RANGE * F.f32(p))
    codes, sf = F.nvfp4_quantize(t, axis=-1, block=16)
    return r_blk, F.nvfp4_dequantize(codes, sf) / P4_RANGE


def qblock_attention(prep, qb, prec_row, d, mode="emulate"):
    """Output rows [S, d] of query block ``qb`` of one head.

    ``prep``: dict from ``prep.prepare_head``; ``prec_row``: uint8 [nb] precision
    of each key block for this query block (16, 8, 4, 0)."""
    S = prep["q_blocks"].shape[1]
    valid = prep["valid"]
    inv_sqrt_d = 1.0 / np.sqrt(d)
    st = _State(S, d)

    # phase 16: bf16 operands; each block's P against its own power-of-two
    # reference (the rounding is the same against any integer exponent)
    q = prep["q_blocks"][qb]
    for kb in np.nonzero(prec_row == BIT16)[0]:
        s = (q @ prep["k_blocks"][kb].T) * inv_sqrt_d
        s = np.where(valid[kb][None, :], s, -np.inf)
        m_blk = _row_max(s)
        p = _exp_rel(s, m_blk)
        if mode == "emulate":
            live = np.isfinite(m_blk)
            xm = np.where(live, m_blk * LOG2E, 0.0)
            shift = np.exp2(np.ceil(xm) - xm)  # >= 1; exp(s - m_blk) = 2^(x - ceil) * shift
            p_num = bf16_round(p / shift[:, None]) * shift[:, None]
        else:
            p_num = p
        st.merge(m_blk, p.sum(1), p_num @ prep["v_blocks"][kb])

    # phase 8: INT8 Q/K codes with block scales; u8 P against each block's own
    # power-of-two reference; INT8 V codes; the V channel scale applied at the boundary
    kbs = np.nonzero(prec_row == BIT8)[0]
    if len(kbs):
        qi = prep["q_i8"][qb].astype(np.float64)
        sq = prep["q_s8"][qb]
        ph = _State(S, d)
        for kb in kbs:
            s_int = qi @ prep["k_i8"][kb].astype(np.float64).T  # exact integers
            x = np.where(valid[kb][None, :], s_int * (sq * prep["k_s8"][kb] * inv_sqrt_d * LOG2E), -np.inf)
            r_blk, w = p8_weights(x)
            ph.merge(r_blk * LN2, w.sum(1), w @ prep["v_i8"][kb].astype(np.float64).T)
        st.merge(ph.m, ph.l, ph.o * prep["v_s8"][None, :])

    # phase 4: NVFP4 Q/K, NVFP4 P (16-key microblocks of 2688 p against each
    # block's power-of-two reference), NVFP4 V; the V channel scale g at the boundary
    kbs = np.nonzero(prec_row == BIT4)[0]
    if len(kbs):
        qd = F.nvfp4_dequantize(prep["q_f4"][qb], prep["q_sf4"][qb])
        ph = _State(S, d)
        for kb in kbs:
            kd = F.nvfp4_dequantize(prep["k_f4"][kb], prep["k_sf4"][kb])
            x = np.where(valid[kb][None, :], (qd @ kd.T) * (inv_sqrt_d * LOG2E), -np.inf)
            r_blk, w = p4_weights(x)
            vt = F.nvfp4_dequantize(prep["v_f4"][kb], prep["v_sf4"][kb])  # [d, S] without g
            ph.merge(r_blk * LN2, w.sum(1), w @ vt.T)
        st.merge(ph.m, ph.l, ph.o * prep["v_g4"][None, :])

    out = np.where(st.l[:, None] > 0, st.o / np.where(st.l > 0, st.l, 1.0)[:, None], 0.0)
    return bf16_round(out) if mode == "emulate" else out


def head_attention(prep, prec_map, d, mode="emulate", qblocks=None):
    """Block-order output [nb, S, d] (rows of ``qblocks`` only, others zero)."""
    nb, S = prep["valid"].shape
    out = np.zeros((nb, S, d))
    for qb in (range(nb) if qblocks is None else qblocks):
        out[qb] = qblock_attention(prep, qb, prec_map[qb], d, mode)
    return out


def scatter(block_out, table, N):
    """Block order → original token order; padding rows are dropped.

    DraftAttention abstract: the reordered tokens are restored to their
    original order after attention."""
    d = block_out.shape[-1]
    out = np.zeros((N, d))
    valid = table >= 0
    out[table[valid]] = block_out[valid]
    return out


def dense_attention(q, k, v):
    """Plain fp64 softmax(q k^T / sqrt d) v over all tokens: [N, d] each."""
    s = (q @ k.T) / np.sqrt(q.shape[1])
    s = s - s.max(1, keepdims=True)
    p = np.exp(s)
    return (p @ v) / p.sum(1, keepdims=True)


def error_terms(prep, prec_map, d, qblocks):
    """Error decomposition of the method on the given query blocks of one head
    (DraftAttention2 abstract and reading note, Method overview: sparsity and
    quantisation are the two approximations; here they are measured apart).

    Returns relative L2 errors against exact dense attention over the real
    rows of the blocks, all in fp64 (``math`` mode, no output rounding):
      ``sparse``  exact attention restricted to the retained key blocks,
      ``quant``   the mixed-precision result minus that exact sparse result,
      ``total``   the mixed-precision result itself;
    so total <= sparse + quant (triangle inequality)."""
    valid = prep["valid"]
    kept = {BIT16, BIT8, BIT4}
    num_s = num_q = num_t = den = 0.0
    for qb in qblocks:
        row = prec_map[qb]
        mixed = qblock_attention(prep, qb, row, d, "math")
        exact_row = np.where(np.isin(row, list(kept)), BIT16, 0).astype(row.dtype)
        sparse = qblock_attention(prep, qb, exact_row, d, "math")
        dense = qblock_attention(prep, qb, np.full_like(row, BIT16), d, "math")
        rv = valid[qb]
        num_s += float(((sparse - dense)[rv] ** 2).sum())
        num_q += float(((mixed - sparse)[rv] ** 2).sum())
        num_t += float(((mixed - dense)[rv] ** 2).sum())
        den += float((dense[rv] ** 2).sum())
    den = max(den, 1e-300)
    return {"sparse": (num_s / den) ** 0.5, "quant": (num_q / den) ** 0.5, "total": (num_t / den) ** 0.5}
