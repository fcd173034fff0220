"""Mixed-precision block-sparse attention (oracle).

DraftAttention2 abstract and reading note (Method overview, bullet 4): one
attention pass per query block runs a phase per precision; the phases share
the softmax statistics (running max and sum) and one output accumulator, and
quantisation scales are folded in at the phase boundaries, so no partial
outputs are written back and merged.  Skipped pairs contribute nothing.

This module follows that structure literally, per query block, in fp64:
phase 16, then phase 8, then phase 4, key blocks in ascending index inside each
phase, one online-softmax state (m, l, O) carried across all of them.

Readings adopted (the pages leave these open):

* scores: 16-bit phase from the bf16 values; 8-bit phase from the exact integer
  product of the INT8 codes times both block scales; 4-bit phase from the
  dequantised NVFP4 values; all times 1/sqrt(d).  Padding keys score -inf.
* P in the 8-bit and 4-bit phases is quantised relative to the per-row maximum
  m_blk of the key block it belongs to, p = exp(s - m_blk) in (0, 1]:
  8-bit code = round(255 p) as an unsigned byte (scale 1/255); 4-bit = NVFP4
  over 16 consecutive keys of the row.  The block's P·V is then weighted by
  exp(m_blk - m) when merged into the shared accumulator.
* the softmax denominator l sums the unquantised exp(s - m) over every retained
  real key of every phase.
* 16-bit phase, ``emulate`` mode: P is rounded to bf16 relative to a power of
  two, 2^r with r = ceil(m_run * log2 e) and m_run the running maximum over the
  16-bit blocks seen so far (ascending key blocks).  Because bf16 rounding
  commutes with scaling by powers of two, the rounded P is then the same for
  any integer-exponent reference a kernel keeps, however lazily it raises it
  (parity unpinned beyond that: the GPU's exponential).  ``math`` mode keeps P
  exact.
* ``emulate`` mode rounds the output to bf16; a query block with no retained
  key block outputs zeros.
"""

from __future__ import annotations

import numpy as np

from . import formats as F
from .rank import BIT4, BIT8, BIT16

LOG2E = 1.4426950408889634


def bf16_round(x):
    """fp64 → fp32 (RN) → bf16 (RN, ties to even), returned as fp64."""
    f = np.asarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


class _State:
    def __init__(self, rows, d):
        self.m = np.full(rows, -np.inf)
        self.l = np.zeros(rows)
        self.o = np.zeros((rows, d))

    def merge(self, m_blk, l_blk, x_blk):
        """Merge a block whose P was taken relative to m_blk (per row)."""
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


def qblock_attention(prep, qb, prec_row, d, mode="emulate"):
    """Output rows [S, d] of query block ``qb`` of one head.

    ``prep``: dict from ``prep.prepare_head``; ``prec_row``: uint8 [nb] precision
    of each key block for this query block (16, 8, 4, 0)."""
    S = prep["q_blocks"].shape[1]
    valid = prep["valid"]
    inv_sqrt_d = 1.0 / np.sqrt(d)
    st = _State(S, d)

    # phase 16: bf16 operands, online softmax across blocks
    q = prep["q_blocks"][qb]
    for kb in np.nonzero(prec_row == BIT16)[0]:
        s = (q @ prep["k_blocks"][kb].T) * inv_sqrt_d
        s = np.where(valid[kb][None, :], s, -np.inf)
        m_new = np.maximum(st.m, _row_max(s))
        if mode == "emulate":
            # P is rounded in bf16 relative to 2^ceil(m_run log2 e), then brought
            # to the accumulator's units (exp(-m_run)) exactly
            p_den = _exp_rel(s, m_new)
            r = np.ceil(m_new * LOG2E)
            shift = np.exp2(r - m_new * LOG2E)  # >= 1; exact fp64 scaling
            p_num = bf16_round(p_den / shift[:, None]) * shift[:, None]
            alpha = np.where(np.isfinite(st.m), np.exp(st.m - np.where(np.isfinite(m_new), m_new, 0)), 0.0)
            st.l = st.l * alpha + p_den.sum(1)
            st.o = st.o * alpha[:, None] + p_num @ prep["v_blocks"][kb]
            st.m = m_new
        else:
            m_blk = _row_max(s)
            p = _exp_rel(s, m_blk)
            st.merge(m_blk, p.sum(1), p @ prep["v_blocks"][kb])

    # phase 8: INT8 Q/K codes with block scales, u8 P, INT8 V with channel scales
    qi = prep["q_i8"][qb].astype(np.float64)
    sq = prep["q_s8"][qb]
    for kb in np.nonzero(prec_row == BIT8)[0]:
        s_int = qi @ prep["k_i8"][kb].astype(np.float64).T  # exact integers
        s = s_int * (sq * prep["k_s8"][kb] * inv_sqrt_d)
        s = np.where(valid[kb][None, :], s, -np.inf)
        m_blk = _row_max(s)
        p = _exp_rel(s, m_blk)
        code = np.rint(255.0 * p)
        x = (code @ prep["v_i8"][kb].astype(np.float64).T) * (prep["v_s8"][None, :] / 255.0)
        st.merge(m_blk, p.sum(1), x)

    # phase 4: NVFP4 Q/K, NVFP4 P (16-key microblocks), NVFP4 V
    qd = F.nvfp4_dequantize(prep["q_f4"][qb], prep["q_sf4"][qb])
    for kb in np.nonzero(prec_row == BIT4)[0]:
        kd = F.nvfp4_dequantize(prep["k_f4"][kb], prep["k_sf4"][kb])
        s = (qd @ kd.T) * inv_sqrt_d
        s = np.where(valid[kb][None, :], s, -np.inf)
        m_blk = _row_max(s)
        p = _exp_rel(s, m_blk)
        pc, psf = F.nvfp4_quantize(p, axis=-1, block=16)
        pd = F.nvfp4_dequantize(pc, psf)
        vt = F.nvfp4_dequantize(prep["v_f4"][kb], prep["v_sf4"][kb]) * prep["v_g4"][:, None]
        st.merge(m_blk, p.sum(1), pd @ vt.T)

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
