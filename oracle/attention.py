"""Mixed-precision block-sparse attention (oracle).

DraftAttention2 abstract and reading note (Method overview, bullet 4): one
attention pass per query block runs a phase per precision; the phases share
the softmax statistics (running max and sum) and one output accumulator, and
quantisation scales are folded in at the phase boundaries, so no partial
outputs are written back and merged.  Skipped pairs contribute nothing.

This module follows that structure literally, per query block, in fp64:
phase 16, then phase 8, then phase 4, one online-softmax state (m, l, O)
carried across all of them; each low-bit phase accumulates in its own
accumulator against a power-of-two reference that starts from the running
maximum of the phases before it, and is folded into that state, with its
channel scales, at the phase boundary.

Readings adopted (the pages leave these open):

* scores: 16-bit phase from the bf16 values; 8-bit phase from the exact integer
  product of the INT8 codes times both block scales; 4-bit phase from the
  dequantised NVFP4 values; all times 1/sqrt(d).  Padding keys score -inf.
* key blocks are taken two at a time ("units"), in the order a kernel that
  pairs neighbouring query blocks (2p, 2p+1) walks them: per low-bit phase,
  the key blocks either query block retains, ascending; when neither query
  block of the pair retains a 16-bit block (nothing has set the reference),
  first those both retain, then the rest, each group ascending.  The list is
  cut into consecutive pairs.  A unit's blocks that this query block does not
  retain contribute nothing to its rows.  (The 16-bit phase's result does not
  depend on the order.)
* P in the 8-bit and 4-bit phases is quantised relative to a running power of
  two 2^r per row (r an integer, log2 units).  The phases share the softmax
  statistics, so a low-bit phase starts from r = ceil(x_run), x_run the row's
  running maximum of s·log2 e over every unit of the phases before it (-inf
  if there was none).  Before a unit, if the unit's row maximum x_max (over
  its retained keys) exceeds r, r becomes ceil(x_max), and what the phase
  accumulated so far is scaled by 2^(r_old - r).  So p = 2^(x - r) is in
  (0, 1]:
  8-bit code = round(255 p) as an unsigned byte (scale 1/255);
  4-bit = NVFP4, over 16 consecutive keys of the row, of 2688 p (2688 = 6·448
  puts the largest p at the top of the e2m1 x e4m3 range), dequantised and
  divided by 2688 again.  Each phase accumulates its P·V in its own
  accumulator; the phases' results meet, with the channel scales, at the end.
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
LN2 = 0.6931471805599453
P4_RANGE = 2688.0  # 6 (largest e2m1) x 448 (largest e4m3)


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


def phase_units(even_row, odd_row, bit):
    """The units of one low-bit phase of the query-block pair (2p, 2p+1),
    whose precision rows are ``even_row`` and ``odd_row`` (None if 2p+1 does
    not exist): the key blocks either assigns to ``bit``, ascending; if
    neither row holds a 16-bit block, those both assign first, then the rest,
    each group ascending.  Cut into consecutive pairs (the last may hold one)."""
    a = even_row == bit
    b = odd_row == bit if odd_row is not None else np.zeros_like(a)
    no16 = not np.any(even_row == BIT16) and (odd_row is None or not np.any(odd_row == BIT16))
    if no16:
        kbs = np.concatenate([np.nonzero(a & b)[0], np.nonzero(a ^ b)[0]]).astype(np.int64)
    else:
        kbs = np.nonzero(a | b)[0].astype(np.int64)
    return [kbs[i:i + 2] for i in range(0, len(kbs), 2)]


class _LowBitPhase:
    """A low-bit phase's P·V accumulator and sum against a running power of two
    2^r per row (r an integer, log2 units; -inf before the first score)."""

    def __init__(self, rows, d, r0=None):
        self.r = np.full(rows, -np.inf) if r0 is None else np.array(r0, dtype=np.float64)
        self.l = np.zeros(rows)
        self.acc = np.zeros((rows, d))

    def enter(self, xs):
        """Take a unit whose blocks have log2-unit scores ``xs`` ([rows, keys]
        each, -inf where not retained): raise r to ceil of the unit's row max
        where that max exceeds r, rescale what is accumulated, add the
        unquantised p to l and return each block's p = 2^(x - r)."""
        x_max = np.max(np.stack([x.max(1) for x in xs]), axis=0)
        self.x_max = x_max
        up = np.isfinite(x_max) & (x_max > self.r)
        r_new = np.where(up, np.ceil(np.where(up, x_max, 0.0)), self.r)
        had = np.isfinite(self.r)
        a = np.where(up, np.where(had, np.exp2(np.where(had, self.r, 0.0) - np.where(up, r_new, 0.0)), 0.0), 1.0)
        self.acc *= a[:, None]
        self.l *= a
        self.r = r_new
        live = np.isfinite(self.r)
        ps = []
        for x in xs:
            ok = np.isfinite(x) & live[:, None]
            p = np.where(ok, np.exp2(np.where(ok, x - np.where(live, self.r, 0.0)[:, None], 0.0)), 0.0)
            self.l += p.sum(1)
            ps.append(p)
        return ps

    def fold_into(self, st, chan_scale):
        """Phase boundary: join the shared state with the phase's channel scale."""
        m_blk = np.where(np.isfinite(self.r), self.r * LN2, -np.inf)
        st.merge(m_blk, self.l, self.acc * chan_scale)


def _row_max(s):
    return s.max(axis=1)


def _exp_rel(s, m):
    """exp(s - m) per row, 0 where s is -inf or the row has no finite score."""
    ok = np.isfinite(m)[:, None] & np.isfinite(s)
    return np.where(ok, np.exp(np.where(ok, s - np.where(np.isfinite(m), m, 0)[:, None], 0)), 0.0)


def qblock_attention(prep, qb, prec_row, d, mode="emulate", partner_row=None, trace=None):
    """Output rows [S, d] of query block ``qb`` of one head.

    ``prep``: dict from ``prep.prepare_head``; ``prec_row``: uint8 [nb] precision
    of each key block for this query block (16, 8, 4, 0); ``partner_row``: the
    same for the other query block of its pair (qb ^ 1), None if there is none.
    The partner only decides how the low-bit phases group key blocks into units
    (``qb`` even: this block is the pair's even one; a missing partner leaves
    this block's own list).
    ``trace``: a dict that receives each low-bit phase's starting reference
    (``r0_8``, ``r0_4``, per row)."""
    S = prep["q_blocks"].shape[1]
    valid = prep["valid"]
    inv_sqrt_d = 1.0 / np.sqrt(d)
    st = _State(S, d)
    x_run = np.full(S, -np.inf)  # running row max of s·log2 e, every phase so far

    # phase 16: bf16 operands, online softmax across blocks
    q = prep["q_blocks"][qb]
    for kb in np.nonzero(prec_row == BIT16)[0]:
        s = (q @ prep["k_blocks"][kb].T) * inv_sqrt_d
        s = np.where(valid[kb][None, :], s, -np.inf)
        x_run = np.maximum(x_run, _row_max(s) * LOG2E)
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
    ph = _LowBitPhase(S, d, np.ceil(x_run))
    if trace is not None:
        trace["r0_8"] = ph.r.copy()
    even, odd = (prec_row, partner_row) if (qb % 2 == 0 or partner_row is None) else (partner_row, prec_row)
    for unit in phase_units(even, odd, BIT8):
        xs = []
        for kb in unit:
            s_int = qi @ prep["k_i8"][kb].astype(np.float64).T  # exact integers
            s = s_int * (sq * prep["k_s8"][kb] * inv_sqrt_d)
            keep = valid[kb][None, :] & (prec_row[kb] == BIT8)
            xs.append(np.where(keep, s * LOG2E, -np.inf))
        for kb, p in zip(unit, ph.enter(xs)):
            code = np.rint(255.0 * p)
            ph.acc += code @ prep["v_i8"][kb].astype(np.float64).T  # exact integers
        x_run = np.maximum(x_run, ph.x_max)
    ph.fold_into(st, prep["v_s8"][None, :] / 255.0)

    # phase 4: NVFP4 Q/K, NVFP4 P (16-key microblocks of 2688 p), NVFP4 V
    qd = F.nvfp4_dequantize(prep["q_f4"][qb], prep["q_sf4"][qb])
    ph = _LowBitPhase(S, d, np.ceil(x_run))
    if trace is not None:
        trace["r0_4"] = ph.r.copy()
    for unit in phase_units(even, odd, BIT4):
        xs = []
        for kb in unit:
            kd = F.nvfp4_dequantize(prep["k_f4"][kb], prep["k_sf4"][kb])
            s = (qd @ kd.T) * inv_sqrt_d
            keep = valid[kb][None, :] & (prec_row[kb] == BIT4)
            xs.append(np.where(keep, s * LOG2E, -np.inf))
        for kb, p in zip(unit, ph.enter(xs)):
            t = F.f32(P4_RANGE * F.f32(p))
            pc, psf = F.nvfp4_quantize(t, axis=-1, block=16)
            vt = F.nvfp4_dequantize(prep["v_f4"][kb], prep["v_sf4"][kb])
            ph.acc += F.nvfp4_dequantize(pc, psf) @ vt.T
    ph.fold_into(st, prep["v_g4"][None, :] / P4_RANGE)

    out = np.where(st.l[:, None] > 0, st.o / np.where(st.l > 0, st.l, 1.0)[:, None], 0.0)
    return bf16_round(out) if mode == "emulate" else out


def partner_of(prec_map, qb):
    """Precision row of the other query block of qb's pair (2p, 2p+1), or None."""
    o = qb ^ 1
    return prec_map[o] if o < len(prec_map) else None


def head_attention(prep, prec_map, d, mode="emulate", qblocks=None):
    """Block-order output [nb, S, d] (rows of ``qblocks`` only, others zero)."""
    nb, S = prep["valid"].shape
    out = np.zeros((nb, S, d))
    for qb in (range(nb) if qblocks is None else qblocks):
        out[qb] = qblock_attention(prep, qb, prec_map[qb], d, mode, partner_of(prec_map, qb))
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


def error_terms(prep, prec_map, d, qblocks, partner=True):
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
        other = partner_of(prec_map, qb) if partner else None
        mixed = qblock_attention(prep, qb, row, d, "math", other)
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
