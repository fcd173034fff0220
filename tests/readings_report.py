"""Accuracy of candidate readings of the low-bit P quantisation (CPU report).

The pages leave open what low-bit P is quantised against (DraftAttention2
reading note, Method overview bullets 3-4: low-bit phases recover the
mid-importance interactions; the phases share the softmax statistics).  This
report measures, for several readings, the error that P's quantisation alone
adds: the same quantised Q/K/V, the same assignment, against the same
attention with exact (unquantised) P, as relative L2 over sampled query
blocks of one head of the mid-size shape.

Readings (per query row):
  blk_exact    reference = the key block's own row maximum (INT8 and NVFP4)
  blk_pow2     reference = that maximum rounded up to a power of two
  phase_pow2   one reference per phase: ceil of the phase's row maximum
  final_pow2   one reference for all phases: ceil of the row's maximum
  running      the previous oracle's reading: a power-of-two reference raised
               per pair of key blocks, started from the running maximum of the
               phases before (replayed here in the query block's own order)
Each with the denominator summing unquantised p, and with ``+ql``: the
denominator summing the quantised weights the numerator uses.

    python tests/readings_report.py [--qblocks 48]

The adopted reading (oracle/attention.py) is blk_pow2 + ql for both low-bit
formats.
"""

from __future__ import annotations

import argparse
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from mixed_precision_block_b200.synth import WORKLOADS, make_qkv  # noqa: E402
from oracle import attention as OA, draft as ODR, formats as F, geometry as OG  # noqa: E402
from oracle import prep as OP, rank as OR  # noqa: E402
from oracle.pipeline import to_f64  # noqa: E402
from oracle.problem import Problem  # noqa: E402

LOG2E = OA.LOG2E


def _q8(p):
    return np.rint(255.0 * p) / 255.0


def _q4(p):
    t = F.f32(OA.P4_RANGE * F.f32(p))
    c, s = F.nvfp4_quantize(t, axis=-1, block=16)
    return F.nvfp4_dequantize(c, s) / OA.P4_RANGE


def _phase_items(pr, qb, row, d):
    """Per phase: list of (x [S, 64] log2-unit scores, -inf unused; V [64, d])."""
    valid = pr["valid"]
    isd = 1.0 / np.sqrt(d)
    out = {16: [], 8: [], 4: []}
    q = pr["q_blocks"][qb]
    for kb in np.nonzero(row == 16)[0]:
        s = (q @ pr["k_blocks"][kb].T) * isd
        out[16].append((np.where(valid[kb][None], s * LOG2E, -np.inf), pr["v_blocks"][kb]))
    qi, sq = pr["q_i8"][qb].astype(np.float64), pr["q_s8"][qb]
    for kb in np.nonzero(row == 8)[0]:
        s = (qi @ pr["k_i8"][kb].astype(np.float64).T) * (sq * pr["k_s8"][kb] * isd)
        vd = pr["v_i8"][kb].astype(np.float64).T * pr["v_s8"][None, :]
        out[8].append((np.where(valid[kb][None], s * LOG2E, -np.inf), vd))
    qd = F.nvfp4_dequantize(pr["q_f4"][qb], pr["q_sf4"][qb])
    for kb in np.nonzero(row == 4)[0]:
        kd = F.nvfp4_dequantize(pr["k_f4"][kb], pr["k_sf4"][kb])
        vt = F.nvfp4_dequantize(pr["v_f4"][kb], pr["v_sf4"][kb]) * pr["v_g4"][:, None]
        out[4].append((np.where(valid[kb][None], (qd @ kd.T) * isd * LOG2E, -np.inf), vt.T))
    return out


def _rowmax(xs):
    return np.max(np.stack([x.max(1) for x in xs]), 0) if xs else None


def reading_output(items, reading, ql, exact=False):
    """fp64 output of one query block under a reading (math mode)."""
    allx = [x for ph in (16, 8, 4) for x, _ in items[ph]]
    S, d = allx[0].shape[0], items[16][0][1].shape[1] if items[16] else (
        items[8][0][1].shape[1] if items[8] else items[4][0][1].shape[1])
    M = _rowmax(allx)
    Mf = np.where(np.isfinite(M), M, 0.0)
    num, l = np.zeros((S, d)), np.zeros(S)
    for x, v in items[16]:
        p = np.exp2(x - Mf[:, None])
        num += p @ v
        l += p.sum(1)
    run = np.full(S, -np.inf)
    for x, _ in items[16]:
        run = np.maximum(run, x.max(1))
    for ph, qf in ((8, _q8), (4, _q4)):
        its = items[ph]
        if not its:
            continue
        if reading == "running":
            # reference raised per consecutive pair of blocks, from the running max
            r = np.where(np.isfinite(run), np.ceil(np.where(np.isfinite(run), run, 0)), -np.inf)
            for i in range(0, len(its), 2):
                unit = its[i:i + 2]
                um = _rowmax([x for x, _ in unit])
                up = np.isfinite(um) & (~np.isfinite(r) | (um > r))
                r = np.where(up, np.ceil(np.where(up, um, 0)), r)
                run = np.maximum(run, um)
                for x, v in unit:
                    rf = np.where(np.isfinite(r), r, 0.0)
                    p = np.where(np.isfinite(x), np.exp2(x - rf[:, None]), 0.0)
                    pq = p if exact else qf(p)
                    w = np.exp2(rf - Mf)[:, None]
                    num += (pq * w) @ v
                    l += ((pq if ql else p) * w).sum(1)
            continue
        phm = _rowmax([x for x, _ in its])
        for x, v in its:
            xb = x.max(1)
            ref = {"blk_exact": xb, "blk_pow2": np.ceil(xb), "phase_pow2": np.ceil(phm),
                   "final_pow2": np.ceil(M)}[reading]
            rf = np.where(np.isfinite(ref), ref, 0.0)
            p = np.where(np.isfinite(x), np.exp2(x - rf[:, None]), 0.0)
            pq = p if exact else qf(p)
            w = np.exp2(rf - Mf)[:, None]
            num += (pq * w) @ v
            l += ((pq if ql else p) * w).sum(1)
    return np.where(l[:, None] > 0, num / np.where(l > 0, l, 1)[:, None], 0.0)


def measure(budget, nq=48, seed=0):
    wl = WORKLOADS["mid"].with_(budget=budget, H=1)
    q, k, v = make_qkv(wl, "cpu")
    op = Problem.from_workload(wl)
    pr = OP.prepare_head(op, to_f64(q[0, 0]), to_f64(k[0, 0]), to_f64(v[0, 0]), OG.block_tokens(op))
    D = ODR.draft_scores(pr["q_avg"], pr["k_avg"], pr["q_max"], pr["k_max"], op.lam, op.d)
    n16, n8, n4, _ = OG.budget_counts(op)
    pmap = OR.assign(D, n16, n8, n4)
    qbs = np.random.default_rng(seed).choice(op.nb, nq, replace=False)
    items = {qb: _phase_items(pr, qb, pmap[qb], op.d) for qb in qbs}
    ref = {qb: reading_output(items[qb], "blk_exact", False, exact=True) for qb in qbs}
    den = sum(float((ref[qb][pr["valid"][qb]] ** 2).sum()) for qb in qbs)
    res = {}
    for rd in ("blk_exact", "blk_pow2", "phase_pow2", "final_pow2", "running"):
        for ql in (False, True):
            n = sum(float(((reading_output(items[qb], rd, ql) - ref[qb])[pr["valid"][qb]] ** 2).sum())
                    for qb in qbs)
            res[rd + ("+ql" if ql else "")] = (n / den) ** 0.5
    # the adopted reading, computed by the oracle itself
    n = 0.0
    for qb in qbs:
        o = OA.qblock_attention(pr, qb, pmap[qb], op.d, "math")
        n += float(((o - ref[qb])[pr["valid"][qb]] ** 2).sum())
    res["oracle (adopted)"] = (n / den) ** 0.5
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--qblocks", type=int, default=48)
    a = ap.parse_args()
    budgets = [(85.0, 0.0, 7.5, 7.5), (50.0, 0.0, 50.0, 0.0), (50.0, 50.0, 0.0, 0.0),
               (50.0, 25.0, 15.0, 10.0), (80.7, 14.4, 4.8, 0.0), (70.0, 20.0, 8.0, 2.0)]
    rows = [(b, measure(b, a.qblocks)) for b in budgets]
    names = list(rows[0][1].keys())
    print("| reading | " + " | ".join("/".join(f"{x:g}" for x in b) for b, _ in rows) + " |")
    print("|---|" + "---|" * len(rows))
    for n in names:
        print(f"| {n} | " + " | ".join(f"{r[n]:.2e}" for _, r in rows) + " |")


if __name__ == "__main__":
    main()
