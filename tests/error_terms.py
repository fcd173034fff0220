"""Error decomposition of the method on the synthetic workloads (oracle only).

For sampled query blocks of sampled heads it reports, against exact dense
attention, the relative L2 error of exact attention restricted to the
retained key blocks (``sparse``), of the mixed-precision result against that
exact sparse result (``quant``), and of the mixed-precision result itself
(``total``); see ``oracle.attention.error_terms``.  Runs on the CPU:

    python tests/error_terms.py [workload ...] [--qblocks N] [--heads N] [--lams 0,0.5,1]

and prints one markdown table row per (workload, lambda).
"""

from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from mixed_precision_block_b200.synth import WORKLOADS, make_qkv  # noqa: E402
from oracle import attention, pipeline  # noqa: E402
from oracle.problem import Problem  # noqa: E402


def sample_qblocks(nb, n, seed=0):
    """n query blocks spread over the head: both ends and a seeded spread."""
    if n >= nb:
        return list(range(nb))
    rng = np.random.default_rng(seed)
    pick = {0, nb - 1} | set(rng.choice(nb, size=n, replace=False).tolist())
    return sorted(pick)[:n]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("workloads", nargs="*", default=["tiny", "mid", "video", "video4bit"])
    ap.add_argument("--qblocks", type=int, default=8)
    ap.add_argument("--heads", type=int, default=1)
    ap.add_argument("--lams", default=None, help="comma-separated lambda values (default: the workload's)")
    args = ap.parse_args()
    print("| workload | budget skip/4/8/16 | lambda | heads x q-blocks | sparse | quant | total | s |")
    print("|---|---|---|---|---|---|---|---|")
    for name in args.workloads:
        base = WORKLOADS[name]
        lams = [base.lam] if args.lams is None else [float(x) for x in args.lams.split(",")]
        q, k, v = make_qkv(base)
        for lam in lams:
            wl = base.with_(lam=lam)
            p = Problem.from_workload(wl)
            t0 = time.time()
            acc = {"sparse": 0.0, "quant": 0.0, "total": 0.0}
            heads = min(args.heads, wl.B * wl.H)
            for bh in range(heads):
                b, h = divmod(bh, wl.H)
                qh, kh, vh = (pipeline.to_f64(x[b, h]) for x in (q, k, v))
                qbs = sample_qblocks(p.nb, args.qblocks, seed=bh)
                r = pipeline.run_head(p, qh, kh, vh, mode="math", qblocks=[])
                t = attention.error_terms(r["prep"], r["map"], p.d, qbs)
                for key in acc:
                    acc[key] += t[key] ** 2
            res = {key: (val / heads) ** 0.5 for key, val in acc.items()}
            print(f"| {name} | {'/'.join(f'{x:g}' for x in wl.budget)} | {lam:g} | {heads} x "
                  f"{min(args.qblocks, p.nb)} | {res['sparse']:.4f} | {res['quant']:.4f} | {res['total']:.4f} | "
                  f"{time.time() - t0:.0f} |", flush=True)


if __name__ == "__main__":
    main()
