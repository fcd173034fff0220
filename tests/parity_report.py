"""Parity figures of the GPU path on the five workloads (needs a GPU).

    python tests/parity_report.py [workload ...]

For each workload, the output of the whole call (through the C ABI) on sampled
query blocks of sampled heads (both ends of the block order, the heaviest and
the empty query blocks, and a seeded spread; every block of the tiny workload)
against the oracle in emulate mode, and against exact fp64 dense attention on
the same rows; one markdown table row per workload.  The GPU parity tests
assert the same comparison against the tolerance; this prints the numbers.
"""

from __future__ import annotations

import os
import sys
import time

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import parity as PT  # noqa: E402
from mixed_precision_block_b200.synth import WORKLOADS, make_qkv  # noqa: E402
from oracle import geometry as OG, prep as OP  # noqa: E402

SAMPLES = {"tiny": (None, None), "mid": ([0, 7], 24), "video": ([5, 19], 12),
           "video4bit": ([11, 2], 12), "long": ([17], 8)}


def report(name):
    wl = WORKLOADS[name]
    heads, nq = SAMPLES[name]
    q, k, v = make_qkv(wl, "cuda")
    p, ws, out = PT.run_gpu(wl, q, k, v)
    op = PT.oracle_problem(wl)
    table = OG.block_tokens(op)
    heads = range(wl.B * wl.H) if heads is None else heads
    num_o = num_d = den_o = den_d = 0.0
    worst = 0.0
    nrows = 0
    t0 = time.time()
    for bh in heads:
        qh, kh, vh = PT.head_inputs(q, k, v, bh, wl.B, wl.H)
        pr = OP.prepare_head(op, qh, kh, vh, table)
        pmap = np.asarray(PT.g(p, ws, "MAP", bh)).reshape(op.nb, op.nb)
        if nq is None:
            qbs = list(range(op.nb))
        else:
            rng = np.random.default_rng(bh)
            counts = (pmap != 0).sum(1)
            qbs = [0, op.nb - 1] + list(np.argsort(-counts)[:2]) + list(np.nonzero(counts == 0)[0][:2])
            qbs += list(rng.choice(op.nb, nq, replace=False))
            qbs = sorted(set(int(x) for x in qbs))
        toks, want = PT.oracle_rows(op, pr, pmap, qbs)
        b, h = divmod(bh, wl.H)
        got = out[b, h].float().cpu().numpy().astype(np.float64)[toks]
        dense = PT.dense_rows(qh, kh, vh, toks)
        num_o += float(((got - want) ** 2).sum())
        den_o += float((want ** 2).sum())
        num_d += float(((got - dense) ** 2).sum())
        den_d += float((dense ** 2).sum())
        worst = max(worst, PT.rel_l2(got, want))
        nrows += len(toks)
    del ws, out
    torch.cuda.empty_cache()
    return (f"| {name} | {'/'.join(f'{x:g}' for x in wl.budget)} | {len(list(heads))} | {nrows} | "
            f"{(num_o / den_o) ** 0.5:.2e} | {worst:.2e} | {(num_d / den_d) ** 0.5:.4f} | {time.time() - t0:.0f} |")


def main():
    names = sys.argv[1:] or list(SAMPLES)
    print("| workload | budget skip/4/8/16 | heads | rows | rel L2 vs oracle | worst head | rel L2 vs fp64 dense | s |")
    print("|---|---|---|---|---|---|---|---|")
    for n in names:
        print(report(n), flush=True)


if __name__ == "__main__":
    main()
