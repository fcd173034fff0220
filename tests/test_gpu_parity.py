"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Small workloads are compared in full; the three full-size video workloads on
sampled heads, blocks and query blocks.  See tests/parity.py for the
tolerances.
"""

import numpy as np
import pytest
import torch

from mixed_precision_block_b200.synth import WORKLOADS, Workload, make_qkv
from oracle import draft as ODR, geometry as OG, prep as OP, rank as OR
from oracle.pipeline import to_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from mixed_precision_block_b200 import da2
    import parity as PT


def _full_check(wl, heads=None, dense_ref=True):
    q, k, v = make_qkv(wl, "cuda")
    p, ws, out = PT.run_gpu(wl, q, k, v)
    op = PT.oracle_problem(wl)
    n16, n8, n4, _ = OG.budget_counts(op)
    PT.check_perm(p, ws, op)
    heads = range(wl.B * wl.H) if heads is None else heads
    table = OG.block_tokens(op)
    outs = []
    for bh in heads:
        qh, kh, vh = PT.head_inputs(q, k, v, bh, wl.B, wl.H)
        pr = OP.prepare_head(op, qh, kh, vh, table)
        PT.check_prep_head(p, ws, op, pr, bh, n8, n4)
        D = ODR.draft_map(pr["q_avg"], pr["k_avg"], pr["q_max"], pr["k_max"], op.lam, op.d)
        sg = PT.g(p, ws, "SCORES", bh)
        PT.check_scores_rows(sg, D)
        pmap = PT.check_assignment(p, ws, op, bh, sg)
        assert [(pmap == x).sum() for x in (16, 8, 4)] == [n16, n8, n4]
        toks, rows = PT.oracle_rows(op, pr, pmap, range(op.nb))
        b, h = divmod(bh, wl.H)
        got = out[b, h].float().cpu().numpy().astype(np.float64)[toks]
        err = PT.rel_l2(got, rows)
        assert err <= PT.OUT_TOL, (bh, err)
        outs.append(err)
        if dense_ref:
            dn = PT.dense_rows(qh, kh, vh, toks)
            outs.append(PT.rel_l2(got, dn))
    st = da2.view(p, ws, "STATUS")
    assert int(st[0]) == 0 and int(st[1]) == 0  # attention's and the V preparation's bounded waits
    assert da2.da2_check_status(p, ws) == 0
    return outs


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dense", [False, True])
def test_attention_cta_fits_an_sm(d, dense):
    # one CTA per SM, holding two query-block pairs whose softmax warpgroups
    # hide each other's latency: its registers, shared memory and launch
    # attributes must admit it
    assert da2.da2_attention_occupancy(d, dense) == 1


def test_tiny_workload_all_stages():
    _full_check(WORKLOADS["tiny"])


def test_ragged_padded_grid_d128():
    wl = Workload("ragged", 1, 2, 3, 12, 20, 128, 0.5, (40.0, 20.0, 20.0, 20.0), seed=3)
    _full_check(wl)


def test_ragged_padded_grid_d64_batch2():
    wl = Workload("ragged64", 2, 2, 2, 13, 11, 64, 0.25, (30.0, 30.0, 30.0, 10.0), seed=4)
    _full_check(wl)


def test_odd_block_count_padded_d128_tensor_core_path():
    # 27 region blocks (odd: the last query-block pair has one member), padded
    # in y and x, budget without a 4-bit share
    wl = Workload("odd", 1, 2, 3, 20, 20, 128, 0.5, (50.0, 0.0, 30.0, 20.0), seed=9)
    _full_check(wl)


def test_mid_workload_two_heads():
    _full_check(WORKLOADS["mid"], heads=[0, 7])


@pytest.mark.parametrize("budget", [(0.0, 0.0, 100.0, 0.0), (0.0, 100.0, 0.0, 0.0)])
def test_mid_shape_single_low_bit_budgets(budget):
    # every pair in one low-bit phase: the per-block references and the
    # quantised row sums carry the whole output
    _full_check(WORKLOADS["mid"].with_(budget=budget), heads=[0, 11], dense_ref=False)


@pytest.mark.parametrize("budget", [(0.0, 0.0, 0.0, 100.0), (0.0, 0.0, 100.0, 0.0), (0.0, 100.0, 0.0, 0.0),
                                    (100.0, 0.0, 0.0, 0.0), (99.9, 0.0, 0.0, 0.1)])
def test_single_precision_and_degenerate_budgets(budget):
    wl = Workload("edge", 1, 2, 2, 16, 24, 128, 0.5, budget, seed=5)
    _full_check(wl)


def test_all_skipped_outputs_zero():
    wl = Workload("skip", 1, 2, 2, 16, 16, 64, 0.5, (100.0, 0.0, 0.0, 0.0), seed=6)
    q, k, v = make_qkv(wl, "cuda")
    _, _, out = PT.run_gpu(wl, q, k, v)
    assert not out.any()


@pytest.mark.parametrize("lam", [0.0, 1.0])
def test_lambda_extremes(lam):
    _full_check(WORKLOADS["tiny"].with_(lam=lam, seed=7))


def test_full_dense_budget_matches_own_dense_kernel():
    wl = Workload("dense", 1, 2, 2, 16, 24, 128, 0.5, (0.0, 0.0, 0.0, 100.0), seed=8)
    q, k, v = make_qkv(wl, "cuda")
    _, _, out = PT.run_gpu(wl, q, k, v)
    dn = torch.empty_like(q)
    da2.da2_dense_attention(q, k, v, dn)
    torch.cuda.synchronize()
    a = out.float().cpu().numpy().astype(np.float64)
    b = dn.float().cpu().numpy().astype(np.float64)
    assert PT.rel_l2(a, b) < 1e-3


@pytest.mark.parametrize("N,d", [(1000, 128), (64, 64), (4097, 128), (130, 64), (64, 128), (191, 128)])
def test_dense_kernel_against_fp64(N, d):
    g = torch.Generator(device="cuda").manual_seed(N + d)
    q, k, v = (torch.randn((1, 2, N, d), generator=g, device="cuda") * s for s in (1.0, 1.0, 1.0))
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    out = torch.empty_like(q)
    da2.da2_dense_attention(q, k, v, out)
    torch.cuda.synchronize()
    for h in range(2):
        qh, kh, vh = (to_f64(x[0, h]) for x in (q, k, v))
        want = PT.dense_rows(qh, kh, vh, np.arange(N))
        got = out[0, h].float().cpu().numpy().astype(np.float64)
        assert PT.rel_l2(got, want) < 4e-3


def test_rank_from_scores_ties_and_zeros():
    wl = Workload("ties", 1, 3, 2, 16, 16, 64, 0.5, (40.0, 20.0, 20.0, 20.0))
    p = da2.Problem.from_workload(wl)
    op = PT.oracle_problem(wl)
    nb = op.nb
    rng = np.random.default_rng(0)
    s = np.empty((3, nb, nb), np.float32)
    s[0] = rng.choice(np.array([0.0, 1e-3, 0.5], np.float32), size=(nb, nb))  # heavy ties
    s[1] = 0.25  # every score equal
    s[2] = rng.random((nb, nb)).astype(np.float32)
    s[2][rng.random((nb, nb)) < 0.5] = 0.0
    ws = da2.workspace(p)
    da2.da2_rank_from_scores(p, torch.from_numpy(s).cuda(), ws)
    torch.cuda.synchronize()
    for bh in range(3):
        PT.check_assignment(p, ws, op, bh, s[bh])


# ------------------------------------------------------------------ full size

BLOCK_TOL = 6e-3  # per query block: a wrong block is O(1), bf16 rounding alone ~1e-3


def _sampled_check(wl, heads=(1, 8, 15, 22), n_qblocks=64, seed=0):
    """Full-size workload: every stage on the GPU; the oracle on sampled heads
    spread over the 24, and on each of them n_qblocks query blocks — a seeded
    spread plus the two with the most retained key blocks and up to two with
    none.  The output must be within OUT_TOL per head and BLOCK_TOL per query
    block (so that one wrong block cannot hide in a head's norm)."""
    q, k, v = make_qkv(wl, "cuda")
    p, ws, out = PT.run_gpu(wl, q, k, v)
    assert da2.da2_check_status(p, ws) == 0
    op = PT.oracle_problem(wl)
    n16, n8, n4, _ = OG.budget_counts(op)
    PT.check_perm(p, ws, op)
    table = OG.block_tokens(op)
    rng = np.random.default_rng(seed)
    summary = []
    for bh in heads:
        qh, kh, vh = PT.head_inputs(q, k, v, bh, wl.B, wl.H)
        pr = OP.prepare_head(op, qh, kh, vh, table)
        PT.check_prep_head(p, ws, op, pr, bh, n8, n4, blocks=rng.choice(op.nb, 64, replace=False))
        sg = PT.g(p, ws, "SCORES", bh)
        rows = rng.choice(op.nb, 32, replace=False)
        D = ODR.draft_map(pr["q_avg"][rows], pr["k_avg"], pr["q_max"][rows], pr["k_max"], op.lam, op.d)
        PT.check_scores_rows(sg[rows], D)
        pmap = PT.check_assignment(p, ws, op, bh, sg)
        counts = (pmap != 0).sum(1)
        heavy = list(np.argsort(-counts, kind="stable")[:2])
        empty = list(np.nonzero(counts == 0)[0][:2])
        pool = np.setdiff1d(np.arange(op.nb), heavy + empty)
        qbs = heavy + empty + list(rng.choice(pool, n_qblocks - len(heavy) - len(empty), replace=False))
        b, h = divmod(bh, wl.H)
        got_head = out[b, h].float().cpu().numpy().astype(np.float64)
        num = den = 0.0
        worst = 0.0
        for qb in qbs:
            toks, want = PT.oracle_rows(op, pr, pmap, [qb])
            got = got_head[toks]
            num += float(((got - want) ** 2).sum())
            den += float((want ** 2).sum())
            if counts[qb] == 0:
                assert not got.any(), (bh, qb)  # an empty query block outputs zeros
                continue
            e = PT.rel_l2(got, want)
            worst = max(worst, e)
        err = (num / max(den, 1e-300)) ** 0.5
        summary.append((bh, err, worst))
        assert err <= PT.OUT_TOL, (bh, err)
        assert worst <= BLOCK_TOL, (bh, worst)
        del pr
    print("head, rel L2, worst query block:", summary)
    del ws, out
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_video_full_size_sampled():
    _sampled_check(WORKLOADS["video"])


@pytest.mark.slow
@pytest.mark.parametrize("lam", [0.0, 0.5, 1.0])
def test_video4bit_full_size_lambda_sweep(lam):
    heads = (1, 8, 15, 22) if lam == 0.5 else (3, 20)
    _sampled_check(WORKLOADS["video4bit"].with_(lam=lam), heads=heads)


@pytest.mark.slow
def test_long_full_size_sampled():
    _sampled_check(WORKLOADS["long"])
