"""Pins for the oracle's mixed-precision attention (CPU).

* a 0/0/0/100 budget must give dense softmax attention (torch's fp64
  scaled_dot_product_attention is the reference), padding included;
* a partial 16-bit budget must give dense attention restricted to the kept
  key blocks (a boolean mask on the same library routine);
* a 100 % skip budget gives zeros;
* Q = 0 makes every score equal, which fixes the low-bit phases in closed form;
* a single-precision low-bit budget stays within the error bound that P's
  quantisation alone allows, against exact attention on the dequantised
  operands;
* emulate mode differs from math mode only by bf16 rounding.
"""

import numpy as np
import pytest
import torch

from oracle import attention, formats as F, geometry, pipeline, prep
from oracle.problem import Problem
from mixed_precision_block_b200.synth import Workload, make_qkv


def _inputs(T=2, Hh=12, Ww=10, d=32, H=1, seed=0, budget=(0, 0, 0, 100), lam=0.5):
    wl = Workload("t", 1, H, T, Hh, Ww, d, lam, budget, seed=seed)
    q, k, v = make_qkv(wl)
    p = Problem.from_workload(wl)
    return p, pipeline.to_f64(q)[0, 0], pipeline.to_f64(k)[0, 0], pipeline.to_f64(v)[0, 0]


def _sdpa(q, k, v, mask=None):
    t = [torch.from_numpy(x)[None, None] for x in (q, k, v)]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(*t, attn_mask=m)[0, 0].numpy()


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_full_16bit_budget_is_dense_attention():
    p, q, k, v = _inputs()
    r = pipeline.run_head(p, q, k, v, mode="math")
    assert _rel(r["out"], _sdpa(q, k, v)) < 1e-13
    r = pipeline.run_head(p, q, k, v, mode="emulate")
    assert 1e-4 < _rel(r["out"], _sdpa(q, k, v)) < 4e-3  # bf16 P and output


def test_partial_16bit_budget_is_masked_dense_attention():
    p, q, k, v = _inputs(budget=(60, 0, 0, 40))
    r = pipeline.run_head(p, q, k, v, mode="math")
    tab = r["prep"]["table"]
    keep = r["map"] == 16
    # token-level mask from the block-level assignment
    tok_blk = np.zeros(p.N, dtype=np.int64)
    for b in range(p.nb):
        tok_blk[tab[b][tab[b] >= 0]] = b
    mask = keep[tok_blk][:, tok_blk]
    want = _sdpa(q, k, v, mask)
    rows = mask.any(1)
    assert rows.all()  # this budget leaves no query region empty here
    assert _rel(r["out"], want) < 1e-13


def test_all_skipped_gives_zeros():
    p, q, k, v = _inputs(budget=(100, 0, 0, 0))
    r = pipeline.run_head(p, q, k, v, mode="emulate")
    assert not r["out"].any()


def test_q_zero_closed_forms():
    p, q, k, v = _inputs(Hh=12, Ww=10)
    q = np.zeros_like(q)
    # 8-bit only: every score 0 → p = 1 → code 255 → mean of the INT8-dequantised V
    p8 = Problem(**{**p.__dict__, "budget": (0, 0, 100, 0)})
    r = pipeline.run_head(p8, q, k, v, mode="math")
    vb = r["prep"]["v_i8"].astype(np.float64) * r["prep"]["v_s8"][None, :, None]  # [nb, d, S]
    vt = np.concatenate([vb[b][:, r["prep"]["valid"][b]] for b in range(p.nb)], axis=1)
    np.testing.assert_allclose(r["out"], np.broadcast_to(vt.mean(1), r["out"].shape), rtol=1e-12)
    # 4-bit only: p = 1 is quantised as 2688 p → sf = e4m3(2688/6) = 448 (the
    # largest e4m3), code = e2m1(2688/448) = 6 (the largest e2m1): exact, weight 1
    assert F.e4m3_round(2688.0 / 6.0) == 448.0
    assert F.e2m1_round(2688.0 / 448.0) == 6.0
    p4 = Problem(**{**p.__dict__, "budget": (0, 100, 0, 0)})
    r = pipeline.run_head(p4, q, k, v, mode="math")
    pr = r["prep"]
    vd = prep.dequant_v_nvfp4(pr["v_f4"], pr["v_sf4"], pr["v_g4"])
    vt = np.concatenate([vd[b][:, pr["valid"][b]] for b in range(p.nb)], axis=1)
    np.testing.assert_allclose(r["out"], np.broadcast_to(vt.mean(1), r["out"].shape), rtol=1e-12)


def _dequant_dense(p, pr, fmt):
    """Token-order dequantised Q, K, V of one head for the given phase format."""
    tab = pr["table"]
    valid = tab >= 0
    if fmt == 8:
        qd = pr["q_i8"] * pr["q_s8"][:, None, None]
        kd = pr["k_i8"] * pr["k_s8"][:, None, None]
        vd = (pr["v_i8"] * pr["v_s8"][None, :, None]).transpose(0, 2, 1)
    else:
        qd = F.nvfp4_dequantize(pr["q_f4"], pr["q_sf4"])
        kd = F.nvfp4_dequantize(pr["k_f4"], pr["k_sf4"])
        vd = prep.dequant_v_nvfp4(pr["v_f4"], pr["v_sf4"], pr["v_g4"]).transpose(0, 2, 1)
    out = []
    for x in (qd, kd, vd):
        y = np.zeros((p.N, p.d))
        y[tab[valid]] = x[valid]
        out.append(y)
    return out


@pytest.mark.parametrize("fmt", [8, 4])
def test_low_bit_phase_within_p_quantisation_bound(fmt):
    budget = (0, 0, 100, 0) if fmt == 8 else (0, 100, 0, 0)
    p, q, k, v = _inputs(Hh=12, Ww=10, budget=budget)
    r = pipeline.run_head(p, q, k, v, mode="math")
    qd, kd, vd = _dequant_dense(p, r["prep"], fmt)
    exact = _sdpa(qd, kd, vd)
    # bound: each weight's error is at most e * exp(m_blk - m) / l, e the
    # largest rounding error of one quantised p in (0, 1] relative to its block max
    # (INT8: half a step of 1/255; NVFP4: the sf step plus saturation, < 0.18)
    e = 0.5 / 255 if fmt == 8 else 0.18
    s = qd @ kd.T / np.sqrt(p.d)
    tab = r["prep"]["table"]
    m = s.max(1)
    l = np.exp(s - m[:, None]).sum(1)
    bound = np.zeros((p.N, p.d))
    for b in range(p.nb):
        toks = tab[b][tab[b] >= 0]
        mb = s[:, toks].max(1)
        bound += (e * np.exp(mb - m) / l)[:, None] * np.abs(vd[toks]).sum(0)[None, :]
    err = np.abs(r["out"] - exact)
    assert err.max() > 0
    assert np.all(err <= bound * (1 + 1e-9) + 1e-12)
    # and the phase stays close to exact attention on its own operands
    assert _rel(r["out"], exact) < (0.01 if fmt == 8 else 0.06)


def test_emulate_is_math_plus_bf16_rounding():
    p, q, k, v = _inputs(budget=(10, 40, 50, 0))
    a = pipeline.run_head(p, q, k, v, mode="math")["out"]
    b = pipeline.run_head(p, q, k, v, mode="emulate")["out"]
    np.testing.assert_array_equal(b, attention.bf16_round(a))


def test_scatter_restores_token_order():
    p = Problem(1, 1, 2, 10, 13, 4, 0.5, (0, 0, 0, 100))
    tab = geometry.block_tokens(p)
    x = np.random.default_rng(0).standard_normal((p.N, 4))
    blocks, _ = prep.gather_blocks(x, tab)
    np.testing.assert_array_equal(attention.scatter(blocks, tab, p.N), x)


def test_phase_units_order_of_the_pair():
    # the even block keeps 8-bit blocks 0, 2, 3, 5, 6; the odd one 1, 3, 4.
    # No 16-bit block in the pair: 3 (kept by both) first, then 0 1 2 4 5 6,
    # cut in pairs, from either side
    row = np.array([8, 0, 8, 8, 0, 8, 8, 0], dtype=np.uint8)
    partner = np.array([0, 8, 0, 8, 8, 0, 0, 0], dtype=np.uint8)
    want = [[3, 0], [1, 2], [4, 5], [6]]
    assert [list(u) for u in attention.phase_units(row, partner, 8)] == want
    assert [list(u) for u in attention.phase_units(partner, row, 8)] == want
    # a 16-bit block anywhere in the pair (block 7 of the odd row): the union ascending
    p16 = partner.copy()
    p16[7] = 16
    assert [list(u) for u in attention.phase_units(row, p16, 8)] == [[0, 1], [2, 3], [4, 5], [6]]
    # a block alone: its own list ascending; other precisions are not in the phase
    assert [list(u) for u in attention.phase_units(row, None, 8)] == [[0, 2], [3, 5], [6]]
    assert attention.phase_units(row, partner, 4) == []


def test_unit_order_covers_every_retained_block():
    # Q = 0 makes every score 0, so the order cannot change the result, but
    # the unit order must still cover every retained block exactly once: the
    # closed form of the 8-bit phase (code 255 everywhere: the mean of the
    # INT8-dequantised V of the retained blocks)
    p, q, k, v = _inputs(Hh=12, Ww=10, budget=(40, 0, 60, 0))
    q = np.zeros_like(q)
    r = pipeline.run_head(p, q, k, v, mode="math")
    pr = r["prep"]
    vb = pr["v_i8"].astype(np.float64) * pr["v_s8"][None, :, None]  # [nb, d, S]
    for qb in range(p.nb):
        keep = np.nonzero(r["map"][qb] == 8)[0]
        if len(keep) == 0:
            continue
        vt = np.concatenate([vb[b][:, pr["valid"][b]] for b in keep], axis=1)
        rows = pr["valid"][qb]
        got = attention.qblock_attention(pr, qb, r["map"][qb], p.d, "math", attention.partner_of(r["map"], qb))
        np.testing.assert_allclose(got[rows], np.broadcast_to(vt.mean(1), (rows.sum(), p.d)), rtol=1e-12)


def test_low_bit_reference_raise_by_hand():
    # one row; unit 1 max 0.3 → r = ceil(0.3) = 1; unit 2 max 2.5 → r = 3 and
    # what unit 1 left is scaled by 2^(1-3)
    ph = attention._LowBitPhase(1, 2)
    (p1,) = ph.enter([np.array([[0.3, -np.inf]])])
    assert ph.r[0] == 1.0
    assert p1[0, 0] == 2.0 ** (0.3 - 1.0) and p1[0, 1] == 0.0
    c1 = np.rint(255.0 * p1)  # 157
    assert c1[0, 0] == 157.0
    ph.acc += c1[:, :1] * np.array([[10.0, -20.0]])
    (pa, pb) = ph.enter([np.array([[2.5]]), np.array([[-1.0]])])
    assert ph.r[0] == 3.0
    np.testing.assert_allclose(ph.acc, [[157.0 * 10.0 / 4.0, -157.0 * 20.0 / 4.0]], rtol=0, atol=0)
    assert pa[0, 0] == 2.0 ** -0.5 and pb[0, 0] == 2.0 ** -4.0
    np.testing.assert_allclose(ph.l, [2.0 ** (0.3 - 1.0) / 4.0 + 2.0 ** -0.5 + 2.0 ** -4.0], rtol=1e-15)
    # a unit below the reference leaves it alone; an all -inf unit changes nothing
    ph.enter([np.array([[1.0]])])
    ph.enter([np.array([[-np.inf]])])
    assert ph.r[0] == 3.0


def _terms(budget, qblocks=None):
    p, q, k, v = _inputs(budget=budget)
    r = pipeline.run_head(p, q, k, v, mode="math")
    qbs = range(p.nb) if qblocks is None else qblocks
    return attention.error_terms(r["prep"], r["map"], p.d, qbs)


def test_error_terms_special_cases():
    t = _terms((0, 0, 0, 100))  # everything kept at 16 bits: exact
    assert t["sparse"] < 1e-13 and t["quant"] < 1e-13 and t["total"] < 1e-13
    t = _terms((100, 0, 0, 0))  # everything skipped: the output is zero
    assert abs(t["sparse"] - 1.0) < 1e-13 and t["quant"] < 1e-13 and abs(t["total"] - 1.0) < 1e-13
    t = _terms((0, 0, 100, 0))  # nothing skipped, all INT8: only quantisation error
    assert t["sparse"] < 1e-13 and abs(t["quant"] - t["total"]) < 1e-13 and 0 < t["quant"] < 0.05


def test_error_terms_triangle_and_both_present():
    t = _terms((40, 20, 20, 20))
    assert t["total"] <= t["sparse"] + t["quant"] + 1e-12
    assert t["sparse"] > 0 and t["quant"] > 0


def _two_level_head(d=64):
    """One frame of 8x24 tokens = three full 8x8 regions (key blocks 0, 1, 2).
    Every query is 8 e_0; keys of block 0 are 8 e_0 (score 64/sqrt(64) = 8,
    x = 8 log2 e = 11.54 in log2 units), keys of blocks 1 and 2 are 0 (score
    0).  V rows are small integers, exact in every format's scale."""
    p = Problem(1, 1, 1, 8, 24, d, 0.5, (0, 0, 0, 100))
    tab = geometry.block_tokens(p)
    q = np.zeros((p.N, d))
    q[:, 0] = 8.0
    k = np.zeros((p.N, d))
    k[tab[0], 0] = 8.0
    v = np.random.default_rng(3).integers(-3, 4, size=(p.N, d)).astype(np.float64)
    return p, prep.prepare_head(p, q, k, v), v, tab


def test_low_bit_phase_starts_from_the_shared_running_max():
    # block 0 at 16 bits sets the running max x = 11.54; the 8-bit phase then
    # starts from r = ceil(11.54) = 12, so block 1's p = 2^(0 - 12) gives code
    # rint(255 / 4096) = 0: block 1 adds its unquantised mass 64 e^-8 to the
    # denominator and nothing to the numerator.  (A phase that restarted its
    # reference would take r = 0 and code 255 instead.)
    p, pr, v, tab = _two_level_head()
    row = np.array([16, 8, 0], dtype=np.uint8)
    tr = {}
    out = attention.qblock_attention(pr, 0, row, p.d, "math", None, trace=tr)
    np.testing.assert_array_equal(tr["r0_8"], np.full(64, 12.0))
    want = v[tab[0]].mean(0) / (1.0 + np.exp(-8.0))
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=1e-12, atol=1e-15)


def test_four_bit_phase_continues_the_reference_of_the_eight_bit_phase():
    # block 0 at 8 bits (INT8 codes 127 and scale 8/127 reproduce the score 8
    # exactly) and block 2 at 4 bits: the 4-bit phase starts from ceil(11.54) = 12
    p, pr, v, tab = _two_level_head()
    row = np.array([8, 0, 4], dtype=np.uint8)
    tr = {}
    attention.qblock_attention(pr, 0, row, p.d, "math", None, trace=tr)
    assert np.all(np.isneginf(tr["r0_8"]))  # nothing before the 8-bit phase
    np.testing.assert_array_equal(tr["r0_4"], np.full(64, 12.0))
