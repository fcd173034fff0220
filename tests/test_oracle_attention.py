"""Pins for the oracle's mixed-precision attention (CPU).

* a 0/0/0/100 budget must give dense softmax attention (torch's fp64
  scaled_dot_product_attention is the reference), padding included;
* a partial 16-bit budget must give dense attention restricted to the kept
  key blocks (a boolean mask on the same library routine);
* a 100 % skip budget gives zeros;
* Q = 0 makes every score equal, which fixes the low-bit phases in closed form;
* the low-bit weights of one block, worked by hand from the format tables;
* a low-bit block far below a 16-bit block keeps its own reference (closed
  form), and the 4-bit phase's codes do not move against a larger power-of-two
  reference while the microblock scale stays normal;
* the output of a query block does not depend on how its key blocks are
  numbered or visited (relabelling the blocks leaves it unchanged);
* a single-precision low-bit budget stays within the error bound that P's
  quantisation alone allows, against exact attention on the dequantised
  operands;
* emulate mode differs from math mode only by bf16 rounding;
* the error decomposition's special cases and triangle inequality.
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


def test_p8_weights_by_hand():
    # one row, keys with log2 scores 0.3, -0.7, -1.7, -13 and an unused key:
    # r = ceil(0.3) = 1; p = 2^-0.7 = 0.61557, 2^-1.7 = 0.30779, 2^-2.7 =
    # 0.15389, 2^-14; 255 p = 156.97, 78.49, 39.24, 0.0156 -> codes 157, 78,
    # 39, 0
    x = np.array([[0.3, -0.7, -1.7, -13.0, -np.inf]])
    r, w = attention.p8_weights(x)
    assert r[0] == 1.0
    np.testing.assert_array_equal(w * 255.0, [[157.0, 78.0, 39.0, 0.0, 0.0]])
    # a block max on an integer: p = 1 exactly, code 255; midpoints go to the
    # even code (255 * 2^-1 = 127.5 -> 128)
    r, w = attention.p8_weights(np.array([[2.0, 1.0]]))
    assert r[0] == 2.0
    np.testing.assert_array_equal(w * 255.0, [[255.0, 128.0]])
    # the reference is the block's own: shifting every score by an integer
    # keeps the codes
    r2, w2 = attention.p8_weights(x - 37.0)
    assert r2[0] == -36.0
    np.testing.assert_array_equal(w2, attention.p8_weights(x)[1])


def test_p4_weights_by_hand():
    # one row of 16 keys (one microblock): x = 0.3 and -0.7 (log2 units), the
    # rest unused.  r = ceil(0.3) = 1; p = 2^-0.7 = 0.61557, 2^-1.7 = 0.30779;
    # 2688 p = 1654.66, 827.33; scale = e4m3(1654.66 / 6 = 275.78): e4m3 steps
    # by 32 in [256, 512), so 288; codes e2m1(1654.66 / 288 = 5.745) = 6 and
    # e2m1(827.33 / 288 = 2.873) = 3; weights 6*288/2688 = 9/14 and 3*288/2688 = 9/28
    x = np.full((1, 16), -np.inf)
    x[0, 0], x[0, 1] = 0.3, -0.7
    r, w = attention.p4_weights(x)
    assert r[0] == 1.0
    want = np.zeros((1, 16))
    want[0, 0], want[0, 1] = 9.0 / 14.0, 9.0 / 28.0
    np.testing.assert_allclose(w, want, rtol=1e-15, atol=0)


def test_p4_codes_stay_put_under_a_larger_power_of_two_reference():
    # NVFP4 of 2688 p against a reference 2^j higher: the e4m3 scale shifts by
    # 2^-j exactly while it stays normal (>= 2^-6), so the dequantised weights
    # are the same up to that factor.  (A kernel that keeps one power-of-two
    # reference per row rather than one per block relies on this.)
    rng = np.random.default_rng(5)
    x = rng.uniform(-6.0, 0.0, size=(64, 64))
    x[:, 0] = 0.0  # every row's block max at 2^0
    base = attention.p4_weights(x)[1]
    for j in range(1, 12):
        p = np.exp2(x - j)
        t = F.f32(attention.P4_RANGE * F.f32(p))
        codes, sf = F.nvfp4_quantize(t, axis=-1, block=16)
        w = F.nvfp4_dequantize(codes, sf) / attention.P4_RANGE * 2.0 ** j
        scale = F.e4m3_decode(sf)
        normal = np.repeat(scale >= 2.0 ** -6, 16, axis=-1)
        np.testing.assert_array_equal(w[normal], base[normal])
        if j <= 6:  # the microblock maxima lie within 2^-6 of the block max
            assert normal.all()


def _two_level_head(d=64):
    """One frame of 8x24 tokens = three full 8x8 regions (key blocks 0, 1, 2).
    Every query is 8 e_0; keys of block 0 are 8 e_0 (score 64/sqrt(64) = 8),
    keys of blocks 1 and 2 are 0 (score 0).  V rows are small integers."""
    p = Problem(1, 1, 1, 8, 24, d, 0.5, (0, 0, 0, 100))
    tab = geometry.block_tokens(p)
    q = np.zeros((p.N, d))
    q[:, 0] = 8.0
    k = np.zeros((p.N, d))
    k[tab[0], 0] = 8.0
    v = np.random.default_rng(3).integers(-3, 4, size=(p.N, d)).astype(np.float64)
    return p, prep.prepare_head(p, q, k, v), v, tab


@pytest.mark.parametrize("fmt", [8, 4])
def test_low_bit_block_far_below_keeps_its_own_reference(fmt):
    # block 0 at 16 bits scores 8, block 1 in the low-bit phase scores 0: its
    # p is taken against its own reference 2^ceil(0) = 1 (p = 1: INT8 code 255;
    # NVFP4 2688 p = 2688 exactly), so its 64 keys enter numerator and
    # denominator with weight e^-8 each.  (Against a shared running maximum
    # the INT8 codes would be round(255 e^-8) = 0.)
    p, pr, v, tab = _two_level_head()
    row = np.array([16, fmt, 0], dtype=np.uint8)
    out = attention.qblock_attention(pr, 0, row, p.d, "math")
    if fmt == 8:
        v1 = (pr["v_i8"][1].astype(np.float64) * pr["v_s8"][:, None]).T  # [S, d]
    else:
        v1 = prep.dequant_v_nvfp4(pr["v_f4"], pr["v_sf4"], pr["v_g4"])[1].T
    e = np.exp(-8.0)
    want = (v[tab[0]].sum(0) + e * v1.sum(0)) / (64.0 * (1.0 + e))
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=1e-12, atol=1e-15)


def _alternating_head(d=64):
    """One frame of 8x16 tokens = two 8x8 regions.  Every query is 8 e_0;
    the keys of block 0 alternate between 0 and -0.75 e_0 (even slots 0, odd
    slots -0.75); V rows are small integers."""
    p = Problem(1, 1, 1, 8, 16, d, 0.5, (0, 0, 0, 100))
    tab = geometry.block_tokens(p)
    q = np.zeros((p.N, d))
    q[:, 0] = 8.0
    k = np.zeros((p.N, d))
    k[tab[0][1::2], 0] = -0.75
    v = np.random.default_rng(4).integers(-3, 4, size=(p.N, d)).astype(np.float64)
    return p, prep.prepare_head(p, q, k, v), tab


@pytest.mark.parametrize("fmt", [8, 4])
def test_low_bit_weights_enter_the_denominator_quantised(fmt):
    # INT8: q codes 127 (scale 8/127), k codes 0 and -127 (scale 0.75/127):
    # scores 0 and -0.75, x = 0 and -1.082 log2, reference 2^0; p = 1 and
    # 2^-1.082 = 0.47237; codes 255 and round(120.45) = 120.  NVFP4: q = 8 -> scale e4m3(8/6) = 1.375, code 6,
    # so 8.25; k = -0.75 exactly; scores 0 and -0.7734, x = 0 and -1.1158 log2;
    # p = 1 and 0.4614; one 16-key microblock holds both, scale e4m3(2688/6) =
    # 448, codes 6 and e2m1(1240.3/448 = 2.77) = 3: weights 1 and 1/2.  The
    # output is the weighted mean of the dequantised V with exactly these
    # weights in numerator and denominator.
    p, pr, tab = _alternating_head()
    row = np.array([fmt, 0], dtype=np.uint8)
    out = attention.qblock_attention(pr, 0, row, p.d, "math")
    if fmt == 8:
        vd = (pr["v_i8"][0].astype(np.float64) * pr["v_s8"][:, None]).T  # [S, d]
        w_odd = 120.0 / 255.0
    else:
        vd = prep.dequant_v_nvfp4(pr["v_f4"], pr["v_sf4"], pr["v_g4"])[0].T
        w_odd = 0.5
    want = (vd[0::2].sum(0) + w_odd * vd[1::2].sum(0)) / (32.0 + 32.0 * w_odd)
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=1e-12, atol=1e-15)


def test_output_does_not_depend_on_block_numbering():
    # relabel the key blocks of one head (permute the block axis of every
    # prepared operand and of the precision row): each query block's output
    # must stay the same, since no block's contribution depends on another's
    pp, q, k, v = _inputs(Hh=16, Ww=24, budget=(30, 25, 25, 20))
    r = pipeline.run_head(pp, q, k, v, mode="math")
    pr, pmap = r["prep"], r["map"]
    perm = np.random.default_rng(11).permutation(pp.nb)
    keys = ("k_blocks", "k_i8", "k_s8", "k_f4", "k_sf4", "v_blocks", "v_i8", "v_f4", "v_sf4", "valid")
    pr2 = dict(pr)
    for key in keys:
        pr2[key] = pr[key][perm]
    for qb in range(pp.nb):
        a = attention.qblock_attention(pr, qb, pmap[qb], pp.d, "math")
        b = attention.qblock_attention(pr2, qb, pmap[qb][perm], pp.d, "math")
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fmt", [8, 4])
def test_low_bit_phase_within_p_quantisation_bound(fmt):
    budget = (0, 0, 100, 0) if fmt == 8 else (0, 100, 0, 0)
    p, q, k, v = _inputs(Hh=12, Ww=10, budget=budget)
    r = pipeline.run_head(p, q, k, v, mode="math")
    qd, kd, vd = _dequant_dense(p, r["prep"], fmt)
    exact = _sdpa(qd, kd, vd)
    # The output is sum(w~ v) / sum(w~) with w~ the quantised weights; against
    # the exact weights w: out - exact = sum((w~ - w)(v - exact)) / sum(w~).
    # Each |w~ - w| <= e 2^r_blk, e the largest rounding error of one
    # quantised p relative to its block's power-of-two reference (INT8: half a
    # step of 1/255; NVFP4: the top e2m1 half-step of the scale plus the
    # scale's own rounding, < 0.18).
    e = 0.5 / 255 if fmt == 8 else 0.18
    s = qd @ kd.T / np.sqrt(p.d)
    tab = r["prep"]["table"]
    m = s.max(1)
    w = np.exp(s - m[:, None])
    mb = np.zeros_like(s)
    for b in range(p.nb):
        toks = tab[b][tab[b] >= 0]
        mb[:, toks] = s[:, toks].max(1, keepdims=True)
    mb = np.ceil(mb * attention.LOG2E) * attention.LN2  # the power-of-two reference
    dw = e * np.exp(mb - m[:, None])
    w_low = np.maximum(w.sum(1) - dw.sum(1), 1e-300)
    bound = (np.einsum("nk,nkd->nd", dw, np.abs(vd[None, :, :] - exact[:, None, :]))) / w_low[:, None]
    err = np.abs(r["out"] - exact)
    assert err.max() > 0
    assert np.all(err <= bound * (1 + 1e-9) + 1e-12)
    # and the phase stays close to exact attention on its own operands
    assert _rel(r["out"], exact) < (0.005 if fmt == 8 else 0.05)


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


def _four_bit_running(pr, qb, pmap, d, S=64):
    """The 4-bit phase of query block ``qb`` as a tensor-core kernel that keeps
    the phase in one fp32 accumulator computes it: one power-of-two reference
    per row, started from the row maximum of the earlier phases and raised to
    ceil of a unit's maximum, over the key blocks of the query-block pair
    (2p, 2p+1) merged in ascending order and taken two at a time.  Returns the
    phase's (reference, sum, numerator) like a merged partial."""
    row = pmap[qb]
    other = pmap[qb ^ 1] if (qb ^ 1) < len(pmap) else np.zeros_like(row)
    valid, isd = pr["valid"], 1.0 / np.sqrt(d)
    x_run = np.full(S, -np.inf)
    q = pr["q_blocks"][qb]
    for kb in np.nonzero(row == 16)[0]:
        s = np.where(valid[kb][None], (q @ pr["k_blocks"][kb].T) * isd, -np.inf)
        x_run = np.maximum(x_run, s.max(1) * attention.LOG2E)
    qi = pr["q_i8"][qb].astype(np.float64)
    for kb in np.nonzero(row == 8)[0]:
        s = (qi @ pr["k_i8"][kb].astype(np.float64).T) * (pr["q_s8"][qb] * pr["k_s8"][kb] * isd)
        x_run = np.maximum(x_run, np.where(valid[kb][None], s, -np.inf).max(1) * attention.LOG2E)
    qd = F.nvfp4_dequantize(pr["q_f4"][qb], pr["q_sf4"][qb])
    kbs = np.nonzero((row == 4) | (other == 4))[0]
    R = np.where(np.isfinite(x_run), np.ceil(np.where(np.isfinite(x_run), x_run, 0)), -np.inf)
    acc, L = np.zeros((S, d)), np.zeros(S)
    for i in range(0, len(kbs), 2):
        xs = []
        for kb in kbs[i:i + 2]:
            kd = F.nvfp4_dequantize(pr["k_f4"][kb], pr["k_sf4"][kb])
            keep = valid[kb][None] & (row[kb] == 4)
            xs.append((kb, np.where(keep, (qd @ kd.T) * isd * attention.LOG2E, -np.inf)))
        um = np.max(np.stack([x.max(1) for _, x in xs]), 0)
        up = np.isfinite(um) & (~np.isfinite(R) | (um > R))
        Rn = np.where(up, np.ceil(np.where(up, um, 0)), R)
        fin = np.isfinite(R)
        a = np.where(up, np.where(fin, np.exp2(np.where(fin, R, 0) - np.where(up, Rn, 0)), 0.0), 1.0)
        acc *= a[:, None]
        L *= a
        R = Rn
        Rf = np.where(np.isfinite(R), R, 0.0)
        for kb, x in xs:
            p = np.where(np.isfinite(x), np.exp2(x - Rf[:, None]), 0.0)
            t = F.f32(attention.P4_RANGE * F.f32(p))
            c, sf = F.nvfp4_quantize(t, axis=-1, block=16)
            w = F.nvfp4_dequantize(c, sf) / attention.P4_RANGE
            acc += w @ F.nvfp4_dequantize(pr["v_f4"][kb], pr["v_sf4"][kb]).T
            L += w.sum(1)
    return np.where(np.isfinite(R), R * attention.LN2, -np.inf), L, acc * pr["v_g4"][None, :]


@pytest.mark.parametrize("budget", [(50, 50, 0, 0), (30, 60, 0, 10), (50, 25, 15, 10)])
def test_four_bit_running_reference_stays_close(budget):
    # One running power-of-two reference per row reproduces the per-block
    # reference's codes exactly while every microblock scale stays normal;
    # past that (a block more than ~2^-15 below the reference) the scale
    # loses bits.  On blob inputs the difference stays far inside the output
    # tolerance: relative L2 <= 1e-4 of the 4-bit phase's contribution.
    pp, q, k, v = _inputs(T=4, Hh=16, Ww=32, d=64, budget=budget, seed=2)
    r = pipeline.run_head(pp, q, k, v, mode="math")
    pr, pmap = r["prep"], r["map"]
    num = den = 0.0
    for qb in range(pp.nb):
        if not np.any(pmap[qb] == 4):
            continue
        st = attention._State(64, pp.d)
        for kb in np.nonzero(pmap[qb] == 4)[0]:
            kd = F.nvfp4_dequantize(pr["k_f4"][kb], pr["k_sf4"][kb])
            qd = F.nvfp4_dequantize(pr["q_f4"][qb], pr["q_sf4"][qb])
            x = np.where(pr["valid"][kb][None], (qd @ kd.T) * attention.LOG2E / np.sqrt(pp.d), -np.inf)
            rb, w = attention.p4_weights(x)
            st.merge(rb * attention.LN2, w.sum(1), w @ F.nvfp4_dequantize(pr["v_f4"][kb], pr["v_sf4"][kb]).T)
        want = st.o * pr["v_g4"][None, :] / np.where(st.l > 0, st.l, 1)[:, None]
        m, L, acc = _four_bit_running(pr, qb, pmap, pp.d)
        got = acc / np.where(L > 0, L, 1)[:, None]
        vv = pr["valid"][qb]
        num += float(((got - want)[vv] ** 2).sum())
        den += float((want[vv] ** 2).sum())
    assert den > 0
    assert (num / den) ** 0.5 <= 1e-4
