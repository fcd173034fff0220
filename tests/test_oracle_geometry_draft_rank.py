"""Pins for the oracle's region packing, pooling, draft map and ranking (CPU).

Region packing and budget counts are checked against hand-worked tables;
pooling against torch's own 2-D pooling routines; the draft map against a
hand-worked two-region case and its lambda = 0 / lambda = 1 special cases; the
ranking against the brute-force definition of a rank.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import draft, geometry, prep, rank
from oracle.problem import Problem


def P(T, Hh, Ww, d=16, H=1, lam=0.5, budget=(25, 25, 25, 25)):
    return Problem(1, H, T, Hh, Ww, d, lam, tuple(budget))


# ---------------------------------------------------------------- geometry

@pytest.mark.parametrize("T,Hh,Ww", [(1, 8, 8), (2, 16, 16), (3, 45, 80), (2, 48, 84), (1, 10, 13), (4, 1, 1)])
def test_block_table_is_bijection(T, Hh, Ww):
    p = P(T, Hh, Ww)
    tab = geometry.block_tokens(p)
    real = tab[tab >= 0]
    assert tab.shape == (p.nb, 64)
    np.testing.assert_array_equal(np.sort(real), np.arange(p.N))
    assert (tab < 0).sum() == p.nb * 64 - p.N
    # every region keeps at least one real token
    assert (tab >= 0).any(1).all()


def test_block_table_hand_cases(golden):
    for case in golden("region_table.json")["cases"]:
        p = Problem(1, 1, case["T"], case["Hh"], case["Ww"], 16, 0.5, (25, 25, 25, 25), case["rh"], case["rw"])
        tab = geometry.block_tokens(p)
        assert p.nb == case["nb"]
        for blk, slot, tok in case["entries"]:
            assert tab[blk, slot] == tok, (blk, slot)


def test_budget_counts_table(golden):
    for case in golden("budget_counts.json")["cases"]:
        wl = oracle.CONFIGS[case["name"]]
        assert wl.nb == case["nb"]
        assert tuple(wl.budget) == tuple(float(x) for x in case["budget"])
        got = geometry.budget_counts(wl)
        assert got == (case["n16"], case["n8"], case["n4"], case["skip"]), case["name"]
        assert sum(got) == case["P"]


def test_budget_counts_follow_percentages():
    p = P(3, 45, 80, budget=(33.3, 22.2, 11.1, 33.4))
    n16, n8, n4, sk = geometry.budget_counts(p)
    pairs = p.nb ** 2
    for n, pct in ((n16, 33.4), (n8, 11.1), (n4, 22.2)):
        assert abs(n - pairs * pct / 100) <= 1.0
    with pytest.raises(ValueError):
        geometry.budget_counts(P(1, 8, 8, budget=(0, 50, 50, 10)))


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("T,Hh,Ww", [(2, 16, 16), (2, 10, 13), (1, 45, 20)])
def test_pooling_matches_torch_pool2d(T, Hh, Ww):
    p = P(T, Hh, Ww, d=8)
    g = torch.Generator().manual_seed(5)
    x = torch.randn(p.N, 8, generator=g, dtype=torch.float64)
    blocks, valid = prep.gather_blocks(x.numpy(), geometry.block_tokens(p))
    avg, mx = prep.pool(blocks, valid)
    img = x.reshape(T, Hh, Ww, 8).permute(0, 3, 1, 2)  # frames as a batch, channels
    t_avg = torch.nn.functional.avg_pool2d(img, 8, 8, ceil_mode=True, count_include_pad=False)
    t_max = torch.nn.functional.max_pool2d(img, 8, 8, ceil_mode=True)
    # [T, d, nRy, nRx] → block order [(t, ry, rx), d]
    t_avg = t_avg.permute(0, 2, 3, 1).reshape(-1, 8).numpy()
    t_max = t_max.permute(0, 2, 3, 1).reshape(-1, 8).numpy()
    np.testing.assert_allclose(avg, t_avg, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(mx, t_max)


def test_maxpool_is_signed_and_ignores_padding():
    p = P(1, 9, 9, d=1)
    x = -np.arange(1, p.N + 1, dtype=np.float64)[:, None]  # all negative
    blocks, valid = prep.gather_blocks(x, geometry.block_tokens(p))
    _, mx = prep.pool(blocks, valid)
    # block 3 holds only token (8, 8) = 80 → value -81; a padding zero must not win
    assert mx[3, 0] == -81.0
    assert mx[0, 0] == -1.0


# ---------------------------------------------------------------- draft map

def test_draft_hand_case(golden):
    g = golden("draft_hand.json")
    args = [np.array(g[k], dtype=np.float64) for k in ("q_avg", "k_avg", "q_max", "k_max")]
    for case in g["cases"]:
        D = draft.draft_map(*args, case["lam"], g["d"])
        np.testing.assert_allclose(D, np.array(case["D"]), rtol=1e-14, atol=0)


def test_draft_lambda_special_cases():
    rng = np.random.default_rng(7)
    qa, ka, qm, km = (rng.standard_normal((12, 32)) * 3 for _ in range(4))
    a = torch.from_numpy(qa @ ka.T / np.sqrt(32)).softmax(-1).numpy()
    b = torch.from_numpy(qm @ km.T / np.sqrt(32)).softmax(-1).numpy()
    np.testing.assert_allclose(draft.draft_map(qa, ka, qm, km, 0.0, 32), a, rtol=1e-13)
    np.testing.assert_allclose(draft.draft_map(qa, ka, qm, km, 1.0, 32), b, rtol=1e-13)
    D = draft.draft_map(qa, ka, qm, km, 0.3, 32)
    np.testing.assert_allclose(D.sum(1), 1.0, rtol=1e-13)


# ---------------------------------------------------------------- ranking

def _brute_ranks(D):
    f = D.ravel().astype(np.float64)
    n = f.size
    r = np.zeros(n, dtype=np.int64)
    for i in range(n):
        r[i] = np.sum(f > f[i]) + np.sum((f == f[i]) & (np.arange(n) < i))
    return r.reshape(D.shape)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ranks_match_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    D = rng.choice(np.array([0.0, 1e-3, 0.25, 0.5, 0.5000001], dtype=np.float32), size=(9, 9))
    D[0, 0] = -0.0
    np.testing.assert_array_equal(rank.pair_ranks(D), _brute_ranks(D))


def test_assign_counts_order_and_ties():
    rng = np.random.default_rng(4)
    D = rng.random((20, 20)).astype(np.float32)
    m = rank.assign(D, 40, 60, 100)
    assert [(m == v).sum() for v in (16, 8, 4, 0)] == [40, 60, 100, 200]
    # higher score never gets a lower precision
    lv = {16: 3, 8: 2, 4: 1, 0: 0}
    lvl = np.vectorize(lv.get)(m)
    for a in range(3):
        assert D[lvl == a + 1].min() >= D[lvl == a].max()
    # all-equal scores: the lowest pair indices win
    m = rank.assign(np.full((5, 5), 0.2, np.float32), 3, 2, 1)
    assert list(m.ravel()[:7]) == [16, 16, 16, 8, 8, 4, 0]


def test_rank_rejects_nonfinite():
    with pytest.raises(ValueError):
        rank.pair_ranks(np.array([[1.0, np.nan]], np.float32))
