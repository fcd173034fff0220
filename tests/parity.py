"""Stage-by-stage comparison of the CUDA path with the CPU oracle.

Used by the ``-m gpu`` tests.  Every comparison takes the GPU's intermediate
buffers (read through ``da2_debug_view``) and the oracle's results for the same
bf16 inputs; the oracle never sees a GPU value except where a stage's input is
deliberately taken from the GPU (the ranking is checked on the GPU's fp32
scores, the attention on the GPU's assignment), so that each stage is judged on
its own.

Tolerances (from the stated parity bar):
* bit-exact: permutation, pooled max, INT8/NVFP4 codes and scales, assignment;
* pooled mean: |g - o| <= 1e-4 |o| + 1e-4 rms(o);
* draft scores: relative 1e-4 where D >= 1e-30, absolute 1e-30 below;
* output: relative L2 <= 2e-3 against the oracle's emulation of the same
  quantisation (bf16 P in the 16-bit phase, bf16 output).
"""

from __future__ import annotations

import numpy as np
import torch

from mixed_precision_block_b200 import da2
from oracle import attention as OA, geometry as OG, prep as OP, rank as OR, draft as ODR
from oracle.pipeline import to_f64
from oracle.problem import Problem

OUT_TOL = 2e-3


def oracle_problem(wl) -> Problem:
    return Problem.from_workload(wl)


def run_gpu(wl, q, k, v, stages=("prep", "draft", "attn")):
    p = da2.Problem.from_workload(wl)
    ws = da2.workspace(p, q.device)
    out = torch.zeros_like(q)
    if "prep" in stages:
        da2.da2_prepare(p, q, k, v, ws)
    if "draft" in stages:
        da2.da2_draft_rank(p, ws)
    if "attn" in stages:
        da2.da2_attention(p, q, k, v, ws, out)
    torch.cuda.synchronize()
    return p, ws, out


def unpack_nibbles(t):
    t = t.cpu().numpy().astype(np.uint8)
    out = np.empty(t.shape[:-1] + (t.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = t & 15
    out[..., 1::2] = t >> 4
    return out


def qk_sf_natural(atoms):
    """[nb, d/64, 32, 16] scale atoms -> [nb, 64, d/16] (slot, microblock); checks the repeat."""
    a = np.asarray(atoms)
    nb, nch = a.shape[0], a.shape[1]
    words = a.reshape(nb, nch, 32, 4, 4)  # [blk, chunk, line, word, byte]
    np.testing.assert_array_equal(words[:, :, :, 2:], words[:, :, :, :2])
    out = np.empty((nb, 64, nch * 4), dtype=np.uint8)
    for w in range(2):
        for c in range(nch):
            out[:, 32 * w:32 * w + 32, 4 * c:4 * c + 4] = words[:, c, :, w, :]
    return out


def v_sf_natural(atoms, d):
    """[nb, 32, 16] scale atoms -> [nb, d, 4] (channel, microblock)."""
    a = np.asarray(atoms).reshape(-1, 32, 4, 4)  # [blk, line, word, byte]
    out = np.empty((a.shape[0], d, 4), dtype=np.uint8)
    for w in range(d // 32):
        out[:, 32 * w:32 * w + 32, :] = a[:, :, w, :]
    return out


def g(p, ws, name, bh=None):
    t = da2.view(p, ws, name)
    if bh is not None and name != "PERM":
        t = t[bh]
    return t.cpu().numpy()


def check_perm(p, ws, op):
    np.testing.assert_array_equal(g(p, ws, "PERM").astype(np.int64), OG.block_tokens(op))


def check_prep_head(p, ws, op, pr, bh, n8, n4, blocks=None):
    """Bit-exact / 1e-4 checks of one head's prepared operands (all or some blocks)."""
    sel = slice(None) if blocks is None else np.asarray(blocks)
    for t in ("q", "k"):
        T = t.upper()
        avg_g = g(p, ws, f"{T}_AVG", bh)[sel].astype(np.float64)
        avg_o = pr[f"{t}_avg"][sel]
        rms = np.sqrt(np.mean(pr[f"{t}_avg"] ** 2))
        assert np.all(np.abs(avg_g - avg_o) <= 1e-4 * np.abs(avg_o) + 1e-4 * rms), f"{T}_AVG"
        np.testing.assert_array_equal(g(p, ws, f"{T}_MAX", bh)[sel].astype(np.float64), pr[f"{t}_max"][sel])
        if n8:
            np.testing.assert_array_equal(g(p, ws, f"{T}_I8", bh)[sel], pr[f"{t}_i8"][sel], err_msg=f"{T}_I8")
            np.testing.assert_array_equal(g(p, ws, f"{T}_S8", bh)[sel].astype(np.float64), pr[f"{t}_s8"][sel])
        if n4:
            np.testing.assert_array_equal(unpack_nibbles(da2.view(p, ws, f"{T}_F4")[bh])[sel], pr[f"{t}_f4"][sel],
                                          err_msg=f"{T}_F4")
            np.testing.assert_array_equal(qk_sf_natural(g(p, ws, f"{T}_SF4", bh))[sel], pr[f"{t}_sf4"][sel],
                                          err_msg=f"{T}_SF4")
    if n8:
        # V's INT8 codes are held as bf16 values in [block][slot][channel] order
        v8 = da2.view(p, ws, "V_I8")[bh].float().cpu().numpy().astype(np.int64).transpose(0, 2, 1)
        np.testing.assert_array_equal(v8[sel], pr["v_i8"][sel].astype(np.int64), err_msg="V_I8")
        np.testing.assert_array_equal(g(p, ws, "V_S8", bh).astype(np.float64), pr["v_s8"])
    if n4:
        np.testing.assert_array_equal(unpack_nibbles(da2.view(p, ws, "V_F4")[bh])[sel], pr["v_f4"][sel],
                                      err_msg="V_F4")
        np.testing.assert_array_equal(v_sf_natural(g(p, ws, "V_SF4", bh), op.d)[sel], pr["v_sf4"][sel],
                                      err_msg="V_SF4")
        np.testing.assert_array_equal(g(p, ws, "V_G4", bh).astype(np.float64), pr["v_g4"])


def check_scores_rows(scores_gpu, D_oracle):
    """Draft scores: relative 1e-4 (absolute 1e-30 for D below 1e-30)."""
    d64 = scores_gpu.astype(np.float64)
    err = np.abs(d64 - D_oracle)
    big = D_oracle >= 1e-30
    assert np.all(err[big] <= 1e-4 * D_oracle[big]), float((err[big] / D_oracle[big]).max())
    assert np.all(err[~big] <= 1e-30)


def check_assignment(p, ws, op, bh, scores_gpu):
    n16, n8, n4, _ = OG.budget_counts(op)
    want = OR.assign(scores_gpu, n16, n8, n4)
    got = g(p, ws, "MAP", bh)
    np.testing.assert_array_equal(got, want)
    # lists / counts agree with the map
    counts = g(p, ws, "COUNTS", bh)
    lists = g(p, ws, "LISTS", bh).astype(np.int64) & 0xFFFF
    for qb in range(0, got.shape[0], max(1, got.shape[0] // 64)):
        c16, c8, c4 = counts[qb, :3]
        row = lists[qb]
        for prec, lo, hi in ((16, 0, c16), (8, c16, c16 + c8), (4, c16 + c8, c16 + c8 + c4)):
            np.testing.assert_array_equal(row[lo:hi], np.nonzero(got[qb] == prec)[0])
    return got


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def oracle_rows(op, pr, prec_map, qblocks, mode="emulate"):
    """Oracle output rows of the given query blocks in token order: (tokens, rows)."""
    tab = pr["table"]
    toks, rows = [], []
    for qb in qblocks:
        o = OA.qblock_attention(pr, qb, prec_map[qb], op.d, mode)
        ok = tab[qb] >= 0
        toks.append(tab[qb][ok])
        rows.append(o[ok])
    return np.concatenate(toks), np.concatenate(rows)


def dense_rows(qh, kh, vh, toks):
    """fp64 dense attention for the given query tokens of one head."""
    s = (qh[toks] @ kh.T) / np.sqrt(qh.shape[1])
    s -= s.max(1, keepdims=True)
    w = np.exp(s)
    return (w @ vh) / w.sum(1, keepdims=True)


def head_inputs(q, k, v, bh, B, H):
    b, h = divmod(bh, H)
    return to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
