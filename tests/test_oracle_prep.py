"""Pins for the oracle's Q/K and V quantisers and its plain dense attention (CPU only).

V's INT8 codes are checked through the invariants of a symmetric per-channel
quantiser rather than by recomputing its formula: the channel's largest
magnitude maps to +-127, every value comes back within half a step, an
all-zero channel gives scale 0, and padding slots hold code 0.  NVFP4 V is
checked by an exact round trip of values built on the format's grid with a
different microscale for every (channel, 16-token group): that fails if the
microblocks ran along channels instead of along the tokens (the reduction axis
of P·V), or if the per-channel outer scale were off.  Q and K the same way:
one INT8 scale per 64-token block, NVFP4 microblocks along 16 channels of a
token.  The dense attention is checked against torch's fp64
scaled-dot-product attention.
"""

import numpy as np
import torch

from oracle import attention as OA, formats as F, prep as OP


def _table(n_tokens, nb, S=64):
    """Blocks of S consecutive tokens, the last one padded with -1."""
    t = np.arange(nb * S).reshape(nb, S)
    return np.where(t < n_tokens, t, -1)


def test_v_int8_per_channel_invariants():
    rng = np.random.default_rng(5)
    n, d = 100, 8
    v = rng.normal(size=(n, d)).astype(np.float32).astype(np.float64)
    v[:, 3] = 0.0  # an all-zero channel
    v[17, 5] = -9.0  # a negative extreme
    blocks, valid = OP.gather_blocks(v, _table(n, 2))
    amax = OP.v_channel_amax(v)
    codes_t, scale = OP.v_int8(blocks, amax)
    assert codes_t.shape == (2, d, 64) and codes_t.dtype == np.int8
    codes = codes_t.transpose(0, 2, 1).astype(np.int64)  # [nb, S, d]
    assert np.abs(codes).max() <= 127
    # the scale is the channel's absmax over 127 (to fp32 precision), 0 for the zero channel
    assert scale[3] == 0.0 and np.all(codes[..., 3] == 0)
    live = amax > 0
    np.testing.assert_allclose(scale[live] * 127.0, amax[live], rtol=2e-7)
    # the largest magnitude of every channel reaches the end of the code range, with its sign
    for c in np.nonzero(live)[0]:
        t = int(np.argmax(np.abs(v[:, c])))
        assert codes[t // 64, t % 64, c] == (127 if v[t, c] > 0 else -127)
    assert codes[17 // 64, 17 % 64, 5] == -127
    # every real value comes back within half a quantisation step; padding stays 0
    recon = codes * scale[None, None, :]
    err = np.abs(recon - blocks)[valid]
    assert np.all(err <= 0.5 * scale[None, :] * (1 + 1e-5) + 1e-12)
    assert np.all(codes[~valid] == 0)


def test_v_nvfp4_round_trips_on_its_grid_along_tokens():
    rng = np.random.default_rng(6)
    d, S = 3, 64
    g = np.array([1.0, 0.5, 0.25])  # per-channel outer scales (powers of two: exact)
    e2m1_vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e4m3_vals = np.unique(np.abs(F.e4m3_decode(np.arange(256))))
    e4m3_vals = e4m3_vals[np.isfinite(e4m3_vals) & (e4m3_vals >= 2.0 ** -6) & (e4m3_vals <= 448.0)]
    v = np.zeros((S, d))
    for c in range(d):
        for j in range(S // 16):
            # group 0 of every channel carries the channel's largest value, 6 * 448 * g
            s = 448.0 if j == 0 else float(rng.choice(e4m3_vals))
            vals = rng.choice(e2m1_vals, 16) * rng.choice([-1.0, 1.0], 16)
            vals[rng.integers(16)] = 6.0 * rng.choice([-1.0, 1.0])  # the microblock's max: sf = s exactly
            v[16 * j:16 * j + 16, c] = g[c] * s * vals
    blocks, valid = OP.gather_blocks(v, _table(S, 1))
    amax = OP.v_channel_amax(v)
    np.testing.assert_array_equal(amax, 6.0 * 448.0 * g)
    codes_t, sf_t, g_out = OP.v_nvfp4(blocks, amax)
    np.testing.assert_array_equal(g_out, g)
    assert codes_t.shape == (1, d, S) and sf_t.shape == (1, d, S // 16)
    back = OP.dequant_v_nvfp4(codes_t, sf_t, g_out)[0].T  # [S, d]
    np.testing.assert_array_equal(back, v)


def test_dense_attention_matches_torch_sdpa():
    rng = np.random.default_rng(7)
    for n, d in [(37, 16), (64, 64), (5, 128)]:
        q, k, v = (rng.normal(size=(n, d)) for _ in range(3))
        want = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(x)[None, None] for x in (q, k, v)))[0, 0].numpy()
        np.testing.assert_allclose(OA.dense_attention(q, k, v), want, rtol=1e-12, atol=1e-12)


def test_qk_int8_one_scale_per_block():
    rng = np.random.default_rng(8)
    n, d = 100, 16
    x = rng.normal(size=(n, d)).astype(np.float32).astype(np.float64)
    x[70:, :] *= 0.01  # the second block is much smaller: its own scale keeps its resolution
    blocks, valid = OP.gather_blocks(x, _table(n, 2))
    codes, scale = OP.qk_int8(blocks)
    assert codes.shape == (2, 64, d) and scale.shape == (2,)
    for b in range(2):
        amax = np.abs(blocks[b][valid[b]]).max()
        np.testing.assert_allclose(scale[b] * 127.0, amax, rtol=2e-7)
        assert np.abs(codes[b].astype(np.int64)).max() == 127
        err = np.abs(codes[b].astype(np.float64) * scale[b] - blocks[b])[valid[b]]
        assert np.all(err <= 0.5 * scale[b] * (1 + 1e-5) + 1e-12)
    assert np.all(codes[~valid] == 0)


def test_qk_nvfp4_round_trips_on_its_grid_along_channels():
    rng = np.random.default_rng(9)
    d = 64
    e2m1_vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e4m3_vals = np.unique(np.abs(F.e4m3_decode(np.arange(256))))
    e4m3_vals = e4m3_vals[np.isfinite(e4m3_vals) & (e4m3_vals >= 2.0 ** -6) & (e4m3_vals <= 448.0)]
    x = np.zeros((64, d))
    for t in range(64):
        for j in range(d // 16):  # one microscale per (token, 16 consecutive channels)
            s = float(rng.choice(e4m3_vals))
            vals = rng.choice(e2m1_vals, 16) * rng.choice([-1.0, 1.0], 16)
            vals[rng.integers(16)] = 6.0 * rng.choice([-1.0, 1.0])
            x[t, 16 * j:16 * j + 16] = s * vals
    blocks, _ = OP.gather_blocks(x, _table(64, 1))
    codes, sf = OP.qk_nvfp4(blocks)
    assert codes.shape == (1, 64, d) and sf.shape == (1, 64, d // 16)
    np.testing.assert_array_equal(F.nvfp4_dequantize(codes, sf), blocks)
