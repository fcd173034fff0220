"""Pins for the oracle's number formats (CPU only).

The e4m3 rounding is checked against torch's float8_e4m3fn cast (a library
implementation of the same format), the e2m1 rounding against a hand table,
and the INT8 / NVFP4 quantisers against exact round trips of values already on
their grids.
"""

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle.attention import bf16_round


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(0)
    # all grid points, all midpoints between neighbours, and random values
    grid = np.unique(np.abs(F.e4m3_decode(np.arange(256))[np.isfinite(F.e4m3_decode(np.arange(256)))]))
    grid = grid[grid <= 448]
    mids = (grid[1:] + grid[:-1]) / 2
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), 20000))
    x = np.concatenate([grid, mids, rnd, -rnd, [0.0, 2.0 ** -10, 3 * 2.0 ** -11]])
    x = x.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(F.e4m3_round(x), _torch_e4m3(x))


def test_e4m3_saturates_and_codes_round_trip():
    assert F.e4m3_round(500.0) == 448.0 and F.e4m3_round(1e9) == 448.0
    assert F.e4m3_round(-470.0) == -448.0
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])  # 0x7F/0xFF are NaN
    vals = F.e4m3_decode(codes)
    np.testing.assert_array_equal(F.e4m3_round(vals), vals)
    np.testing.assert_array_equal(F.e4m3_encode(vals), codes.astype(np.uint8))
    # decode agrees with torch's reinterpretation of the same byte
    tv = torch.from_numpy(codes.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(vals, tv.astype(np.float64))


def test_e2m1_hand_table(golden):
    t = golden("e2m1_rounding.json")["cases"]
    x = np.array([c[0] for c in t], dtype=np.float32).astype(np.float64)
    want_v = np.array([c[1] for c in t])
    want_c = np.array([c[2] for c in t], dtype=np.uint8)
    got_v = F.e2m1_round(x)
    np.testing.assert_array_equal(got_v, want_v)
    np.testing.assert_array_equal(np.signbit(got_v), np.signbit(want_v))
    np.testing.assert_array_equal(F.e2m1_encode(got_v), want_c)


def test_e2m1_codes_round_trip():
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_decode(codes)
    np.testing.assert_array_equal(F.e2m1_round(vals), vals)
    np.testing.assert_array_equal(F.e2m1_encode(vals), codes)


def test_int8_round_trip_on_grid():
    rng = np.random.default_rng(1)
    for s in (2.0 ** -5, 3 * 2.0 ** -7, 5 * 2.0 ** -3, 7.0):
        c = rng.integers(-127, 128, size=(64, 128)).astype(np.float64)
        c[3, 5] = 127.0  # the block reaches the top code
        x = c * s
        codes, scale = F.int8_quantize(x, np.abs(x).max())
        assert float(scale) == s
        np.testing.assert_array_equal(codes.astype(np.float64), c)
        np.testing.assert_array_equal(codes.astype(np.float64) * scale, x)


def test_int8_zero_block_and_clamp():
    codes, scale = F.int8_quantize(np.zeros((4, 4)), 0.0)
    assert float(scale) == 0.0 and not codes.any()
    # a value above amax (never happens in prep, but the clamp must hold)
    codes, _ = F.int8_quantize(np.array([2.0, -2.0]), 1.0)
    assert list(codes) == [127, -127]


def test_nvfp4_round_trip_on_grid():
    rng = np.random.default_rng(2)
    e2 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for sf in (0.171875, 1.0, 2.0 ** -7, 3.5, 448.0 / 6 * 0 + 72.0):
        sfv = F.e4m3_round(sf)
        assert sfv == sf
        vals = rng.choice(e2, size=(8, 64)) * rng.choice([-1, 1], size=(8, 64))
        vals[:, ::16] = 6.0  # every microblock reaches the top code
        x = vals * sf
        codes, sfc = F.nvfp4_quantize(x)
        np.testing.assert_array_equal(F.e4m3_decode(sfc), np.full((8, 4), sf))
        np.testing.assert_array_equal(F.nvfp4_dequantize(codes, sfc), x)


def test_nvfp4_axis_and_zero_microblock():
    x = np.zeros((32, 3))
    x[16:, 1] = np.linspace(-1, 1, 16)
    codes, sf = F.nvfp4_quantize(x, axis=0)
    assert codes.shape == (32, 3) and sf.shape == (2, 3)
    assert not codes[:16].any() and not sf[0].any()
    back = F.nvfp4_dequantize(codes, sf, axis=0)
    assert np.abs(back - x).max() <= float(F.e4m3_decode(sf[1, 1])) * 1.0 + 1e-12


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(50000) * np.exp(rng.uniform(-20, 20, 50000))
    # exact ties: bf16 value + half an ulp
    base = torch.randn(1000).bfloat16().float().numpy().astype(np.float64)
    ulp = np.abs(base) * 2.0 ** -8
    x = np.concatenate([x, base + ulp / 2, base - ulp / 2]).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(bf16_round(x), want)


@pytest.mark.parametrize("v", [0.0, -0.0])
def test_signed_zero_codes(v):
    assert F.e2m1_encode(F.e2m1_round(v)) == (8 if np.signbit(v) else 0)


def test_bf16_rounding_commutes_with_powers_of_two():
    # the 16-bit phase's P rounding relies on it: rounding relative to any
    # integer-exponent reference gives the same value
    rng = np.random.default_rng(4)
    x = rng.random(20000) * np.exp(rng.uniform(-30, 0, 20000))
    for k in (-8, -3, 1, 5, 8):
        np.testing.assert_array_equal(bf16_round(x * 2.0 ** k), bf16_round(x) * 2.0 ** k)
