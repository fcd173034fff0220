"""Number formats used by the low-bit phases (oracle).

The pages name the formats but not their scales: INT8 for the 8-bit phase and
NVFP4 for the 4-bit phase (DraftAttention2 reading note, Method overview
bullet 2).  Written here from the format definitions:

* e4m3 (fp8 "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits;
  no infinities, max finite 448, min normal 2^-6, subnormals m * 2^-9.
* e2m1 (fp4): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; the values are
  +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}.

Rounding is round-to-nearest, ties to even, with saturation to the largest
finite value ("satfinite").  A negative input that rounds to zero keeps its
sign (IEEE rule), so its code has the sign bit set.

All functions take float64 arrays holding values that are already exact fp32
numbers and return exact results; fp32 operations are spelled out with
``np.float32`` so that each rounding step is visible.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0


def _round_to_grid(x, min_exp: int, mant_bits: int, vmax: float):
    """RNE onto a floating grid with exponent floor ``min_exp`` (subnormals below
    2^min_exp share its quantum) and ``mant_bits`` mantissa bits; saturates."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # log2 can be off by one next to powers of two; correct it exactly
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= a, e + 1, e)
    e = np.maximum(e, min_exp)
    quantum = np.ldexp(1.0, (e - mant_bits).astype(np.int64))
    r = np.rint(a / quantum) * quantum  # np.rint: half to even; a/quantum exact
    r = np.minimum(r, vmax)
    r = np.where(a > 0, r, 0.0)
    return np.copysign(r, x)


def e4m3_round(x):
    """Value of e4m3 RNE-satfinite(x)."""
    return _round_to_grid(x, -6, 3, E4M3_MAX)


def e2m1_round(x):
    """Value of e2m1 RNE-satfinite(x)."""
    return _round_to_grid(x, 0, 1, E2M1_MAX)


def e4m3_encode(v):
    """Bit pattern (uint8) of an e4m3 value produced by ``e4m3_round``."""
    v = np.asarray(v, dtype=np.float64)
    s = np.signbit(v).astype(np.uint8)
    a = np.abs(v)
    out = np.zeros(a.shape, dtype=np.uint8)
    sub = a < 2.0 ** -6
    m_sub = np.rint(a / 2.0 ** -9).astype(np.int64)  # exact for grid values
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(sub, 1.0, a))).astype(np.int64)
    m_nor = np.rint((a / np.ldexp(1.0, e) - 1.0) * 8).astype(np.int64)
    out = np.where(sub, m_sub, ((e + 7) << 3) | m_nor).astype(np.uint8)
    return out | (s << 7)


def e4m3_decode(code):
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, e - 7))
    return s * val


def e2m1_encode(v):
    """Nibble code (uint8, 0..15) of an e2m1 value produced by ``e2m1_round``."""
    v = np.asarray(v, dtype=np.float64)
    s = np.signbit(v).astype(np.uint8)
    a = np.abs(v)
    # magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 are codes 0..7 in order
    mag = np.searchsorted(np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]), a)
    return (mag.astype(np.uint8) | (s << 3)).astype(np.uint8)


def e2m1_decode(code):
    c = np.asarray(code, dtype=np.int64)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    return np.where(c & 0x8, -1.0, 1.0) * mags[c & 0x7]


def f32(x):
    """Round to fp32 (the precision every scale and product below is taken in)."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def f32_div(a, b):
    return (np.asarray(a, np.float32) / np.asarray(b, np.float32)).astype(np.float64)


def f32_mul(a, b):
    return (np.asarray(a, np.float32) * np.asarray(b, np.float32)).astype(np.float64)


def int8_quantize(x, amax):
    """Symmetric INT8: scale = fp32(amax/127), codes = clamp(rint(fp32(x * fp32(127/amax))), ±127).

    ``amax == 0`` gives scale 0 and all-zero codes.  Returns (codes int8, scale)."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.asarray(amax, dtype=np.float64)
    safe = np.where(amax > 0, amax, 1.0)
    inv = f32_div(127.0, safe)
    y = f32_mul(x, inv)
    c = np.clip(np.rint(y), -127, 127)
    c = np.where(amax > 0, c, 0.0)
    scale = np.where(amax > 0, f32_div(safe, 127.0), 0.0)
    return c.astype(np.int8), scale


def nvfp4_quantize(x, axis=-1, block=16):
    """NVFP4 along ``axis`` in microblocks of ``block`` consecutive elements.

    Per microblock: sf = e4m3(fp32(amax / 6)); a zero sf gives all-zero codes;
    otherwise code = e2m1(fp32(x * fp32(1 / sf))).  Returns
    (e2m1 nibble codes uint8 with x's shape, e4m3 sf codes uint8 with the
    blocked axis divided by ``block``)."""
    x = np.moveaxis(np.asarray(x, dtype=np.float64), axis, -1)
    n = x.shape[-1]
    assert n % block == 0
    xb = x.reshape(x.shape[:-1] + (n // block, block))
    amax = np.abs(xb).max(-1)
    sf_val = e4m3_round(f32_div(amax, 6.0))
    nz = sf_val > 0
    inv = np.where(nz, f32_div(1.0, np.where(nz, sf_val, 1.0)), 0.0)
    y = f32_mul(xb, inv[..., None])
    codes = e2m1_encode(e2m1_round(y))
    codes = np.where(nz[..., None], codes, 0).astype(np.uint8)
    codes = np.moveaxis(codes.reshape(x.shape), -1, axis)
    sf = np.moveaxis(e4m3_encode(sf_val), -1, axis)
    return codes, sf


def nvfp4_dequantize(codes, sf, axis=-1, block=16):
    c = np.moveaxis(np.asarray(codes), axis, -1)
    s = np.moveaxis(np.asarray(sf), axis, -1)
    vals = e2m1_decode(c).reshape(c.shape[:-1] + (c.shape[-1] // block, block))
    out = vals * e4m3_decode(s)[..., None]
    return np.moveaxis(out.reshape(c.shape), -1, axis)
