"""Pins the oracle's IEEE binary16 conversion against numpy's float16 cast.

The oracle writes the conversion out from the format's definition; numpy's
cast is an independent implementation of the same IEEE rounding (nearest,
ties to even).  The oracle additionally saturates at +-65504 instead of
overflowing to infinity and maps NaN to 0 (its stated scale-storage rule).
"""

import numpy as np


def _orc_vec(orc, xs):
    f = orc.lib().orc_float_to_half
    return np.array([f(float(x)) for x in xs], dtype=np.uint16)


def _np_half_bits(xs):
    with np.errstate(over="ignore"):
        h = np.asarray(xs, dtype=np.float32).astype(np.float16)
    a = np.abs(np.asarray(xs, dtype=np.float32))
    h = np.where(a >= 65504.0, np.copysign(np.float16(65504.0), h), h).astype(np.float16)
    h = np.where(np.isnan(np.asarray(xs, dtype=np.float32)), np.float16(0.0), h).astype(np.float16)
    return h.view(np.uint16)


def test_half_to_float_exhaustive(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    f = orc.lib().orc_half_to_float
    got = np.array([f(int(b)) for b in bits], dtype=np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_float_to_half_every_midpoint(orc):
    """Every tie between neighbouring finite halves, and points a float ulp either side."""
    h = np.arange(0, 0x7bff, dtype=np.uint16)          # positive finite halves but the max
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)            # exact in float32
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2)
    below = np.nextafter(mid, np.float32(0))
    above = np.nextafter(mid, np.float32(np.inf))
    xs = np.concatenate([mid, below, above, -mid, -above])
    assert np.array_equal(_orc_vec(orc, xs), _np_half_bits(xs))


def test_float_to_half_random_and_special(orc):
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-9, 6, 20000),
        np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.0, 65520.0, 1e30, -1e30, np.inf, -np.inf,
                  np.nan, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -14,
                  2.0 ** -14 * 0.99999, 6e-8, 3e-8], dtype=np.float32),
    ])
    assert np.array_equal(_orc_vec(orc, xs), _np_half_bits(xs))
