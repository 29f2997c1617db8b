"""Pins for the oracle's binary16 conversions against numpy's (a library routine
that implements the same IEEE 754 definition independently)."""
import numpy as np


def _np_f16_to_f64(h):
    return np.array([h], np.uint16).view(np.float16).astype(np.float64)[0]


def _np_f64_to_f16(v):
    return int(np.array([v], np.float64).astype(np.float16).view(np.uint16)[0])


def test_every_half_decodes_like_numpy(orc):
    allh = np.arange(65536, dtype=np.uint16)
    ref = allh.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(int(h)) for h in allh])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    # signed zeros keep their sign
    assert np.signbit(orc.f16_to_f64(0x8000)) and not np.signbit(orc.f16_to_f64(0x0000))


def test_round_trip_every_finite_half(orc):
    for h in range(65536):
        v = _np_f16_to_f64(h)
        if np.isnan(v):
            continue
        assert orc.f64_to_f16(v) == h


def test_midpoints_round_to_even(orc):
    # every midpoint between consecutive positive finite halves is a tie in the
    # binary16 grid; IEEE round-to-nearest-even must pick the even significand
    for h in range(0, 0x7BFF):
        a, b = _np_f16_to_f64(h), _np_f16_to_f64(h + 1)
        mid = (a + b) / 2.0          # exact in fp64
        want = h if (h & 1) == 0 else h + 1
        assert orc.f64_to_f16(mid) == want, hex(h)
        assert orc.f64_to_f16(-mid) == want | 0x8000


def test_random_doubles_match_numpy(orc):
    g = np.random.default_rng(7)
    vals = np.concatenate([
        g.standard_normal(20000) * 10.0 ** g.uniform(-9, 5, 20000),
        g.uniform(65400, 65600, 2000), g.uniform(0, 1e-7, 2000)])
    for v in vals:
        assert orc.f64_to_f16(v) == _np_f64_to_f16(v), v


def test_overflow_and_specials(orc):
    assert orc.f64_to_f16(65504.0) == 0x7BFF
    assert orc.f64_to_f16(65519.999) == 0x7BFF
    assert orc.f64_to_f16(65520.0) == 0x7C00          # tie -> even -> infinity
    assert orc.f64_to_f16(float("inf")) == 0x7C00
    assert orc.f64_to_f16(-1e300) == 0xFC00
    assert (orc.f64_to_f16(float("nan")) & 0x7C00) == 0x7C00 and (orc.f64_to_f16(float("nan")) & 0x3FF)
    assert orc.f64_to_f16(2.0 ** -25) == 0x0000        # tie between 0 and 2^-24 -> 0
    assert orc.f64_to_f16(3 * 2.0 ** -25) == 0x0002    # tie between 1 and 2 ulps -> 2
    assert orc.f64_to_f16(-0.0) == 0x8000
