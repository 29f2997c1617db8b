"""Facts of binary16 arithmetic that the tensor-core batch kernel's grading rests
on, checked exhaustively or on dense samples on the CPU (numpy, IEEE 754):

- Section 3.1 grades a channel by the thresholds its |x| reaches (|x| >= theta,
  theta fp32). For every binary16 value a and every theta, a >= theta exactly
  when a >= RU16(theta), theta rounded up to binary16 (so the kernel may compare
  in binary16);
- x m with x and m binary16 and m in [1, 2) (the scale's significand) is exact in
  fp32, and hi = RN16(x m), lo = RN16(x m - hi) leave x m - hi - lo below half
  an ulp of lo: the two binary16 parts carry x m to about 22 bits, and the
  difference x m - hi is itself exact in fp32, so a fused multiply-add rounds it
  once, as the two-step form does;
- the bin midpoint and zero point enter as x s (mid - z) with x s exact in fp32."""
import numpy as np
import pytest

ALL_POS = np.arange(0, 0x7C01, dtype=np.uint16).view(np.float16)   # +0 .. +inf


def ru16(t):
    """Smallest binary16 >= t (t fp32), NaN for NaN."""
    t = np.float32(t)
    if np.isnan(t):
        return np.float16(np.nan)
    with np.errstate(over="ignore"):
        h = np.float16(t)
    if np.float32(h) < t:
        h = np.nextafter(h, np.float16(np.inf))
    return h


@pytest.mark.parametrize("seed", [1, 2])
def test_threshold_decision_survives_rounding_up(seed):
    rng = np.random.default_rng(seed)
    a32 = ALL_POS.astype(np.float32)
    ths = list(rng.lognormal(-2.0, 5.0, 1500).astype(np.float32))
    # values of binary16 and their fp32 neighbours, subnormal, zero, signs, overflow
    picks = ALL_POS[rng.integers(0, len(ALL_POS) - 1, 300)].astype(np.float32)
    ths += list(picks) + list(np.nextafter(picks, np.float32(np.inf))) + list(np.nextafter(picks, np.float32(0)))
    ths += [0.0, -0.0, -1.0, 1e-9, 5.9604645e-08, 6.1035156e-05, 65504.0, 65520.0, 70000.0, np.inf]
    for th in ths:
        th = np.float32(th)
        want = a32 >= th
        got = ALL_POS >= ru16(th)
        assert np.array_equal(want, got), th
    # NaN thresholds are reached by no |x|
    assert not np.any(ALL_POS >= ru16(np.float32(np.nan)))


def test_hi_lo_parts_of_x_times_significand():
    rng = np.random.default_rng(3)
    xb = rng.integers(0, 0x7C00, 200000).astype(np.uint16) | (rng.integers(0, 2, 200000).astype(np.uint16) << 15)
    x = xb.view(np.float16)
    m = (rng.integers(0, 1024, 200000).astype(np.uint16) | np.uint16(0x3C00)).view(np.float16)   # [1, 2)
    v = x.astype(np.float32) * m.astype(np.float32)
    # exact in fp32: the fp64 product of the same values agrees
    assert np.array_equal(v.astype(np.float64), x.astype(np.float64) * m.astype(np.float64))
    ok = np.abs(v) < 32768.0
    with np.errstate(over="ignore", invalid="ignore"):
        hi = v.astype(np.float16)
        d = v - hi.astype(np.float32)
    ok &= np.isfinite(d)
    # x m - hi is exact in fp32 (no rounding in the subtraction)
    assert np.array_equal(d[ok].astype(np.float64), v[ok].astype(np.float64) - hi[ok].astype(np.float64))
    lo = d[ok].astype(np.float16)
    r = v[ok].astype(np.float64) - hi[ok].astype(np.float64) - lo.astype(np.float64)
    # what is left is at most half an ulp of lo, or below the smallest binary16 step
    ulp_lo = np.spacing(np.abs(lo)).astype(np.float64)
    assert np.all(np.abs(r) <= np.maximum(0.5 * ulp_lo, 2.0 ** -25))
    # relative to x m: about 22 significant bits where nothing underflows
    big = np.abs(v[ok]) >= 2.0 ** -4
    assert np.all(np.abs(r[big]) <= np.abs(v[ok][big]) * 2.0 ** -21)


def test_x_times_scale_is_exact_in_fp32():
    rng = np.random.default_rng(4)
    x = rng.integers(0, 0x7C00, 100000).astype(np.uint16).view(np.float16)
    s = rng.integers(1, 0x7C00, 100000).astype(np.uint16).view(np.float16)
    with np.errstate(over="ignore"):
        p32 = x.astype(np.float32) * s.astype(np.float32)
    fin = np.isfinite(p32)
    p64 = x.astype(np.float64) * s.astype(np.float64)
    # no rounding unless the product leaves fp32's normal range
    tiny = np.abs(p64) < 2.0 ** -126
    sel = fin & ~tiny
    assert np.array_equal(p32[sel].astype(np.float64), p64[sel])
