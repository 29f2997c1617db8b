"""Pins for the oracle's grading ("GRINQH" Section 3.1) and per-class compaction,
against numpy's searchsorted / stable argsort (independent library routines)."""
import numpy as np

from activation_graded_bit_b200 import workloads as wl

CL = np.array([0, 2, 3, 4, 8], np.uint8)


def _class_index_np(x_bits, theta):
    ax = np.abs(x_bits.view(np.float16).astype(np.float64))
    j = np.searchsorted(np.asarray(theta, np.float64), ax, side="right")
    j[np.isnan(ax)] = 0
    return j


def test_grade_matches_searchsorted(orc):
    x = wl.activations_outlier(4096, 1, key=(99, 1))[0]
    theta = np.array([0.3, 0.8, 1.5, 2.6], np.float32)
    bits = orc.grade(x, theta, CL)
    assert np.array_equal(bits, CL[_class_index_np(x, theta)])


def test_grade_ties_nan_zero(orc):
    theta = np.array([0.5, 1.0, 2.0, 4.0], np.float32)
    vals = np.array([0.5, 1.0, 2.0, 4.0, -4.0, 0.0, -0.0, np.nan, np.inf, 0.499], np.float16)
    bits = orc.grade(vals.view(np.uint16), theta, CL)
    # |x| == theta_i belongs to the upper class; NaN and 0 to class 0
    assert list(bits) == [2, 3, 4, 8, 8, 0, 0, 0, 8, 0]
    # a zero threshold puts +-0 into class 1
    bits = orc.grade(np.array([0.0, -0.0], np.float16).view(np.uint16),
                     np.array([0.0, 1, 2, 3], np.float32), CL)
    assert list(bits) == [2, 2]


def test_grade_is_a_count_for_unsorted_thresholds(orc):
    x = wl.activations_gaussian(512, 1, key=(99, 2))[0]
    theta = np.array([1.0, 0.2, 3.0, 0.7], np.float32)
    ax = np.abs(x.view(np.float16).astype(np.float64))
    cnt = (ax[:, None] >= theta[None, :].astype(np.float64)).sum(1)
    assert np.array_equal(orc.grade(x, theta, CL), CL[cnt])


def test_compact_matches_stable_argsort(orc):
    g = np.random.default_rng(5)
    for K in (1, 7, 1024, 4099):
        j = g.integers(0, 5, K)
        bits = CL[j]
        idx, off = orc.compact(bits, CL)
        assert np.array_equal(idx, np.argsort(j, kind="stable"))
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(j, minlength=5))]))


def test_compact_empty_and_missing_class(orc):
    idx, off = orc.compact(np.zeros(0, np.uint8), CL)
    assert len(idx) == 0 and list(off) == [0] * 6
    bits = np.array([8, 8, 0, 8], np.uint8)
    idx, off = orc.compact(bits, CL)
    assert list(idx) == [2, 0, 1, 3] and list(off) == [0, 1, 1, 1, 1, 4]
