"""Pins for the oracle's 8-bit RTN quantiser ("GRINQH" Section 3.3 and Section 4:
uniform asymmetric RTN, G = 128): closed-form examples, the RTN error bound and
the per-(row, 128-column group) axis."""
import numpy as np


def _s(orc, bits):
    return orc.f16_to_f64(int(bits))


def test_exact_grid_group(orc):
    # one row, one group whose min/max give range = 255 * 2^-10 exactly, so the
    # scale is 2^-10, the zero point is 128 and every code is known by hand
    u = 2.0 ** -10
    w = np.array([(2 * j - 128) * u for j in range(127)] + [127 * u], np.float32)[None, :]
    q, s, z = orc.rtn_quantize(w)
    assert _s(orc, s[0, 0]) == u
    assert _s(orc, z[0, 0]) == 128.0
    assert list(q[0, :127]) == [2 * j for j in range(127)]
    assert q[0, 127] == 255


def test_ties_round_to_even(orc):
    u = 2.0 ** -10
    base = [-128 * u, 127 * u]                    # fixes s = 2^-10, z = 128
    w = np.array(base + [2.5 * u, 3.5 * u, -2.5 * u, -3.5 * u], np.float32)[None, :]
    q, s, z = orc.rtn_quantize(w)
    assert list(q[0, 2:]) == [128 + 2, 128 + 4, 128 - 2, 128 - 4]


def test_error_bound_and_range(orc):
    g = np.random.default_rng(3)
    W = (g.standard_normal((37, 300)) * 0.02).astype(np.float32)
    q, s, z = orc.rtn_quantize(W)
    K, N = W.shape
    ng = (N + 127) // 128
    assert s.shape == (K, ng)
    for k in range(K):
        for gi in range(ng):
            cols = slice(128 * gi, min(N, 128 * gi + 128))
            sc = _s(orc, s[k, gi]); zp = _s(orc, z[k, gi])
            wg = W[k, cols].astype(np.float64)
            # scale: fp16 of range/255 within half an fp16 ulp (relative 2^-11)
            r = (wg.max() - wg.min()) / 255.0
            assert abs(sc - r) <= r * 2.0 ** -11
            assert zp == int(zp) and 0 <= zp <= 255
            rec = sc * (q[k, cols].astype(np.float64) - zp)
            inside = (q[k, cols] > 0) & (q[k, cols] < 255)
            assert np.all(np.abs(rec - wg)[inside] <= sc / 2 * (1 + 1e-12))
            # the group min and max map to codes near the ends of the range
            assert q[k, cols].min() <= 1 and q[k, cols].max() >= 254


def test_group_axis_is_columns_of_one_row(orc):
    # a large value in row 0, columns 128.. must only change row 0's second group
    W = np.full((3, 200), 0.01, np.float32)
    W[:, ::2] = -0.01
    W0 = W.copy()
    W[0, 150] = 5.0
    q0, s0, z0 = orc.rtn_quantize(W0)
    q1, s1, z1 = orc.rtn_quantize(W)
    assert s1[0, 1] != s0[0, 1]
    assert s1[0, 0] == s0[0, 0] and np.array_equal(s1[1:], s0[1:])
    assert np.array_equal(q1[0, :128], q0[0, :128]) and np.array_equal(q1[1:], q0[1:])


def test_constant_and_positive_groups(orc):
    W = np.zeros((2, 128), np.float32)
    W[0, :] = 0.25
    W[1, :] = np.linspace(0.5, 1.0, 128, dtype=np.float32)
    q, s, z = orc.rtn_quantize(W)
    assert s[0, 0] == 0x3C00                       # constant group: scale 1
    assert _s(orc, z[0, 0]) == 0.0                 # -0.25 rounds to 0 after clamp
    assert np.all(q[0] == 0)                       # rne(0.25 / 1) + 0 = 0
    assert _s(orc, z[1, 0]) == 0.0                 # all positive: zero clamps to 0
    assert q[1].max() == 255                       # w / s exceeds 255 and clamps
