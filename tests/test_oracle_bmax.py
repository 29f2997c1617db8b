"""Pins for the oracle at b_max < 8 ("GRINQH" Section 3.3: each weight is quantised
to a b_max-bit integer, b_max in {4, 6, 8} is evaluated, and a width b <= b_max reads
the top b bits, scaled back by 2^(b_max - b), plus the midpoint 2^(b_max - b - 1)).

The b_max-bit RTN is pinned by hand-built grids, ties and the RTN error bound; the
nested code exhaustively against the bin-midpoint definition; the graded product by
the dense dequantised GEMV at full width, removal of skipped rows and a 4x4 brute
force over every width assignment."""
import itertools
import math

import numpy as np
import pytest

from activation_graded_bit_b200 import workloads as wl

BMAX = (2, 4, 6)


def _s(orc, bits):
    return orc.f16_to_f64(int(bits))


@pytest.mark.parametrize("bmax", BMAX)
def test_exact_grid_group(orc, bmax):
    # range = L * 2^-10 with L = 2^b_max - 1 levels: scale 2^-10, zero point
    # 2^(b_max-1), and the codes of grid points are known by hand
    L = 2 ** bmax - 1
    half = 2 ** (bmax - 1)
    u = 2.0 ** -10
    levels = list(range(-half, half))             # w = j * u for j in [-half, half)
    w = np.array([j * u for j in levels], np.float32)[None, :]
    q, s, z = orc.rtn_quantize(w, bmax)
    assert _s(orc, s[0, 0]) == u
    assert _s(orc, z[0, 0]) == float(half)
    assert list(q[0]) == [j + half for j in levels]
    assert int(q.max()) == L


@pytest.mark.parametrize("bmax", (4, 6))
def test_ties_round_to_even(orc, bmax):
    half = 2 ** (bmax - 1)
    u = 2.0 ** -10
    base = [-half * u, (half - 1) * u]            # fixes s = 2^-10, z = half
    w = np.array(base + [1.5 * u, 2.5 * u, -1.5 * u, -2.5 * u], np.float32)[None, :]
    q, s, z = orc.rtn_quantize(w, bmax)
    assert list(q[0, 2:]) == [half + 2, half + 2, half - 2, half - 2]


@pytest.mark.parametrize("bmax", BMAX)
def test_error_bound_and_range(orc, bmax):
    L = 2 ** bmax - 1
    W = (np.random.default_rng(bmax).standard_normal((21, 300)) * 0.02).astype(np.float32)
    q, s, z = orc.rtn_quantize(W, bmax)
    K, N = W.shape
    for k in range(K):
        for gi in range((N + 127) // 128):
            cols = slice(128 * gi, min(N, 128 * gi + 128))
            sc = _s(orc, s[k, gi]); zp = _s(orc, z[k, gi])
            wg = W[k, cols].astype(np.float64)
            r = (wg.max() - wg.min()) / L
            assert abs(sc - r) <= r * 2.0 ** -11
            assert zp == int(zp) and 0 <= zp <= L
            assert int(q[k, cols].max()) <= L
            rec = sc * (q[k, cols].astype(np.float64) - zp)
            inside = (q[k, cols] > 0) & (q[k, cols] < L)
            assert np.all(np.abs(rec - wg)[inside] <= sc / 2 * (1 + 1e-12))


@pytest.mark.parametrize("bmax", BMAX)
def test_code_is_bin_midpoint(orc, bmax):
    for b in range(1, bmax):
        width = 2 ** (bmax - b)
        for q in range(2 ** bmax):
            lo = math.floor(q / width) * width
            assert orc.code(q, b, bmax) == lo + width / 2.0, (q, b)
    for q in range(2 ** bmax):
        assert orc.code(q, bmax, bmax) == q
        assert orc.code(q, 0, bmax) == -1


@pytest.mark.parametrize("bmax", BMAX)
def test_nesting_bound_and_mean(orc, bmax):
    n = 2 ** bmax
    prev = None
    for b in range(1, bmax + 1):
        err = [abs(orc.code(q, b, bmax) - q) for q in range(n)]
        assert max(err) == (0 if b == bmax else 2 ** (bmax - 1 - b))
        mean = sum(err) / float(n)
        assert mean == (0 if b == bmax else 2 ** (bmax - b) / 4.0)
        if prev is not None:
            assert max(err) <= prev[0] and mean <= prev[1]
        prev = (max(err), mean)


def _dense(q, s, z):
    N = q.shape[1]
    S = np.repeat(s.view(np.float16).astype(np.float64), 128, axis=1)[:, :N]
    Z = np.repeat(z.view(np.float16).astype(np.float64), 128, axis=1)[:, :N]
    return S * (q.astype(np.float64) - Z)


@pytest.mark.parametrize("bmax", (4, 6))
def test_full_width_equals_dense_gemv(orc, bmax):
    W = wl.weights_gaussian(200, 300, key=(71, bmax))
    x = wl.activations_outlier(200, 1, key=(72, bmax))[0]
    q, s, z = orc.rtn_quantize(W, bmax)
    y, bound = orc.vmm(x, q, s, z, np.full(200, bmax, np.uint8), bmax=bmax)
    ref = x.view(np.float16).astype(np.float64) @ _dense(q, s, z)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.all(bound >= np.abs(y))


@pytest.mark.parametrize("bmax", (4, 6))
def test_skipped_rows_contribute_nothing(orc, bmax):
    K, N = 64, 140
    W = wl.weights_gaussian(K, N, key=(73, bmax))
    q, s, z = orc.rtn_quantize(W, bmax)
    x = wl.activations_gaussian(K, 1, key=(74, bmax))[0]
    bits = np.random.default_rng(bmax).choice(np.arange(0, bmax + 1, 2, dtype=np.uint8), K)
    y, _ = orc.vmm(x, q, s, z, bits, bmax=bmax)
    keep = bits > 0
    y2, _ = orc.vmm(x[keep], q[keep], s[keep], z[keep], bits[keep], bmax=bmax)
    assert np.array_equal(y, y2)


@pytest.mark.parametrize("bmax", (4, 6))
def test_brute_force_4x4_all_width_assignments(orc, bmax):
    W = wl.weights_gaussian(4, 4, key=(75, bmax), std=0.5)
    q, s, z = orc.rtn_quantize(W, bmax)
    x = wl.activations_gaussian(4, 1, key=(76, bmax))[0]
    xf = x.view(np.float16).astype(np.float64)
    sf = s.view(np.float16).astype(np.float64)[:, 0]
    zf = z.view(np.float16).astype(np.float64)[:, 0]
    for b in itertools.product(range(bmax + 1), repeat=4):
        b = np.array(b, np.uint8)
        y, _ = orc.vmm(x, q, s, z, b, bmax=bmax)
        ref = np.zeros(4)
        for k in range(4):
            if b[k] == bmax:
                code = q[k].astype(np.float64)
            elif b[k] > 0:
                wdt = 2.0 ** (bmax - int(b[k]))
                code = np.floor(q[k] / wdt) * wdt + wdt / 2.0
            else:
                continue
            ref += xf[k] * sf[k] * (code - zf[k])
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-15), b
