"""Pins for the oracle's graded product ("GRINQH" Section 3 and Fig. 2): full
width equals the dense dequantised GEMV, skipped rows contribute nothing, and a
4x4 brute force over all 9^4 width assignments against the bin-midpoint form."""
import itertools
import math

import numpy as np

from activation_graded_bit_b200 import workloads as wl


def _dense_dequant(orc, q, s, z):
    K, N = q.shape
    sf = s.view(np.float16).astype(np.float64)
    zf = z.view(np.float16).astype(np.float64)
    S = np.repeat(sf, 128, axis=1)[:, :N]
    Z = np.repeat(zf, 128, axis=1)[:, :N]
    return S * (q.astype(np.float64) - Z)


def _midpoint_codes(q, b):
    # centre of the 2^(8-b)-wide bin that holds q, written with real division
    out = np.empty(q.shape, np.float64)
    for k in range(q.shape[0]):
        if b[k] == 8:
            out[k] = q[k]
        elif b[k] > 0:
            w = 2.0 ** (8 - int(b[k]))
            out[k] = np.floor(q[k] / w) * w + w / 2.0
        else:
            out[k] = np.nan
    return out


def test_full_width_equals_dense_gemv(orc):
    W = wl.weights_gaussian(300, 260, key=(7, 1))
    x = wl.activations_outlier(300, 1, key=(7, 2))[0]
    q, s, z = orc.rtn_quantize(W)
    y, bound = orc.vmm(x, q, s, z, np.full(300, 8, np.uint8))
    ref = x.view(np.float16).astype(np.float64) @ _dense_dequant(orc, q, s, z)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert np.all(bound >= np.abs(y))


def test_skipped_rows_contribute_nothing(orc):
    K, N = 64, 140
    W = wl.weights_gaussian(K, N, key=(7, 3))
    q, s, z = orc.rtn_quantize(W)
    x = wl.activations_gaussian(K, 1, key=(7, 4))[0]
    g = np.random.default_rng(1)
    bits = g.choice(np.array([0, 2, 3, 4, 8], np.uint8), K)
    y, _ = orc.vmm(x, q, s, z, bits)
    keep = bits > 0
    y2, _ = orc.vmm(x[keep], q[keep], s[keep], z[keep], bits[keep])
    assert np.array_equal(y, y2)
    x3 = x.copy()
    x3[~keep] = np.float16(1000.0).view(np.uint16)
    y3, _ = orc.vmm(x3, q, s, z, bits)
    assert np.array_equal(y, y3)


def test_brute_force_4x4_all_width_assignments(orc):
    W = wl.weights_gaussian(4, 4, key=(7, 5), std=0.5)
    q, s, z = orc.rtn_quantize(W)
    x = wl.activations_gaussian(4, 1, key=(7, 6))[0]
    xf = x.view(np.float16).astype(np.float64)
    sf = s.view(np.float16).astype(np.float64)[:, 0]
    zf = z.view(np.float16).astype(np.float64)[:, 0]
    for b in itertools.product(range(9), repeat=4):
        b = np.array(b, np.uint8)
        y, _ = orc.vmm(x, q, s, z, b)
        codes = _midpoint_codes(q, b)
        ref = np.zeros(4)
        for k in range(4):
            if b[k]:
                ref += xf[k] * sf[k] * (codes[k] - zf[k])
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-15), b


def test_group_scale_applies_to_its_columns(orc):
    # dense check on a shape with a ragged last group and K != N
    W = wl.weights_rowstd_loguniform(33, 333, key=(7, 7))
    x = wl.activations_student_t(33, 1, key=(7, 8))[0]
    q, s, z = orc.rtn_quantize(W)
    bits = np.random.default_rng(2).choice(np.array([0, 2, 3, 4, 8], np.uint8), 33)
    y, _ = orc.vmm(x, q, s, z, bits)
    codes = _midpoint_codes(q, bits)
    sf = np.repeat(s.view(np.float16).astype(np.float64), 128, 1)[:, :333]
    zf = np.repeat(z.view(np.float16).astype(np.float64), 128, 1)[:, :333]
    Wh = np.where((bits > 0)[:, None], sf * (codes - zf), 0.0)
    ref = x.view(np.float16).astype(np.float64) @ Wh
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_threads_do_not_change_result(orc):
    W = wl.weights_gaussian(200, 1000, key=(7, 9))
    x = wl.activations_outlier(200, 1, key=(7, 10))[0]
    q, s, z = orc.rtn_quantize(W)
    bits = np.random.default_rng(3).choice(np.array([0, 2, 3, 4, 8], np.uint8), 200)
    y1, b1 = orc.vmm(x, q, s, z, bits, nthreads=1)
    y4, b4 = orc.vmm(x, q, s, z, bits, nthreads=4)
    assert np.array_equal(y1, y4) and np.array_equal(b1, b4)
