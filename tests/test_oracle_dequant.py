"""Pins for the oracle's full-width dequantisation and dense prefill product
("GRINQH" Section 4, prefill unpacks the weights at b_max and runs a dense
matrix-matrix product; Section 3.3, w_hat = s (q - z)): hand-built values,
round-to-nearest-even ties of binary16, the half-ulp bound against the exact
product, and the dense product against a per-element loop on a small case."""
import numpy as np
import pytest

from activation_graded_bit_b200 import workloads as wl


def _f16(v):
    return int(np.array([v], np.float16).view(np.uint16)[0])


def test_hand_built_values(orc):
    # s = 2^-10, z = 128: w_hat = (q - 128) 2^-10, exact in binary16
    q = np.array([[0, 1, 127, 128, 129, 255]], np.uint8)
    s = np.array([[_f16(2.0 ** -10)]], np.uint16)
    z = np.array([[_f16(128.0)]], np.uint16)
    out = orc.dequant_f16(q, s, z).view(np.float16).astype(np.float64)[0]
    assert list(out) == [(v - 128) * 2.0 ** -10 for v in (0, 1, 127, 128, 129, 255)]
    assert orc.dequant_f16(np.array([[128]], np.uint8), s, z)[0, 0] == 0   # +0, not -0


def test_ties_round_to_even(orc):
    # s = 1 + 2^-10 (binary16 spacing 2^-10 at 1): s * 3 = 3 + 3*2^-10 needs
    # 12 bits; spacing at 3 is 2^-9, so 3*2^-10 = 1.5 ulp -> rounds to 2 ulp (even)
    s = np.array([[_f16(1.0 + 2.0 ** -10)]], np.uint16)
    z = np.array([[0]], np.uint16)
    out = orc.dequant_f16(np.array([[3, 5]], np.uint8), s, z).view(np.float16).astype(np.float64)[0]
    assert out[0] == 3.0 + 2 * 2.0 ** -9
    # s * 5 = 5 + 5*2^-10; spacing at 5 is 2^-8: 5*2^-10 = 1.25 ulp -> 1 ulp
    assert out[1] == 5.0 + 2.0 ** -8


def test_half_ulp_bound_against_exact_product(orc):
    W = wl.weights_rowstd_loguniform(40, 300, key=(61, 1))
    for bmax in (8, 6, 4):
        q, s, z = orc.rtn_quantize(W, bmax)
        w16 = orc.dequant_f16(q, s, z).view(np.float16).astype(np.float64)
        S = np.repeat(s.view(np.float16).astype(np.float64), 128, axis=1)[:, :300]
        Z = np.repeat(z.view(np.float16).astype(np.float64), 128, axis=1)[:, :300]
        exact = S * (q.astype(np.float64) - Z)
        # binary16 round to nearest: relative error at most 2^-11 in the normal range
        normal = np.abs(exact) >= 2.0 ** -14
        assert np.all(np.abs(w16 - exact)[normal] <= np.abs(exact)[normal] * 2.0 ** -11)
        assert np.all(np.abs(w16 - exact)[~normal] <= 2.0 ** -25)


def test_prefill_product_small_case(orc):
    X = wl.activations_outlier(9, 3, key=(62, 1), chan_key=(62,))
    W = wl.weights_gaussian(9, 5, key=(62, 2))
    q, s, z = orc.rtn_quantize(W)
    w16 = orc.dequant_f16(q, s, z)
    Y, bound = orc.prefill(X, w16)
    xf = X.view(np.float16).astype(np.float64)
    wf = w16.view(np.float16).astype(np.float64)
    for t in range(3):
        for n in range(5):
            acc = 0.0
            b = 0.0
            for k in range(9):
                acc += xf[t, k] * wf[k, n]
                b += abs(xf[t, k] * wf[k, n])
            assert Y[t, n] == pytest.approx(acc, rel=1e-13, abs=1e-15)
            assert bound[t, n] == pytest.approx(b, rel=1e-13)
