"""Pins for the oracle's nested look-up-table codes ("GRINQH" Section 3.3: nested
non-uniform codes such as k-means codes, no midpoint term because the nested levels
are centred; Section 4 and Appendix E.2: any-precision LLM weights at b_max = 8).

Product: a table that holds the uniform codes' bin midpoints gives exactly the
uniform graded product; one-hot rows read the heap entry 2^b + (q >> (b_max - b));
the low b_max - b bits and the rows of width 0 are never read.
Construction: every split is the best 2-partition of its cluster's members
(exhaustive search over all subsets on small rows), centroids are the members'
means (numpy), children average to their parent, codes follow the weights' order,
the squared error does not grow with the width, and the tables are the binary16
roundings of the centroids."""
import itertools

import numpy as np
import pytest

from activation_graded_bit_b200 import workloads as wl


def _rand_bits(rng, K, bmax, p0=0.2):
    bits = rng.integers(1, bmax + 1, K).astype(np.uint8)
    bits[rng.random(K) < p0] = 0
    return bits


@pytest.mark.parametrize("bmax", (2, 4, 6, 8))
def test_table_of_uniform_levels_gives_the_uniform_product(orc, bmax):
    # one 128-column group per row, scale 2^-7 and an integer zero point: every
    # uniform reconstruction s (code - z) is an integer times 2^-7 (exact in
    # binary16), so a table holding them must reproduce orc.vmm bit for bit
    rng = np.random.default_rng(bmax)
    K, N = 40, 100
    q = rng.integers(0, 1 << bmax, (K, N)).astype(np.uint8)
    zi = rng.integers(0, 1 << bmax, K)
    scale = np.full((K, 1), np.float16(2.0 ** -7)).view(np.uint16)
    zero = zi.astype(np.float16).reshape(K, 1).view(np.uint16)
    E = 1 << (bmax + 1)
    lut = np.zeros((K, E), np.float16)
    for k in range(K):
        for b in range(1, bmax + 1):
            w = 2.0 ** (bmax - b)                     # bin width of width b in b_max-bit units
            for c in range(1 << b):
                code = c * w + (w / 2.0 if b < bmax else 0.0)
                lut[k, (1 << b) + c] = np.float16((code - zi[k]) * 2.0 ** -7)
    x = wl.activations_outlier(K, 1, key=(301, bmax))[0]
    bits = _rand_bits(rng, K, bmax)
    y_lut, b_lut = orc.vmm_lut(x, q, lut.view(np.uint16), bits, bmax)
    y_uni, b_uni = orc.vmm(x, q, scale, zero, bits, bmax=bmax)
    assert np.array_equal(y_lut, y_uni)
    assert np.array_equal(b_lut, b_uni)


@pytest.mark.parametrize("bmax", (4, 8))
def test_one_hot_rows_read_the_heap_entry(orc, bmax):
    rng = np.random.default_rng(10 + bmax)
    K, N = 12, 70
    q = rng.integers(0, 1 << bmax, (K, N)).astype(np.uint8)
    lut = rng.standard_normal((K, 1 << (bmax + 1))).astype(np.float16)
    for k in (0, 5, 11):
        for b in range(1, bmax + 1):
            x = np.zeros(K, np.float16)
            x[k] = 1.0
            bits = np.zeros(K, np.uint8)
            bits[k] = b
            y, _ = orc.vmm_lut(x.view(np.uint16), q, lut.view(np.uint16), bits, bmax)
            heap = (1 << b) + q[k].astype(np.int64) // (1 << (bmax - b))
            assert np.array_equal(y, lut[k, heap].astype(np.float64)), (k, b)


def test_low_bits_and_skipped_rows_are_never_read(orc):
    bmax = 8
    rng = np.random.default_rng(3)
    K, N = 30, 90
    q = rng.integers(0, 256, (K, N)).astype(np.uint8)
    lut = rng.standard_normal((K, 512)).astype(np.float16).view(np.uint16)
    x = wl.activations_student_t(K, 1, key=(302,))[0]
    bits = _rand_bits(rng, K, bmax, p0=0.3)
    y0, _ = orc.vmm_lut(x, q, lut, bits, bmax)
    q2 = q.copy()
    lut2 = lut.copy()
    for k in range(K):
        b = int(bits[k])
        low = (1 << (bmax - b)) - 1 if b else 0xFF
        q2[k] = (q[k] & ~np.uint8(low)) | (rng.integers(0, 256, N).astype(np.uint8) & np.uint8(low))
        if b == 0:
            lut2[k] = rng.integers(0, 0x7C00, 512).astype(np.uint16)
        else:
            keep = np.zeros(512, bool)
            keep[1 << b:2 << b] = True                 # only width b's entries matter
            lut2[k, ~keep] = rng.integers(0, 0x7C00, int((~keep).sum())).astype(np.uint16)
    y1, _ = orc.vmm_lut(x, q2, lut2, bits, bmax)
    assert np.array_equal(y0, y1)


def test_width_above_bmax_is_rejected(orc):
    q = np.zeros((2, 4), np.uint8)
    lut = np.zeros((2, 32), np.uint16)
    with pytest.raises(ValueError):
        orc.vmm_lut(np.zeros(2, np.uint16), q, lut, np.array([1, 5], np.uint8), 4)


def _clusters(q, bmax, b):
    return q.astype(np.int64) >> (bmax - b)


def _sse(v):
    return float(((v - v.mean()) ** 2).sum()) if len(v) else 0.0


@pytest.mark.parametrize("seed", range(6))
def test_every_split_is_the_best_two_partition(orc, seed):
    # exhaustive search over every subset of a cluster's members
    rng = np.random.default_rng(seed)
    N, bmax = 9, 3
    w = rng.standard_normal(N).astype(np.float32)
    if seed % 2:
        w[3] = w[5]                                    # a tie
    q, _, _ = orc.lut_build(w[None, :], bmax)
    w64 = w.astype(np.float64)
    for b in range(1, bmax + 1):
        parent = _clusters(q[0], bmax, b - 1)
        child = _clusters(q[0], bmax, b)
        for p in np.unique(parent):
            members = np.nonzero(parent == p)[0]
            v = w64[members]
            got = _sse(v[child[members] == 2 * p]) + _sse(v[child[members] == 2 * p + 1])
            best = _sse(v)
            for r in range(1, len(v)):
                for sub in itertools.combinations(range(len(v)), r):
                    mask = np.zeros(len(v), bool)
                    mask[list(sub)] = True
                    best = min(best, _sse(v[mask]) + _sse(v[~mask]))
            assert got <= best * (1 + 1e-12) + 1e-15, (b, p, got, best)


@pytest.mark.parametrize("bmax", (2, 5, 8))
def test_centroids_are_member_means_and_nest(orc, bmax):
    W = wl.weights_rowstd_loguniform(6, 700, key=(303, bmax))
    q, lut, cent = orc.lut_build(W, bmax)
    for k in range(W.shape[0]):
        w = W[k].astype(np.float64)
        assert cent[k, 1] == pytest.approx(w.mean(), rel=1e-13, abs=1e-15)
        for b in range(1, bmax + 1):
            cl = _clusters(q[k], bmax, b)
            for c in range(1 << b):
                m = cl == c
                if m.any():
                    assert cent[k, (1 << b) + c] == pytest.approx(w[m].mean(), rel=1e-12, abs=1e-15)
                else:                                  # an empty child keeps its parent's value
                    assert cent[k, (1 << b) + c] == cent[k, (1 << (b - 1)) + c // 2]
                if b > 1 and c % 2 == 0:
                    n0, n1 = int((cl == c).sum()), int((cl == c + 1).sum())
                    if n0 + n1:
                        avg = (n0 * cent[k, (1 << b) + c] + n1 * cent[k, (1 << b) + c + 1]) / (n0 + n1)
                        assert avg == pytest.approx(cent[k, (1 << (b - 1)) + c // 2], rel=1e-12, abs=1e-15)
    # the tables are the binary16 roundings (nearest even) of the centroids
    ref = cent.astype(np.float16).view(np.uint16)
    ref[:, 0] = 0
    assert np.array_equal(lut, ref)


def test_codes_follow_the_weights_order(orc):
    rng = np.random.default_rng(7)
    W = rng.standard_normal((3, 500)).astype(np.float32)
    W[:, 100:110] = W[:, 0:1]                          # ties
    q, _, _ = orc.lut_build(W, 8)
    for k in range(3):
        o = np.argsort(W[k], kind="stable")
        assert np.all(np.diff(q[k][o].astype(np.int64)) >= 0)
        assert len(set(q[k, 100:110].tolist() + [int(q[k, 0])])) == 1


def test_squared_error_does_not_grow_with_width(orc):
    W = wl.weights_gaussian(5, 1000, key=(304,))
    bmax = 8
    q, _, cent = orc.lut_build(W, bmax)
    for k in range(5):
        prev = np.inf
        for b in range(0, bmax + 1):
            idx = (1 << b) + _clusters(q[k], bmax, b)
            e = float(((W[k].astype(np.float64) - cent[k, idx]) ** 2).sum())
            assert e <= prev * (1 + 1e-12)
            prev = e


def test_constant_row_and_exact_reconstruction(orc):
    bmax = 4
    # a constant row: one code, every centroid the constant
    W = np.full((1, 50), 0.375, np.float32)
    q, lut, cent = orc.lut_build(W, bmax)
    assert np.all(q == 0) and np.all(cent[0, 1:] == 0.375)
    # m <= b_max + 1 distinct values: each split separates a cluster with two or
    # more distinct values, so by width b_max every value has its own code
    rng = np.random.default_rng(9)
    vals = np.array([-1.5, 0.25, 0.5, 3.0, 7.0], np.float32)
    W = vals[rng.integers(0, 5, 300)][None, :]
    q, _, cent = orc.lut_build(W, bmax)
    rec = cent[0, (1 << bmax) + q[0].astype(np.int64)]
    assert np.array_equal(rec, W[0].astype(np.float64))
