"""The library's offline table construction (grinqh_lut_build, host code, no GPU)
against the oracle's ("GRINQH" Section 3.3 and Appendix E.2: nested k-means codes by
incremental upscaling): identical codes and binary16 tables on weights of the pages'
shapes and distributions, binary16 rounding checked against numpy on constant rows
(subnormals, ties, overflow), and the host-side argument checks."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import build
    build.build()
    from activation_graded_bit_b200 import grinqh
    return grinqh


@pytest.mark.parametrize("bmax", (2, 4, 6, 8))
@pytest.mark.parametrize("K,N,kind", [(7, 1000, "gauss"), (5, 4096, "rowstd"), (9, 130, "gauss"), (3, 1, "gauss"),
                                      (4, 37, "ties")])
def test_matches_the_oracle(g, orc, bmax, K, N, kind):
    if kind == "gauss":
        W = wl.weights_gaussian(K, N, key=(501, bmax, K, N))
    elif kind == "rowstd":
        W = wl.weights_rowstd_loguniform(K, N, key=(502, bmax))
    else:   # few distinct values, many ties
        W = wl.rng(503, bmax).integers(-3, 4, (K, N)).astype(np.float32) * np.float32(0.125)
    codes, lut = g.lut_build(W, bmax)
    q, lut_ref, _ = orc.lut_build(W, bmax)
    assert np.array_equal(codes.numpy(), q)
    assert np.array_equal(lut.numpy().view(np.uint16), lut_ref)


def test_binary16_rounding_of_constant_rows(g):
    vals = [0.0, -0.0, 1.0, -2.5, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -14, 2 ** -15 + 2 ** -25, 2 ** -24,
            2 ** -25, 3 * 2 ** -26, 1e-7, 65504.0, 65519.0, 65520.0, -70000.0, 0.1, 1.0 / 3.0]
    vals += list(wl.rng(504).standard_normal(200) * np.exp(wl.rng(505).uniform(-20, 12, 200)))
    W = np.repeat(np.array(vals, np.float32)[:, None], 3, axis=1)
    codes, lut = g.lut_build(W, 2)
    with np.errstate(over="ignore"):
        ref = np.array(vals, np.float32).astype(np.float16).view(np.uint16)
    ref[1] = 0x0000   # the mean of negative zeros is +0: the sums start from +0 (as in the oracle)
    got = lut.numpy().view(np.uint16)
    assert np.all(codes.numpy() == 0)
    for i in range(1, 8):   # every entry of every width is the constant
        assert np.array_equal(got[:, i], ref), i


def test_rejects_bad_arguments(g):
    W = np.zeros((2, 4), np.float32)
    for bm in (0, 3, 5, 9):
        with pytest.raises(g.GrinqhError):
            g.lut_build(W, bm)
    W[1, 2] = np.nan
    with pytest.raises(g.GrinqhError):
        g.lut_build(W, 4)
    W[1, 2] = np.inf
    with pytest.raises(g.GrinqhError):
        g.lut_build(W, 4)
    with pytest.raises(g.GrinqhError):
        g.lut_build(np.zeros((0, 4), np.float32), 4)


def test_accepts_a_cpu_tensor(g, orc):
    W = wl.weights_gaussian(3, 200, key=(506,))
    c1, l1 = g.lut_build(torch.from_numpy(W), 8)
    c2, l2 = g.lut_build(W, 8)
    assert torch.equal(c1, c2) and torch.equal(l1, l2)
