"""GPU packing of given codes and the graded product over nested look-up-table codes
against the fp64 oracle ("GRINQH" Section 3.3: nested non-uniform codes, no midpoint
term; Section 4 and Appendix E.2: any-precision LLM weights).

Bit-exact: the planes of given codes (read back at full width) and zero scale/zero
words; one-hot rows; all-skipped rows give y = 0.
Within |y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6: every width on ragged
shapes for b_max in {2, 4, 6, 8}, tables from the oracle's nested 2-means
construction, uniform RTN codes read as table indices, a full-size q_proj, and a
tall layer whose CTAs stage their rows in several passes."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, assert_close, dev_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _sel(g, bits, classes):
    import oracle
    idx, off = oracle.compact(bits, np.array(classes, np.uint8))
    return g.Selection(torch.from_numpy(bits).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(off).cuda(),
                       tuple(classes))


def _run(g, p, lut, x, sel, N):
    y = Guarded(N, torch.float32)
    ws = g.vmm_workspace(p.layout)
    g.vmm_lut(p, dev_u16(lut), dev_u16(x), sel, ws, y=y.t)
    torch.cuda.synchronize()
    y.check()
    assert int(ws[:16].count_nonzero()) == 0
    return y.t.cpu().numpy()


@pytest.mark.parametrize("bmax", (2, 4, 6, 8))
@pytest.mark.parametrize("K,N", [(1024, 1024), (37, 300), (130, 1029), (3, 2049)])
def test_pack_codes_round_trip(g, bmax, K, N):
    rng = np.random.default_rng(K * 7 + N + bmax)
    codes = rng.integers(0, 256, (K, N)).astype(np.uint8)      # bits above b_max set too
    p = g.pack_codes(torch.from_numpy(codes).cuda(), b_max=bmax)
    assert p.layout.b_max == bmax
    full = torch.full((K,), bmax, dtype=torch.uint8, device="cuda")
    back = g.unpack_codes(p, full).cpu().numpy()
    assert np.array_equal(back, codes & np.uint8((1 << bmax) - 1))
    assert int(p.meta_words().count_nonzero()) == 0


@pytest.mark.parametrize("bmax", (2, 4, 6, 8))
@pytest.mark.parametrize("K,N", [(333, 1100), (1024, 2048)])
def test_every_width_against_the_oracle(g, orc, bmax, K, N):
    W = wl.weights_rowstd_loguniform(K, N, key=(401, bmax, K))
    q, lut, _ = orc.lut_build(W, bmax)
    p = g.pack_codes(torch.from_numpy(q).cuda(), b_max=bmax)
    cl = tuple(range(bmax + 1))
    rng = np.random.default_rng(bmax * 1000 + K)
    for trial in range(3):
        x = wl.activations_student_t(K, 1, key=(402, bmax, K, trial))[0]
        bits = rng.integers(0, bmax + 1, K).astype(np.uint8)
        y = _run(g, p, lut, x, _sel(g, bits, cl), N)
        yr, bound = orc.vmm_lut(x, q, lut, bits, bmax)
        assert_close(y, yr, bound, "vmm_lut b_max=%d" % bmax)


def test_uniform_codes_read_as_table_indices(g, orc):
    # grinqh_pack's records: the b_max-bit RTN codes index the tables; the
    # records' scale/zero words are not read
    K, N, bmax = 500, 1500, 8
    W = wl.weights_gaussian(K, N, key=(403,))
    p = g.pack(torch.from_numpy(W).cuda())
    q, _, _ = orc.rtn_quantize(W)
    lut = wl.rng(404).standard_normal((K, 512)).astype(np.float16).view(np.uint16)
    x = wl.activations_outlier(K, 1, key=(405,))[0]
    cl = (0, 2, 3, 4, 8)
    bits = np.array(cl, np.uint8)[wl.rng(406).integers(0, 5, K)]
    y = _run(g, p, lut, x, _sel(g, bits, cl), N)
    yr, bound = orc.vmm_lut(x, q, lut, bits, bmax)
    assert_close(y, yr, bound, "RTN codes as indices")


@pytest.mark.parametrize("bmax", (4, 8))
def test_one_hot_rows_are_exact(g, orc, bmax):
    K, N = 64, 1300
    rng = np.random.default_rng(407 + bmax)
    q = rng.integers(0, 1 << bmax, (K, N)).astype(np.uint8)
    lut = rng.standard_normal((K, 1 << (bmax + 1))).astype(np.float16).view(np.uint16)
    p = g.pack_codes(torch.from_numpy(q).cuda(), b_max=bmax)
    cl = tuple(range(bmax + 1))
    for k in rng.choice(K, 5, replace=False):
        for b in range(1, bmax + 1):
            x = np.zeros(K, np.float16)
            x[k] = 1.0
            bits = np.zeros(K, np.uint8)
            bits[k] = b
            y = _run(g, p, lut, x.view(np.uint16), _sel(g, bits, cl), N)
            yr, _ = orc.vmm_lut(x.view(np.uint16), q, lut, bits, bmax)
            assert np.array_equal(y.astype(np.float64), yr), (k, b)


def test_all_rows_skipped_give_zero(g):
    K, N, bmax = 300, 2100, 8
    q = np.random.default_rng(408).integers(0, 256, (K, N)).astype(np.uint8)
    lut = np.full((K, 512), 0x3C00, np.uint16)
    p = g.pack_codes(torch.from_numpy(q).cuda(), b_max=bmax)
    x = wl.activations_gaussian(K, 1, key=(409,))[0]
    y = _run(g, p, lut, x, _sel(g, np.zeros(K, np.uint8), (0, 2, 3, 4, 8)), N)
    assert np.all(y == 0.0)


def test_full_size_q_proj(g, orc):
    # Llama3-8B q_proj shape, nested tables at b_max = 8, classes {0,2,3,4,8}
    # graded to 3 average bits; columns sampled by whole groups, the last included
    K, N, bmax = 4096, 4096, 8
    cl = (0, 2, 3, 4, 8)
    W = wl.weights_gaussian(K, N, key=(410, 0))
    q, lut, _ = orc.lut_build(W, bmax)
    p = g.pack_codes(torch.from_numpy(q).cuda(), b_max=bmax)
    Xc = wl.activations_outlier(K, 128, key=(410, 1), chan_key=(410,))
    x = wl.activations_outlier(K, 1, key=(410, 2), chan_key=(410,))[0]
    P = orc.maxent_distribution(np.array(cl, np.uint8), 3.0)
    th = g.calibrate(dev_u16(Xc), cl, P=P)
    sel = g.select(dev_u16(x), th, cl)
    y = g.vmm_lut(p, dev_u16(lut), dev_u16(x), sel, g.vmm_workspace(p.layout)).cpu().numpy()
    bits = sel.bits.cpu().numpy()
    assert abs(bits.mean() - 3.0) < 0.5
    rng = np.random.default_rng(11)
    gs = sorted(set(list(rng.choice(N // 128, 3, replace=False)) + [N // 128 - 1]))
    cols = np.concatenate([np.arange(128 * c, 128 * c + 128) for c in gs])
    yr, bound = orc.vmm_lut(x, q[:, cols], lut, bits, bmax)
    assert_close(y[cols], yr, bound, "q_proj tables")


def test_tall_layer_multi_pass(g, orc):
    # K / R > 16384 rows per CTA with one column tile: several staging passes
    K, N, bmax = 1_400_000, 40, 4
    rng = np.random.default_rng(411)
    q = rng.integers(0, 16, (K, N)).astype(np.uint8)
    lut = rng.standard_normal((K, 32)).astype(np.float16).view(np.uint16)
    p = g.pack_codes(torch.from_numpy(q).cuda(), b_max=bmax)
    x = wl.activations_gaussian(K, 1, key=(412,))[0]
    cl = (0, 2, 3, 4)
    bits = np.array(cl[1:], np.uint8)[rng.integers(0, 3, K)]   # every row active: ~18,900 rows per CTA
    y = _run(g, p, lut, x, _sel(g, bits, cl), N)
    yr, bound = orc.vmm_lut(x, q, lut, bits, bmax, nthreads=8)
    assert_close(y, yr, bound, "tall tables")
