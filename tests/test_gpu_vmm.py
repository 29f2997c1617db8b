"""GPU graded VMM vs the fp64 oracle ("GRINQH" Fig. 2, Section 3.3):
|y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6 on every column checked."""
import itertools

import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, assert_close, dev_u16

pytestmark = pytest.mark.gpu

CL = (0, 2, 3, 4, 8)


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _selection_from_host(g, bits, classes, orc):
    idx, off = orc.compact(bits, np.array(classes, np.uint8))
    return g.Selection(torch.from_numpy(bits).cuda(), torch.from_numpy(idx).cuda(),
                       torch.from_numpy(off).cuda(), tuple(classes))


def _vmm_guarded(g, p, x_dev, sel, ws):
    y = Guarded(p.N, torch.float32)
    g.vmm(p, x_dev, sel, ws, y=y.t)
    torch.cuda.synchronize()
    y.check()
    assert int(ws[:16].count_nonzero()) == 0, "status word set"
    return y.t.cpu().numpy()


def test_config0_end_to_end(g, orc):
    K = N = 1024
    W = wl.weights_gaussian(K, N, key=(0, 0, 0, 0))
    Xc = wl.activations_outlier(K, 128, key=(0, 0, 0, 1), chan_key=(0, 0, 0))
    X = wl.activations_outlier(K, 16, key=(0, 0, 0, 2), chan_key=(0, 0, 0))
    p = g.pack(torch.from_numpy(W).cuda())
    th = g.calibrate(dev_u16(Xc), CL, P=orc.maxent_distribution(np.array(CL, np.uint8), 4.0))
    q, s, z = orc.rtn_quantize(W)
    th_ref = orc.thresholds(Xc, orc.maxent_distribution(np.array(CL, np.uint8), 4.0))
    assert np.array_equal(th.cpu().numpy(), th_ref)
    ws = g.vmm_workspace(p.layout)
    for v in X:
        xd = dev_u16(v)
        sel = g.select(xd, th, CL)
        y = _vmm_guarded(g, p, xd, sel, ws)
        bits, _, _ = orc.select(v, th_ref, np.array(CL, np.uint8))
        assert np.array_equal(sel.bits.cpu().numpy(), bits)
        yr, bound = orc.vmm(v, q, s, z, bits)
        assert_close(y, yr, bound, "config0")


def test_one_hot_rows_are_exact(g, orc):
    K, N = 64, 700
    W = wl.weights_rowstd_loguniform(K, N, key=(41, 1))
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    ws = g.vmm_workspace(p.layout)
    rng = np.random.default_rng(4)
    for k in rng.choice(K, 12, replace=False):
        for b in (1, 2, 3, 4, 5, 6, 7, 8):
            x = np.zeros(K, np.float16)
            x[k] = 1.0
            bits = np.zeros(K, np.uint8)
            bits[k] = b
            sel = _selection_from_host(g, bits, tuple(range(9)), orc)
            y = _vmm_guarded(g, p, dev_u16(x.view(np.uint16)), sel, ws)
            yr, _ = orc.vmm(x.view(np.uint16), q, s, z, bits)
            # s*(code - z) is exact in fp32, and so is every partial sum here
            assert np.array_equal(y.astype(np.float64), yr), (k, b)


def test_full_width_is_dense_gemv(g, orc):
    K, N = 300, 1500
    W = wl.weights_gaussian(K, N, key=(41, 2))
    x = wl.activations_outlier(K, 1, key=(41, 3))[0]
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    sel = g.select(dev_u16(x), None, (8,))
    y = _vmm_guarded(g, p, dev_u16(x), sel, g.vmm_workspace(p.layout))
    yr, bound = orc.vmm(x, q, s, z, np.full(K, 8, np.uint8))
    assert_close(y, yr, bound, "all 8-bit")


def test_skipped_rows_are_never_used(g, orc):
    # class-0 rows get NaN scales and random plane bytes: y must stay finite and
    # equal to the oracle on the untouched layer
    K, N = 512, 1024
    W = wl.weights_gaussian(K, N, key=(41, 4))
    x = wl.activations_outlier(K, 1, key=(41, 5))[0]
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    th = np.array([0.8, 1.2, 1.8, 2.5], np.float32)
    bits, _, _ = orc.select(x, th, np.array(CL, np.uint8))
    skip = np.nonzero(bits == 0)[0]
    assert skip.size > 50
    L = p.layout
    planes, meta = p.planes(), p.meta_bytes()
    sk = torch.from_numpy(skip).cuda()
    nan_words = torch.full((skip.size, L.n_tiles, 8), 0x7E007E00, dtype=torch.int32, device="cuda")
    meta[sk] = nan_words.view(torch.uint8).view(skip.size, L.n_tiles, 32)   # NaN scale and zero
    planes[sk] = torch.randint(0, 256, (skip.size, L.n_tiles, L.record_bytes), dtype=torch.uint8, device="cuda")
    sel = g.select(dev_u16(x), torch.from_numpy(th).cuda(), CL)
    y = _vmm_guarded(g, p, dev_u16(x), sel, g.vmm_workspace(L))
    assert np.all(np.isfinite(y))
    yr, bound = orc.vmm(x, q, s, z, bits)
    assert_close(y, yr, bound, "poisoned skipped rows")


def test_brute_force_4x4(g, orc):
    W = wl.weights_gaussian(4, 4, key=(41, 6), std=0.5)
    x = wl.activations_gaussian(4, 1, key=(41, 7))[0]
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    ws = g.vmm_workspace(p.layout)
    xd = dev_u16(x)
    classes = tuple(range(9))
    worst = 0.0
    for b in itertools.product(range(9), repeat=4):
        bits = np.array(b, np.uint8)
        sel = _selection_from_host(g, bits, classes, orc)
        y = g.vmm(p, xd, sel, ws).cpu().numpy()
        yr, bound = orc.vmm(x, q, s, z, bits)
        worst = max(worst, assert_close(y, yr, bound, str(b)))
    assert int(ws[:16].count_nonzero()) == 0, "status word set"


def test_brute_force_4x4_threshold_driven(g, orc):
    W = wl.weights_gaussian(4, 4, key=(41, 8), std=0.5)
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    ws = g.vmm_workspace(p.layout)
    th = np.array([0.25, 0.5, 1.0, 2.0], np.float32)
    thd = torch.from_numpy(th).cuda()
    mags = np.array([0.1, 0.3, 0.6, 1.5, 3.0], np.float16)
    for m in itertools.product(range(5), repeat=4):
        x = mags[list(m)] * np.array([1, -1, 1, -1], np.float16)
        xb = x.view(np.uint16)
        sel = g.select(dev_u16(xb), thd, CL)
        y = g.vmm(p, dev_u16(xb), sel, ws).cpu().numpy()
        bits, _, _ = orc.select(xb, th, np.array(CL, np.uint8))
        assert np.array_equal(sel.bits.cpu().numpy(), bits)
        yr, bound = orc.vmm(xb, q, s, z, bits)
        assert_close(y, yr, bound, str(m))


@pytest.mark.parametrize("K,N", [(1, 1), (1, 513), (37, 300), (1025, 1029), (5000, 64), (2, 4096), (4096, 130)])
def test_ragged_shapes(g, orc, K, N):
    W = wl.weights_rowstd_loguniform(K, N, key=(42, K, N))
    x = wl.activations_student_t(K, 1, key=(43, K, N))[0]
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    th = np.array([0.3, 0.7, 1.3, 2.4], np.float32)
    sel = g.select(dev_u16(x), torch.from_numpy(th).cuda(), CL)
    y = _vmm_guarded(g, p, dev_u16(x), sel, g.vmm_workspace(p.layout))
    bits, _, _ = orc.select(x, th, np.array(CL, np.uint8))
    yr, bound = orc.vmm(x, q, s, z, bits)
    assert_close(y, yr, bound, "%dx%d" % (K, N))


def test_all_rows_skipped(g, orc):
    K, N = 100, 700
    W = wl.weights_gaussian(K, N, key=(44, 1))
    p = g.pack(torch.from_numpy(W).cuda())
    x = np.zeros(K, np.float16).view(np.uint16)
    sel = g.select(dev_u16(x), torch.tensor([0.5, 1, 2, 3], dtype=torch.float32, device="cuda"), CL)
    y = _vmm_guarded(g, p, dev_u16(x), sel, g.vmm_workspace(p.layout))
    assert np.all(y == 0.0)


def _sampled_columns(N, rng, groups=3):
    ng = (N + 127) // 128
    gs = sorted(set(list(rng.choice(ng, groups, replace=False)) + [ng - 1]))
    cols = np.concatenate([np.arange(128 * q, min(N, 128 * q + 128)) for q in gs])
    return cols


FULL = [("llama3", wl.LLAMA3_8B, (4.0, 3.0, 2.0)), ("qwen3", wl.QWEN3_8B, (4.0, 3.0))]


@pytest.mark.parametrize("family,shapes,targets", FULL)
def test_full_size_layers_sampled_columns(g, orc, family, shapes, targets):
    rng = np.random.default_rng(5)
    for li, (name, K, N) in enumerate(shapes):
        key = (1 if family == "llama3" else 2, 0, li)
        if family == "llama3":
            W = wl.weights_gaussian(K, N, key=key + (0,))
            Xc = wl.activations_outlier(K, 128, key=key + (1,), chan_key=key)
            X = wl.activations_outlier(K, 2, key=key + (2,), chan_key=key)
        else:
            W = wl.weights_rowstd_loguniform(K, N, key=key + (0,))
            Xc = wl.activations_student_t(K, 128, key=key + (1,))
            X = wl.activations_student_t(K, 2, key=key + (2,))
        p = g.pack(torch.from_numpy(W).cuda())
        cols = _sampled_columns(N, rng)
        q, s, z = orc.rtn_quantize(W[:, cols])
        ws = g.vmm_workspace(p.layout)
        for t in targets:
            P = orc.maxent_distribution(np.array(CL, np.uint8), t)
            th = g.calibrate(dev_u16(Xc), CL, P=P)
            th_ref = orc.thresholds(Xc, P)
            assert np.array_equal(th.cpu().numpy(), th_ref)
            for v in X:
                xd = dev_u16(v)
                sel = g.select(xd, th, CL)
                y = _vmm_guarded(g, p, xd, sel, ws)
                bits, idx, off = orc.select(v, th_ref, np.array(CL, np.uint8))
                assert np.array_equal(sel.idx.cpu().numpy(), idx)
                yr, bound = orc.vmm(v, q, s, z, bits)
                assert_close(y[cols], yr, bound, "%s %s %.0f bits" % (family, name, t))
