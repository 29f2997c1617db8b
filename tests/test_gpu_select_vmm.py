"""The fused call grinqh_select_vmm against the fp64 oracle ("GRINQH" Section 3.1
grading, Fig. 2 / Section 3.3 graded product) and against grinqh_select +
grinqh_vmm (the same graded rows summed in another order: both within the
oracle's bound), and bitwise reproducible from call to call."""
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


def _both(g, p, x_bits, theta, classes):
    """(fused y, separate y) for one input; checks guards, the status word and
    that a second fused call gives the same bits."""
    xd = dev_u16(x_bits)
    th = torch.from_numpy(np.asarray(theta, np.float32)).cuda() if len(classes) > 1 else None
    ws = g.vmm_workspace(p.layout)
    y = Guarded(p.N, torch.float32)
    y.t.fill_(float("nan"))
    g.select_vmm(p, xd, th, classes, ws, y=y.t)
    y2 = g.select_vmm(p, xd, th, classes, g.vmm_workspace(p.layout))
    sel = g.select(xd, th, classes)
    y_sep = g.vmm(p, xd, sel, g.vmm_workspace(p.layout))
    torch.cuda.synchronize()
    y.check()
    assert int(ws[:16].count_nonzero()) == 0, "status word set"
    yf = y.t.cpu().numpy()
    assert np.array_equal(yf.view(np.uint32), y2.cpu().numpy().view(np.uint32)), "fused y not reproducible"
    return yf, y_sep.cpu().numpy()


def _cols(N, rng, groups=3):
    """Whole 128-column groups, the last one always among them."""
    ng = (N + 127) // 128
    pick = sorted(set(rng.choice(ng, size=min(groups, ng), replace=False).tolist()) | {ng - 1})
    return np.concatenate([np.arange(q * 128, min(N, q * 128 + 128)) for q in pick])


def _check_both(orc, W, x, theta, classes, yf, ys, what, cols=None):
    """Fused and separate y both within the oracle's bound (on the columns cols)."""
    if cols is None:
        cols = np.arange(W.shape[1])
    q, s, z = orc.rtn_quantize(W[:, cols])
    bits, _, _ = orc.select(x, np.asarray(theta, np.float32), np.array(classes, np.uint8))
    yr, bound = orc.vmm(x, q, s, z, bits)
    assert_close(yf[cols], yr, bound, "fused " + what)
    assert_close(ys[cols], yr, bound, "select + vmm " + what)


@pytest.mark.parametrize("K,N", [(1, 1), (7, 300), (512, 1024), (1025, 1029), (4096, 1024), (4096, 4096),
                                 (5000, 64), (14336, 4096), (16384, 2048)])
def test_fused_matches_oracle_and_select_then_vmm(g, orc, K, N):
    key = (61, K, N)
    W = wl.weights_gaussian(K, N, key=key)
    p = g.pack(torch.from_numpy(W).cuda())
    Xc = wl.activations_outlier(K, 64, key=key + (1,), chan_key=key)
    th = orc.thresholds(Xc, orc.maxent_distribution(np.array(CL, np.uint8), 3.0))
    x = wl.activations_outlier(K, 1, key=key + (2,), chan_key=key)[0]
    yf, ys = _both(g, p, x, th, CL)
    cols = None if K * N <= 4096 * 4096 else _cols(N, np.random.default_rng(K))
    _check_both(orc, W, x, th, CL, yf, ys, "%dx%d" % (K, N), cols)


@pytest.mark.parametrize("classes,theta", [
    ((8,), []),
    ((0, 8), [0.7]),
    ((2, 4, 6, 8), [0.3, 0.9, 2.0]),
    ((0, 1, 2, 3, 4, 5, 6, 7, 8), [0.1, 0.2, 0.3, 0.5, 0.8, 1.2, 1.9, 3.0]),
    ((0, 2, 3, 4, 8), [0.0, 0.0, 1.0, np.inf]),
    ((0, 2, 3, 4, 8), [1.5, 0.5, 2.5, 0.1]),          # unsorted thresholds: still a count
    ((0, 2, 3, 4, 8), [0.5, np.nan, 2.5, 0.1]),       # a NaN threshold is never reached
])
def test_class_sets_and_thresholds(g, orc, classes, theta):
    K, N = 3000, 1536
    key = (62, len(classes))
    W = wl.weights_gaussian(K, N, key=key)
    p = g.pack(torch.from_numpy(W).cuda())
    x = wl.activations_outlier(K, 1, key=key + (1,))[0]
    yf, ys = _both(g, p, x, theta, classes)
    _check_both(orc, W, x, theta, classes, yf, ys, "classes %s" % (classes,))


def test_special_activations(g, orc):
    vals = np.array([0.5, 1.0, 2.0, 4.0, -4.0, 0.0, -0.0, 0.499, 6.0e-8, 65504.0, -65504.0], np.float16)
    K, N = 1100, 640
    x = np.tile(vals, K // len(vals) + 1)[:K].view(np.uint16)
    W = wl.weights_gaussian(K, N, key=(63, 1))
    p = g.pack(torch.from_numpy(W).cuda())
    th = [0.5, 1.0, 2.0, 4.0]
    yf, ys = _both(g, p, x, th, CL)
    _check_both(orc, W, x, th, CL, yf, ys, "specials")


def test_nan_activation_is_skipped(g, orc):
    """A NaN channel grades to class 0 (width 0) and is never read, so y stays finite."""
    K, N = 600, 300
    x = wl.activations_outlier(K, 1, key=(64, 1))[0].copy()
    x[::7] = np.array([np.nan], np.float16).view(np.uint16)[0]
    W = wl.weights_gaussian(K, N, key=(64, 2))
    p = g.pack(torch.from_numpy(W).cuda())
    th = [0.3, 0.9, 1.5, 3.0]
    yf, ys = _both(g, p, x, th, CL)
    assert np.isfinite(yf).all()
    _check_both(orc, W, x, th, CL, yf, ys, "NaN channels")


def test_k_above_limit_is_unsupported(g):
    import ctypes
    L = g.layout(16385, 64)
    cls = (ctypes.c_uint8 * 5)(*CL)
    ok = 1 << 20
    rc = g._select_vmm(ctypes.byref(L), ok, ok, ok, ctypes.addressof(cls), 5, ok, ok, 1 << 30, None)
    assert rc == 3   # GRINQH_ERR_UNSUPPORTED, before any launch
