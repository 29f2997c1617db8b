"""The batched fused call grinqh_select_vmm_batch: row t of Y is bitwise what
grinqh_select_vmm gives for row t of X, and within the bound of the fp64 oracle
("GRINQH" Section 3.1 per-token grading, Fig. 2 / Section 3.3 graded product;
every token keeps its own widths, as at batch one).
|y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6."""
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


@pytest.mark.parametrize("K,N,T,bmax", [(1024, 1024, 2, 8), (1024, 1024, 5, 8), (333, 1100, 3, 8),
                                        (4096, 4096, 4, 8), (1024, 3072, 3, 6), (14336, 4096, 2, 8)])
def test_batch_rows_equal_single_calls_and_oracle(g, orc, K, N, T, bmax):
    classes = CL if bmax == 8 else tuple(range(0, bmax + 1, 2))
    cl = np.array(classes, np.uint8)
    W = wl.weights_rowstd_loguniform(K, N, key=(95, K, N))
    Xc = wl.activations_outlier(K, 64, key=(96, K, 1), chan_key=(96, K))
    X = wl.activations_outlier(K, T, key=(96, K, 2), chan_key=(96, K))
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    P = orc.maxent_distribution(cl, min(3.0, float(bmax)))
    th = g.calibrate(dev_u16(Xc), classes, P=P)
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    Y = Guarded(T * N, torch.float32)
    ws = g.vmm_batch_workspace(p.layout, T)
    g.select_vmm_batch(p, Xd, th, classes, ws, Y=Y.t.view(T, N))
    torch.cuda.synchronize()
    Y.check()
    assert int(ws[:16].count_nonzero()) == 0
    Yb = Y.t.view(T, N).cpu().numpy()
    q, s, z = orc.rtn_quantize(W, bmax)
    th_ref = orc.thresholds(Xc, P)
    cols = np.arange(N) if K * N <= 4 * 1024 * 1024 else np.concatenate(
        [np.arange(0, 128), np.arange(N - 128, N)])
    qc, sc, zc = (q, s, z) if cols.size == N else orc.rtn_quantize(W[:, cols], bmax)
    for t in range(T):
        y1 = g.select_vmm(p, dev_u16(X[t]), th, classes, g.vmm_workspace(p.layout)).cpu().numpy()
        assert np.array_equal(Yb[t].view(np.uint32), y1.view(np.uint32)), "token %d differs from a single call" % t
        bits, _, _ = orc.select(X[t], th_ref, cl)
        yr, bound = orc.vmm(X[t], qc, sc, zc, bits, bmax=bmax)
        assert_close(Yb[t][cols], yr, bound, "batch token %d" % t)


def test_batch_of_one_and_repeat(g, orc):
    K, N = 512, 2048
    W = wl.weights_gaussian(K, N, key=(97, 0))
    X = wl.activations_outlier(K, 1, key=(97, 1), chan_key=(97,))
    p = g.pack(torch.from_numpy(W).cuda())
    th = torch.tensor([0.5, 1.0, 1.5, 2.0], dtype=torch.float32, device="cuda")
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    ws = g.vmm_batch_workspace(p.layout, 1)
    a = g.select_vmm_batch(p, Xd, th, CL, ws).cpu().numpy()
    b = g.select_vmm_batch(p, Xd, th, CL, ws).cpu().numpy()
    y1 = g.select_vmm(p, dev_u16(X[0]), th, CL, g.vmm_workspace(p.layout)).cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(a[0].view(np.uint32), y1.view(np.uint32))
