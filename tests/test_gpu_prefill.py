"""The prefill path against the fp64 oracle ("GRINQH" Section 4: prefill unpacks
the weights at full b_max precision and runs a dense matrix-matrix product):
grinqh_dequant bit-exact (w_hat = s (q - z) rounded once to binary16), and
grinqh_prefill within |y - y_ref| <= 1e-4 * sum_k |x_k w16_kn| + 1e-6 of the fp64
product over the same binary16 operands."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


@pytest.mark.parametrize("bmax", (8, 6, 4))
@pytest.mark.parametrize("K,N", [(1024, 1024), (37, 300), (130, 1029), (5, 2048), (3, 8)])
def test_dequant_bit_exact(g, orc, bmax, K, N):
    W = wl.weights_rowstd_loguniform(K, N, key=(101, K, N, bmax))
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    out = Guarded(K * N, torch.float16)
    g.dequant(p, out=out.t.view(K, N))
    torch.cuda.synchronize()
    out.check()
    q, s, z = orc.rtn_quantize(W, bmax)
    ref = orc.dequant_f16(q, s, z)
    assert np.array_equal(out.t.cpu().numpy().view(np.uint16).reshape(K, N), ref)


@pytest.mark.parametrize("K,N,T", [(1024, 1024, 1), (1024, 1024, 7), (333, 1100, 64), (4096, 4096, 16)])
def test_prefill_matches_oracle(g, orc, K, N, T):
    W = wl.weights_gaussian(K, N, key=(102, K, N))
    X = wl.activations_outlier(K, T, key=(103, K, T), chan_key=(103, K))
    p = g.pack(torch.from_numpy(W).cuda())
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    Y = Guarded(T * N, torch.float32)
    g.prefill(p, Xd, Y=Y.t.view(T, N))
    torch.cuda.synchronize()
    Y.check()
    q, s, z = orc.rtn_quantize(W)
    w16 = orc.dequant_f16(q, s, z)
    Yr, bound = orc.prefill(X, w16)
    Yg = Y.t.view(T, N).cpu().numpy()
    for t in range(T):
        assert_close(Yg[t], Yr[t], bound[t], "prefill token %d" % t)


def test_prefill_full_width_agrees_with_vmm_at_b_max(g, orc):
    # one token, every row at b_max: the graded product over the same weights;
    # the two differ only by the binary16 rounding of w_hat (at most 2^-11 of
    # each term) and fp32 summation
    K, N = 2048, 3072
    W = wl.weights_gaussian(K, N, key=(104, 0))
    x = wl.activations_outlier(K, 1, key=(104, 1), chan_key=(104,))
    p = g.pack(torch.from_numpy(W).cuda())
    xd = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda()
    y_pre = g.prefill(p, xd)[0].cpu().numpy().astype(np.float64)
    sel = g.select(xd[0], None, (8,))
    y_vmm = g.vmm(p, xd[0], sel, g.vmm_workspace(p.layout)).cpu().numpy().astype(np.float64)
    q, s, z = orc.rtn_quantize(W)
    _, bound = orc.vmm(x[0], q, s, z, np.full(K, 8, np.uint8))
    assert np.all(np.abs(y_pre - y_vmm) <= 2.0 ** -11 * bound + 2e-4 * bound + 2e-6)
