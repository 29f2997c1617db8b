"""Tall layers against the fp64 oracle ("GRINQH" Fig. 2 / Section 3.3): K large
enough that a CTA of grinqh_vmm holds more channel-list positions than it loads
in its first round trip (K / R > 2048) and, beyond that, more rows than one
staging pass holds (K / R > 16384), so the kernel stages its rows in several
passes. Narrow N keeps the oracle to seconds; every column is checked.
|y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6. grinqh_select takes at most 65536
channels (every 1024-channel block reads all of x), so above that the channel list
given to grinqh_vmm is the oracle's selection, as the header tells such callers to
build it themselves; the call refuses these sizes (UNSUPPORTED)."""
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


@pytest.mark.parametrize("K,N,target", [(65_536, 160, 3.0), (200_000, 96, 3.0), (1_400_000, 40, 3.0),
                                        (1_400_000, 40, 8.0)])
def test_tall_layer_multi_pass_staging(g, orc, K, N, target):
    W = wl.weights_gaussian(K, N, key=(91, K, N))
    x = wl.activations_gaussian(K, 1, key=(92, K))[0]
    Xc = wl.activations_gaussian(K, 8, key=(93, K))
    p = g.pack(torch.from_numpy(W).cuda())
    P = orc.maxent_distribution(np.array(CL, np.uint8), target)
    th = g.calibrate(dev_u16(Xc), CL, P=P)
    xd = dev_u16(x)
    th_ref = orc.thresholds(Xc, P)
    assert np.array_equal(th.cpu().numpy(), th_ref)
    bits_ref, idx_ref, off_ref = orc.select(x, th_ref, np.array(CL, np.uint8))
    if K <= 65536:
        sel = g.select(xd, th, CL)
    else:
        with pytest.raises(g.GrinqhError) as e:
            g.select(xd, th, CL)
        assert e.value.code == 3
        sel = g.Selection(torch.from_numpy(bits_ref).cuda(), torch.from_numpy(idx_ref).cuda(),
                          torch.from_numpy(off_ref).cuda(), CL)
    y = Guarded(N, torch.float32)
    ws = g.vmm_workspace(p.layout)
    g.vmm(p, xd, sel, ws, y=y.t)
    torch.cuda.synchronize()
    y.check()
    assert int(ws[:16].count_nonzero()) == 0
    bits = sel.bits.cpu().numpy()
    assert np.array_equal(bits, bits_ref)
    assert np.array_equal(sel.idx.cpu().numpy(), idx_ref)
    del W
    W = wl.weights_gaussian(K, N, key=(91, K, N))
    q, s, z = orc.rtn_quantize(W)
    yr, bound = orc.vmm(x, q, s, z, bits, nthreads=8)
    assert_close(y.t.cpu().numpy(), yr, bound, "tall K=%d" % K)
