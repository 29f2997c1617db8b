"""grinqh_vmm_noalloc (the VMM on the library's static scratch, no workspace)
against grinqh_vmm on the same inputs: y must be the same bits, on two calls in
a row (the second call finds the scratch as the first one left it).

The file name sorts last so that pytest collects it after every other test;
it must also pass alone in a fresh process."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, dev_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


@pytest.mark.parametrize("K,N,target", [(1024, 1024, 4.0), (1025, 1029, 3.0), (4096, 4096, 3.0),
                                        (4096, 14336, 2.0), (14336, 4096, 3.0)])
def test_noalloc_matches_workspace_entry_point(g, K, N, target):
    key = (77, K, N)
    p = g.pack(torch.from_numpy(wl.weights_gaussian(K, N, key=key)).cuda())
    Xc = wl.activations_outlier(K, 64, key=key + (1,), chan_key=key)
    th = g.calibrate(dev_u16(Xc), wl.CLASSES, target_bits=target)
    x = dev_u16(wl.activations_outlier(K, 1, key=key + (2,), chan_key=key)[0])
    sel = g.select(x, th, wl.CLASSES)
    y_ref = g.vmm(p, x, sel, g.vmm_workspace(p.layout))
    outs = []
    for _ in range(2):
        y = Guarded(N, torch.float32)
        y.t.fill_(float("nan"))
        g.vmm_noalloc(p, x, sel, y.t)
        outs.append(y)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y_ref).all())
    for y in outs:
        y.check()
        assert torch.equal(y.t, y_ref), "vmm_noalloc differs from vmm (max |diff| %g)" % float(
            (y.t - y_ref).abs().max())


def test_noalloc_rejects_bad_arguments_before_launch(g):
    """Host validation runs before anything is enqueued; the pointers are never
    dereferenced, so plain integers stand in for device buffers."""
    import ctypes
    L = g.layout(64, 64)
    cls = (ctypes.c_uint8 * 5)(*wl.CLASSES)
    ok = 1 << 20   # 1 MiB-aligned fake address
    args = dict(packed=ok, x=ok, idx=ok, off=ok, y=ok)

    def call(**kw):
        a = dict(args, **kw)
        return g._vmm_noalloc(ctypes.byref(L), a["packed"], a["x"], a["idx"], a["off"], ctypes.addressof(cls), 5,
                              a["y"], None)

    assert call(y=ok + 2) == 2          # y not 4-byte aligned
    assert call(packed=ok + 8) == 2     # packed not 16-byte aligned
    assert call(y=None) == 1            # missing output
    bad = (ctypes.c_uint8 * 2)(4, 2)    # classes not increasing
    assert g._vmm_noalloc(ctypes.byref(L), ok, ok, ok, ok, ctypes.addressof(bad), 2, ok, None) == 1
