"""GPU grading + compaction vs the oracle, bit-exact ("GRINQH" Section 3.1)."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, dev_u16

pytestmark = pytest.mark.gpu

CL = (0, 2, 3, 4, 8)


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _select_compare(g, orc, x_bits, theta, classes):
    K = len(x_bits)
    n = len(classes)
    bits = Guarded(K, torch.uint8)
    idx = Guarded(K, torch.int32)
    off = Guarded(n + 1, torch.int32)
    sel = g.Selection(bits.t, idx.t, off.t, tuple(classes))
    th = torch.from_numpy(np.asarray(theta, np.float32)).cuda() if n > 1 else None
    g.select(dev_u16(x_bits), th, classes, out=sel)
    torch.cuda.synchronize()
    for b in (bits, idx, off):
        b.check()
    rb, ri, ro = orc.select(x_bits, np.asarray(theta, np.float32), np.array(classes, np.uint8))
    assert np.array_equal(bits.t.cpu().numpy(), rb)
    assert np.array_equal(off.t.cpu().numpy(), ro)
    assert np.array_equal(idx.t.cpu().numpy(), ri)


def test_config0_vectors(g, orc):
    K = 1024
    Xc = wl.activations_outlier(K, 128, key=(0, 0, 0, 1), chan_key=(0, 0, 0))
    th = orc.thresholds(Xc, orc.maxent_distribution(np.array(CL, np.uint8), 4.0))
    X = wl.activations_outlier(K, 16, key=(0, 0, 0, 2), chan_key=(0, 0, 0))
    for v in X:
        _select_compare(g, orc, v, th, CL)


@pytest.mark.parametrize("K", [1, 2, 7, 1023, 1024, 1025, 4096, 4099, 14336, 65535, 65536])
def test_sizes(g, orc, K):
    x = wl.activations_student_t(K, 1, key=(21, K))[0]
    _select_compare(g, orc, x, [0.2, 0.6, 1.1, 2.5], CL)


def test_above_max_k_is_refused(g):
    # every 1024-channel block reads all of x: above 65536 channels the call is
    # refused before any launch, and the outputs are left untouched
    K = 65537
    x = torch.zeros(K, dtype=torch.int16, device="cuda")
    th = torch.tensor([0.2, 0.6, 1.1, 2.5], dtype=torch.float32, device="cuda")
    with pytest.raises(g.GrinqhError) as e:
        g.select(x, th, CL)
    assert e.value.code == 3


@pytest.mark.parametrize("classes,theta", [
    ((8,), []),
    ((0, 8), [0.7]),
    ((0, 1, 2, 3, 4, 5, 6, 7, 8), [0.1, 0.2, 0.3, 0.5, 0.8, 1.2, 1.9, 3.0]),
    ((2, 4, 6, 8), [0.3, 0.9, 2.0]),
    ((0, 2, 3, 4, 8), [0.0, 0.0, 1.0, np.inf]),
    ((0, 2, 3, 4, 8), [1.5, 0.5, 2.5, 0.1]),          # unsorted: still a count
])
def test_class_sets(g, orc, classes, theta):
    x = wl.activations_outlier(3000, 1, key=(22, len(classes)))[0]
    _select_compare(g, orc, x, theta, classes)


def test_specials(g, orc):
    vals = np.array([0.5, 1.0, 2.0, 4.0, -4.0, 0.0, -0.0, np.nan, np.inf, -np.inf, 0.499, 6.0e-8, 65504.0],
                    np.float16)
    x = np.tile(vals, 50).view(np.uint16)
    _select_compare(g, orc, x, [0.5, 1.0, 2.0, 4.0], CL)
