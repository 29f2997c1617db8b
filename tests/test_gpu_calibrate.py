"""GPU threshold calibration vs the oracle, bit-exact ("GRINQH" Section 3.2,
Appendix A.1 eq. (2))."""
import os

import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, dev_u16

pytestmark = pytest.mark.gpu

CL = (0, 2, 3, 4, 8)
GOLD = os.path.join(os.path.dirname(__file__), "golden", "table3_bmax8_precision_distributions.txt")


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _cal_compare(g, orc, X, classes, P):
    n = len(classes)
    out = Guarded(n - 1, torch.float32)
    g.calibrate(dev_u16(X), classes, P=P, out=out.t)
    torch.cuda.synchronize()
    out.check()
    ref = orc.thresholds(X, np.asarray(P, np.float64))
    got = out.t.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (got, ref)
    return got


@pytest.mark.parametrize("target", [4.0, 3.0, 2.0])
def test_config0_calibration(g, orc, target):
    X = wl.activations_outlier(1024, 128, key=(0, 0, 0, 1), chan_key=(0, 0, 0))
    P = orc.maxent_distribution(np.array(CL, np.uint8), target)
    _cal_compare(g, orc, X, CL, P)


def test_maxent_path_matches(g, orc):
    X = wl.activations_outlier(4096, 128, key=(1, 0, 0, 1), chan_key=(1, 0, 0))
    th = g.calibrate(dev_u16(X), CL, P=None, target_bits=3.0).cpu().numpy()
    ref = orc.thresholds(X, orc.maxent_distribution(np.array(CL, np.uint8), 3.0))
    assert np.array_equal(th.view(np.uint32), ref.view(np.uint32))


def test_table3_distributions(g, orc):
    X = wl.activations_student_t(2048, 64, key=(31, 1))
    classes = (0, 2, 4, 6, 8)
    for line in open(GOLD):
        if line.startswith("#") or not line.strip():
            continue
        v = [float(t) for t in line.split()[1:]]
        P = np.array(v) / np.sum(v)
        _cal_compare(g, orc, X, classes, P)


@pytest.mark.parametrize("K,S", [(1, 1), (2, 3), (3, 128), (1000, 1), (14336, 16), (65537, 2)])
def test_sizes(g, orc, K, S):
    X = wl.activations_silu_gated(K, S, key=(32, K, S))
    _cal_compare(g, orc, X, CL, [0.2, 0.2, 0.2, 0.2, 0.2])


def test_special_distributions_and_ties(g, orc):
    X = wl.activations_gaussian(512, 8, key=(33, 1))
    X[:, ::3] = np.float16(1.0).view(np.uint16)          # many ties
    for P in ([0.0, 0.0, 1.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0, 1.0], [1.0, 0.0, 0.0, 0.0, 0.0],
              [0.5, 0.0, 0.25, 0.0, 0.25], [0.15, 0.175, 0.19, 0.205, 0.28]):
        _cal_compare(g, orc, X, CL, P)
