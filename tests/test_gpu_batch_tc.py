"""The batched graded product on the tensor cores (grinqh_select_vmm_batch_tc)
against the fp64 oracle ("GRINQH" Section 3.1 per-token grading, Fig. 2 / Section
3.3 graded product with the bin midpoint; every token keeps its own widths, as at
batch one): |y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6 for every token.
Shapes cover several 64-row stages with a ragged last one, a partial 128-column
group, padded token counts (N of the MMA a multiple of 16), two CTAs along the
token axis, K splits over clusters of 2, 4 and 8 CTAs and none, b_max 8/6/4/2,
classes with odd widths, only width 8 (dense) and only width 0 (y = 0); the
status word stays zero and repeated calls give the same bits."""
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


def _case(g, orc, K, N, T, bmax, classes, key, target=3.0, tokens=None, cols=None):
    cl = np.array(classes, np.uint8)
    W = wl.weights_rowstd_loguniform(K, N, key=key + (0,))
    Xc = wl.activations_outlier(K, 64, key=key + (1,), chan_key=key)
    X = wl.activations_outlier(K, T, key=key + (2,), chan_key=key)
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    if len(classes) > 1:
        P = orc.maxent_distribution(cl, min(target, float(classes[-1])))
        th = g.calibrate(dev_u16(Xc), classes, P=P)
        th_ref = orc.thresholds(Xc, P)
        assert np.array_equal(th.cpu().numpy(), th_ref)
    else:
        th, th_ref = None, np.zeros(0, np.float32)
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y = Guarded(T * N, torch.float32)
    Y.t.fill_(float("nan"))
    g.select_vmm_batch_tc(p, Xd, th, classes, status, Y=Y.t.view(T, N))
    Y2 = g.select_vmm_batch_tc(p, Xd, th, classes, status)
    torch.cuda.synchronize()
    Y.check()
    assert int(status.count_nonzero()) == 0, "status %s" % status.cpu().numpy()
    Yb = Y.t.view(T, N).cpu().numpy()
    assert np.array_equal(Yb.view(np.uint32), Y2.cpu().numpy().view(np.uint32)), "not repeatable"
    cols = np.arange(N) if cols is None else cols
    q, s, z = orc.rtn_quantize(np.ascontiguousarray(W[:, cols]), bmax)
    toks = range(T) if tokens is None else tokens
    for t in toks:
        bits, _, _ = orc.select(X[t], th_ref, cl)
        yr, bound = orc.vmm(X[t], q, s, z, bits, bmax=bmax)
        assert_close(Yb[t][cols], yr, bound, "batch_tc b_max=%d token %d" % (bmax, t))
    return p, Xd, th, Yb


@pytest.mark.parametrize("K,N,T", [(1024, 1024, 16), (520, 300, 5), (1024, 384, 1), (136, 1100, 33)])
def test_batch_tc_matches_oracle(g, orc, K, N, T):
    _case(g, orc, K, N, T, 8, CL, (131, K, N, T))


@pytest.mark.parametrize("bmax", (6, 4, 2))
def test_batch_tc_bmax(g, orc, bmax):
    classes = tuple(range(0, bmax + 1)) if bmax <= 4 else (0, 2, 3, 4, 6)
    _case(g, orc, 1032, 640, 12, bmax, classes, (132, bmax), target=bmax / 2.0)


def test_batch_tc_two_token_chunks_and_large_layer(g, orc):
    # 100 tokens: two CTAs along the token axis (64 + 36); 4096 x 4096 launches 32
    # groups x 2 chunks (no K split); sampled tokens and columns
    N = 4096
    cols = np.concatenate([np.arange(0, 128), np.arange(2048, 2176), np.arange(N - 128, N)])
    _case(g, orc, 4096, N, 100, 8, CL, (133,), tokens=[0, 1, 31, 63, 64, 65, 99], cols=cols)


def test_batch_tc_split_four_and_none(g, orc):
    # 32 groups: a K split over clusters of 4; 80 groups: no split
    cols = np.concatenate([np.arange(0, 128), np.arange(4096 - 128, 4096)])
    _case(g, orc, 1024, 4096, 8, 8, CL, (136, 0), cols=cols)
    cols = np.concatenate([np.arange(0, 128), np.arange(10240 - 256, 10240)])
    _case(g, orc, 256, 10240, 4, 8, CL, (136, 1), cols=cols)


def test_batch_tc_dense_and_empty_class_sets(g, orc):
    _case(g, orc, 512, 1024, 8, 8, (8,), (134, 0))       # every row at 8 bits: the dense product
    _case(g, orc, 512, 1024, 8, 8, (0, 8), (134, 1))     # rows skipped or full
    p, Xd, th, Yb = _case(g, orc, 512, 1024, 8, 8, (0,), (134, 2))   # every row skipped
    assert not np.any(Yb)


def test_batch_tc_agrees_with_per_token_batch(g, orc):
    K, N, T = 2048, 2048, 16
    p, Xd, th, Yt = _case(g, orc, K, N, T, 8, CL, (135,), tokens=[0, 15])
    ws = g.vmm_batch_workspace(p.layout, T)
    Yp = g.select_vmm_batch(p, Xd, th, CL, ws).cpu().numpy()
    # both within the oracle's bound of each token, so within twice of it of each other
    W = wl.weights_rowstd_loguniform(K, N, key=(135, 0))
    q, s, z = orc.rtn_quantize(W)
    X = Xd.cpu().numpy().view(np.uint16)
    Xc = wl.activations_outlier(K, 64, key=(135, 1), chan_key=(135,))
    th_ref = orc.thresholds(Xc, orc.maxent_distribution(np.array(CL, np.uint8), 3.0))
    for t in (3, 9):
        bits, _, _ = orc.select(X[t], th_ref, np.array(CL, np.uint8))
        _, bound = orc.vmm(X[t], q, s, z, bits)
        assert np.all(np.abs(Yt[t].astype(np.float64) - Yp[t]) <= 2e-4 * bound + 2e-6)


def test_batch_tc_refuses_k_not_multiple_of_8(g):
    p = g.pack(torch.randn(12, 256, device="cuda"))
    X = torch.zeros((4, 12), dtype=torch.int16, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    th = torch.tensor([0.5, 1.0, 1.5, 2.0], dtype=torch.float32, device="cuda")
    with pytest.raises(g.GrinqhError) as e:
        g.select_vmm_batch_tc(p, X, th, CL, status)
    assert e.value.code == 3


def test_batch_tc_threshold_ties_and_unrepresentable_thresholds(g, orc):
    """Section 3.1: a channel's class is the number of thresholds its |x| reaches.
    Thresholds equal to some |x| (a tie reaches it), one fp32 step above and below
    a binary16 value, zero, unsorted and above every |x|: the kernel (which
    compares binary16 |x| with the thresholds rounded up to binary16) takes the
    oracle's fp32 decisions, so y agrees within the VMM tolerance for every token."""
    K, N, T = 512, 256, 8
    key = (141,)
    W = wl.weights_rowstd_loguniform(K, N, key=key + (0,))
    X = wl.activations_outlier(K, T, key=key + (2,), chan_key=key)
    ax = np.abs(X.view(np.float16).astype(np.float32))
    a, b, c = float(ax[0, 5]), float(ax[1, 7]), float(ax[2, 9])
    cases = [np.array([a, np.nextafter(np.float32(b), np.float32(np.inf)), np.nextafter(np.float32(c), np.float32(0)),
                       float(ax.max()) * 2.0], np.float32),
             np.array([float(ax.max()) * 2.0, a, 0.0, b], np.float32)]   # unsorted, with zero
    p = g.pack(torch.from_numpy(W).cuda())
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    q, s, z = orc.rtn_quantize(W, 8)
    cl = np.array(CL, np.uint8)
    for th_ref in cases:
        status = torch.zeros(4, dtype=torch.int32, device="cuda")
        Y = g.select_vmm_batch_tc(p, Xd, torch.from_numpy(th_ref).cuda(), CL, status)
        torch.cuda.synchronize()
        assert int(status.count_nonzero()) == 0
        Yb = Y.cpu().numpy()
        for t in range(T):
            bits, _, _ = orc.select(X[t], th_ref, cl)
            yr, bound = orc.vmm(X[t], q, s, z, bits)
            assert_close(Yb[t], yr, bound, "thresholds %s token %d" % (th_ref, t))


def test_batch_tc_flags_values_outside_binary16_range(g):
    """|x| times the scale's significand at 32768 or more (after rounding to
    binary16) has no binary16 operand: the kernel sets bit 1 of the status word;
    below it (|x| <= 16000, significand < 2) the word stays zero."""
    K, N, T = 256, 256, 4
    p = g.pack(torch.randn(K, N, device="cuda") * 0.02)
    th = torch.tensor([0.5, 1.0, 1.5, 2.0], dtype=torch.float32, device="cuda")
    X = torch.zeros((T, K), dtype=torch.float16, device="cuda")
    X[:, ::3] = 16000.0
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    g.select_vmm_batch_tc(p, X.view(torch.int16), th, CL, status)
    torch.cuda.synchronize()
    assert int(status.count_nonzero()) == 0
    X[2, 77] = 40000.0
    g.select_vmm_batch_tc(p, X.view(torch.int16), th, CL, status)
    torch.cuda.synchronize()
    assert int(status[0].item()) == 2, status.cpu().numpy()
