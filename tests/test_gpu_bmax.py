"""GPU pack, codes and graded product for codes of b_max < 8 bits against the fp64
oracle ("GRINQH" Section 3.3: weights quantised to a b_max-bit integer and stored as
2-bit segments, b_max in {4, 6, 8} evaluated; width b reads the top b bits, scaled
back by 2^(b_max - b), plus the midpoint 2^(b_max - b - 1)).

Bit-exact: scales, zero points, b_max-bit codes and nested codes at every width.
Within |y - y_ref| <= 1e-4 * sum_k |x_k w_hat_kn| + 1e-6: the graded product with the
pages' even class sets, ragged shapes, the fused call and the no-workspace call;
exactly equal: one-hot rows."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, assert_close, dev_u16, meta_split

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _even_classes(bmax):
    return tuple(range(0, bmax + 1, 2))


def _pack_check(g, orc, W, bmax, bits):
    K, N = W.shape
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    assert p.layout.b_max == bmax and p.layout.record_bytes == 128 * bmax
    q, s, z = orc.rtn_quantize(W, bmax)
    ms, mz = meta_split(p)
    assert np.array_equal(ms, s), "scale bits differ"
    assert np.array_equal(mz, z), "zero bits differ"
    out = Guarded(K * N, torch.uint8)
    rc = g._unpack(g.ctypes.byref(p.layout), p.packed.data_ptr(), None, out.t.data_ptr(),
                   torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    out.check()
    assert np.array_equal(out.t.cpu().numpy().reshape(K, N), q), "b_max-bit codes differ"
    codes = g.unpack_codes(p, torch.from_numpy(bits).cuda()).cpu().numpy()
    ref = np.zeros_like(q)
    for k in range(K):
        if bits[k]:
            ref[k] = [orc.code(int(v), int(bits[k]), bmax) for v in q[k]]
    assert np.array_equal(codes, ref), "nested codes differ"
    return p, q, s, z


@pytest.mark.parametrize("bmax", (2, 4, 6))
@pytest.mark.parametrize("K,N", [(1024, 1024), (37, 300), (130, 1029), (3, 2049)])
def test_pack_and_codes(g, orc, bmax, K, N):
    W = wl.weights_rowstd_loguniform(K, N, key=(81, bmax, K, N))
    bits = np.random.default_rng(K + N + bmax).integers(0, bmax + 1, K).astype(np.uint8)
    _pack_check(g, orc, W, bmax, bits)


@pytest.mark.parametrize("bmax", (4, 6))
def test_graded_product_even_classes(g, orc, bmax):
    # the pages' configuration: classes {0, 2, ..., b_max}, maximum-entropy
    # thresholds for a target mean width, outlier activations
    K, N = 1024, 1536
    cl = _even_classes(bmax)
    W = wl.weights_gaussian(K, N, key=(82, bmax))
    Xc = wl.activations_outlier(K, 64, key=(83, bmax, 1), chan_key=(83, bmax))
    X = wl.activations_outlier(K, 6, key=(83, bmax, 2), chan_key=(83, bmax))
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    q, s, z = orc.rtn_quantize(W, bmax)
    ws = g.vmm_workspace(p.layout)
    cla = np.array(cl, np.uint8)
    for target in (bmax / 2.0, bmax - 1.0):
        P = orc.maxent_distribution(cla, target)
        th = g.calibrate(dev_u16(Xc), cl, P=P)
        th_ref = orc.thresholds(Xc, P)
        assert np.array_equal(th.cpu().numpy(), th_ref)
        for v in X:
            xd = dev_u16(v)
            sel = g.select(xd, th, cl)
            y = Guarded(N, torch.float32)
            g.vmm(p, xd, sel, ws, y=y.t)
            yf = g.select_vmm(p, xd, th, cl, g.vmm_workspace(p.layout))
            yn = torch.empty(N, dtype=torch.float32, device="cuda")
            g.vmm_noalloc(p, xd, sel, yn)
            torch.cuda.synchronize()
            y.check()
            assert int(ws[:16].count_nonzero()) == 0
            bits, idx, off = orc.select(v, th_ref, cla)
            assert np.array_equal(sel.bits.cpu().numpy(), bits)
            assert np.array_equal(sel.idx.cpu().numpy(), idx)
            yr, bound = orc.vmm(v, q, s, z, bits, bmax=bmax)
            assert_close(y.t.cpu().numpy(), yr, bound, "vmm b_max=%d" % bmax)
            assert_close(yf.cpu().numpy(), yr, bound, "select_vmm b_max=%d" % bmax)
            assert torch.equal(yn, y.t), "no-workspace call differs from grinqh_vmm"


@pytest.mark.parametrize("bmax", (2, 4, 6))
def test_every_width_ragged(g, orc, bmax):
    # every width 0..b_max on a ragged shape (last group and tile partial)
    K, N = 333, 1100
    cl = tuple(range(bmax + 1))
    W = wl.weights_rowstd_loguniform(K, N, key=(84, bmax))
    x = wl.activations_student_t(K, 1, key=(85, bmax))[0]
    bits = np.random.default_rng(bmax).integers(0, bmax + 1, K).astype(np.uint8)
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    q, s, z = orc.rtn_quantize(W, bmax)
    idx, off = orc.compact(bits, np.array(cl, np.uint8))
    sel = g.Selection(torch.from_numpy(bits).cuda(), torch.from_numpy(idx).cuda(), torch.from_numpy(off).cuda(), cl)
    y = g.vmm(p, dev_u16(x), sel, g.vmm_workspace(p.layout))
    torch.cuda.synchronize()
    yr, bound = orc.vmm(x, q, s, z, bits, bmax=bmax)
    assert_close(y.cpu().numpy(), yr, bound, "ragged b_max=%d" % bmax)


@pytest.mark.parametrize("bmax", (4, 6))
def test_one_hot_rows_are_exact(g, orc, bmax):
    K, N = 64, 700
    cl = tuple(range(bmax + 1))
    W = wl.weights_rowstd_loguniform(K, N, key=(86, bmax))
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    q, s, z = orc.rtn_quantize(W, bmax)
    ws = g.vmm_workspace(p.layout)
    for k in np.random.default_rng(bmax).choice(K, 6, replace=False):
        for b in range(1, bmax + 1):
            x = np.zeros(K, np.float16)
            x[k] = 1.0
            bits = np.zeros(K, np.uint8)
            bits[k] = b
            idx, off = orc.compact(bits, np.array(cl, np.uint8))
            sel = g.Selection(torch.from_numpy(bits).cuda(), torch.from_numpy(idx).cuda(),
                              torch.from_numpy(off).cuda(), cl)
            y = g.vmm(p, dev_u16(x.view(np.uint16)), sel, ws)
            torch.cuda.synchronize()
            yr, _ = orc.vmm(x.view(np.uint16), q, s, z, bits, bmax=bmax)
            assert np.array_equal(y.cpu().numpy().astype(np.float64), yr), (k, b)


def test_full_size_q_proj_bmax6(g, orc):
    # Llama3-8B q_proj shape at b_max = 6 with the pages' classes {0,2,4,6},
    # 3 average bits; columns sampled by whole groups, the last one included
    K, N, bmax = 4096, 4096, 6
    cl = _even_classes(bmax)
    W = wl.weights_gaussian(K, N, key=(87, 0))
    Xc = wl.activations_outlier(K, 128, key=(87, 1), chan_key=(87,))
    x = wl.activations_outlier(K, 1, key=(87, 2), chan_key=(87,))[0]
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    P = orc.maxent_distribution(np.array(cl, np.uint8), 3.0)
    th = g.calibrate(dev_u16(Xc), cl, P=P)
    sel = g.select(dev_u16(x), th, cl)
    y = g.vmm(p, dev_u16(x), sel, g.vmm_workspace(p.layout)).cpu().numpy()
    bits = sel.bits.cpu().numpy()
    assert abs(bits.mean() - 3.0) < 0.5
    rng = np.random.default_rng(5)
    gs = sorted(set(list(rng.choice(N // 128, 3, replace=False)) + [N // 128 - 1]))
    cols = np.concatenate([np.arange(128 * c, 128 * c + 128) for c in gs])
    q, s, z = orc.rtn_quantize(W[:, cols], bmax)
    yr, bound = orc.vmm(x, q, s, z, bits, bmax=bmax)
    assert_close(y[cols], yr, bound, "q_proj b_max=6")
