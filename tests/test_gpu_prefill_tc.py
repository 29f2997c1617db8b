"""The fused tensor-core prefill (grinqh_prefill_tc, tcgen05 on sm_100a) against the
fp64 oracle ("GRINQH" Section 4: prefill takes every weight at full b_max precision
and runs a dense product): within |y - y_ref| <= 1e-4 * sum_k |x_k w16_kn| + 1e-6 of
the fp64 product over the same binary16 operands (w16 = fp16_rne(s (q - z)), the
operands grinqh_dequant writes). Shapes cover several 64-row stages with a ragged
last stage, partial 128-column and 256-token tiles, every b_max, more than one CTA
along the token axis, and the 512-token tiles taken from 1024 tokens on; the status
word stays zero."""
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


def _run(g, orc, K, N, T, bmax, key, tokens=None):
    W = wl.weights_rowstd_loguniform(K, N, key=key + (0,))
    X = wl.activations_outlier(K, T, key=key + (1,), chan_key=key)
    p = g.pack(torch.from_numpy(W).cuda(), b_max=bmax)
    Xd = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).cuda()
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    Y = Guarded(T * N, torch.float32)
    Y.t.fill_(float("nan"))
    g.prefill_tc(p, Xd, status, Y=Y.t.view(T, N))
    torch.cuda.synchronize()
    Y.check()
    assert int(status.count_nonzero()) == 0, "a wait inside the kernel gave up"
    q, s, z = orc.rtn_quantize(W, bmax)
    w16 = orc.dequant_f16(q, s, z)
    rows = np.arange(T) if tokens is None else np.array(sorted(set(tokens)))
    Yr, bound = orc.prefill(np.ascontiguousarray(X[rows]), w16)
    Yg = Y.t.view(T, N).cpu().numpy()
    for i, t in enumerate(rows):
        assert_close(Yg[t], Yr[i], bound[i], "prefill_tc b_max=%d token %d" % (bmax, t))
    return p, Xd, Yg


@pytest.mark.parametrize("bmax", (8, 6, 4, 2))
@pytest.mark.parametrize("K,N,T", [(1024, 1024, 1), (1024, 1024, 7), (136, 1100, 64), (8, 8, 3), (520, 384, 33)])
def test_prefill_tc_matches_oracle(g, orc, bmax, K, N, T):
    _run(g, orc, K, N, T, bmax, (111, K, N, T, bmax))


def test_prefill_tc_several_token_tiles(g, orc):
    # 300 tokens: two CTAs along the token axis, the second one ragged; sampled tokens
    T = 300
    rng = np.random.default_rng(7)
    toks = list(rng.choice(T, 10, replace=False)) + [0, 255, 256, T - 1]
    _run(g, orc, 2048, 2048, T, 8, (112,), tokens=toks)


@pytest.mark.parametrize("bmax", (8, 4))
def test_prefill_tc_512_token_tiles(g, orc, bmax):
    # a CTA takes 512 tokens as two 256-token halves sharing the rebuilt weight tile
    # when that grid needs fewer waves: 4096 columns x 1200 tokens is 160 narrow CTAs
    # (two waves on 148 SMs) or 96 wide ones (one wave). Three wide CTAs along the token
    # axis, the last with a partial first half and an empty second half; sampled
    # tokens around the half and tile edges
    T = 1200
    toks = [0, 1, 255, 256, 300, 511, 512, 767, 768, 1023, 1024, 1050, 1151, T - 1]
    _run(g, orc, 136, 4096, T, bmax, (114, bmax), tokens=toks)


def test_prefill_tc_agrees_with_dequant_gemm(g, orc):
    # the same binary16 operands through grinqh_prefill (dequant + library GEMM):
    # both within the oracle's bound, so within twice of it of each other
    K, N, T = 4096, 1024, 48
    p, Xd, Yt = _run(g, orc, K, N, T, 8, (113,), tokens=[0, 17, 47])
    Yc = g.prefill(p, Xd).cpu().numpy()
    W = wl.weights_rowstd_loguniform(K, N, key=(113, 0))
    q, s, z = orc.rtn_quantize(W)
    w16 = orc.dequant_f16(q, s, z)
    X = Xd.cpu().numpy().view(np.uint16)
    for t in (0, 17, 47):
        _, bound = orc.prefill(np.ascontiguousarray(X[t:t + 1]), w16)
        assert np.all(np.abs(Yt[t].astype(np.float64) - Yc[t]) <= 2e-4 * bound[0] + 2e-6)


def test_prefill_tc_refuses_k_not_multiple_of_8(g):
    p = g.pack(torch.randn(12, 256, device="cuda"))
    X = torch.zeros((4, 12), dtype=torch.int16, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    with pytest.raises(g.GrinqhError) as e:
        g.prefill_tc(p, X, status)
    assert e.value.code == 3
