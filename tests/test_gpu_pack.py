"""GPU pack and code decoding vs the oracle: bit-exact RTN codes, scales and zero
points ("GRINQH" Section 3.3, Section 4), and bit-exact nested codes at every width."""
import numpy as np
import pytest
import torch

from activation_graded_bit_b200 import workloads as wl
from gpu_util import Guarded, meta_split

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _pack_and_compare(g, orc, W, bits=None):
    K, N = W.shape
    p = g.pack(torch.from_numpy(W).cuda())
    q, s, z = orc.rtn_quantize(W)
    ms, mz = meta_split(p)
    assert np.array_equal(ms, s), "scale bits differ"
    assert np.array_equal(mz, z), "zero bits differ"
    full = p.meta_words().cpu().numpy().view(np.uint32).reshape(K, p.layout.n_tiles * 8)
    assert np.all(full[:, p.layout.n_groups:] == 0)
    out = Guarded(K * N, torch.uint8)
    rc = g._unpack(g.ctypes.byref(p.layout), p.packed.data_ptr(), None, out.t.data_ptr(),
                   torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    out.check()
    assert np.array_equal(out.t.cpu().numpy().reshape(K, N), q), "8-bit codes differ"
    if bits is not None:
        codes = g.unpack_codes(p, torch.from_numpy(bits).cuda()).cpu().numpy()
        ref = np.zeros_like(q)
        for k in range(K):
            if bits[k]:
                ref[k] = [orc.code(int(v), int(bits[k])) for v in q[k]]
        assert np.array_equal(codes, ref), "nested codes differ"
    return p, q


def test_config0_layer(g, orc):
    W = wl.weights_gaussian(1024, 1024, key=(0, 0, 0, 0))
    bits = np.random.default_rng(0).integers(0, 9, 1024).astype(np.uint8)
    _pack_and_compare(g, orc, W, bits)


@pytest.mark.parametrize("K,N", [(1, 1), (4, 4), (37, 300), (5, 1000), (3, 513), (130, 1029), (2, 128), (9, 640),
                                 (3, 1024), (2, 2049)])
def test_ragged_shapes(g, orc, K, N):
    W = wl.weights_rowstd_loguniform(K, N, key=(11, K, N))
    bits = np.random.default_rng(K * 7 + N).integers(0, 9, K).astype(np.uint8)
    _pack_and_compare(g, orc, W, bits)


def test_special_groups(g, orc):
    u = 2.0 ** -10
    W = np.zeros((6, 256), np.float32)
    W[0, :128] = [(2 * j - 128) * u for j in range(127)] + [127 * u]       # exact grid
    W[0, 128:] = np.array([-128 * u, 127 * u] + [2.5 * u, 3.5 * u, -2.5 * u, -3.5 * u] * 31 + [0.0, 0.0],
                           np.float32)
    W[1, :] = 0.25                                                          # constant
    W[2, :] = np.linspace(0.5, 1.0, 256, dtype=np.float32)                  # all positive
    W[3, :] = -np.linspace(0.5, 1.0, 256, dtype=np.float32)                 # all negative
    W[4, ::2] = 0.0
    W[4, 1::2] = -0.0                                                       # signed zeros
    W[5, :] = np.float32(1e-30) * np.arange(256, dtype=np.float32)          # tiny range: subnormal-ish scale
    _pack_and_compare(g, orc, W, np.arange(6, dtype=np.uint8) + 3)


def test_full_size_sampled_rows(g, orc):
    # the largest config-1 shape at full size; rows are checked on a seeded sample
    K, N = 4096, 14336
    W = wl.weights_gaussian(K, N, key=(1, 0, 4, 0))
    p = g.pack(torch.from_numpy(W).cuda())
    codes = g.unpack_codes(p).cpu().numpy()
    ms, mz = meta_split(p)
    rows = np.sort(np.random.default_rng(1).choice(K, 48, replace=False))
    rows[-1] = K - 1
    q, s, z = orc.rtn_quantize(W[rows])
    assert np.array_equal(codes[rows], q)
    assert np.array_equal(ms[rows], s) and np.array_equal(mz[rows], z)
