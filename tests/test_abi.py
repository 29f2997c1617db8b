"""The C ABI library loads, exports every call include/grinqh.h declares, and
rejects bad arguments on the host before anything reaches a GPU. No test here
passes a pointer that could be launched on: every call fails validation first."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "include", "grinqh.h")


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import build
    build.build()
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _declared():
    txt = open(HDR).read()
    return sorted(set(re.findall(r"\b(grinqh_[a-z_]+)\s*\(", txt)))


def test_every_declared_symbol_is_exported(g):
    names = _declared()
    assert len(names) >= 11
    lib = ctypes.CDLL(g.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(g.EXPORTS) == names


def test_version_and_status_strings(g):
    assert "sm_100a" in g.version()
    for c in range(6):
        assert g._status_string(c).decode() == g.STATUS[c]


def test_layout(g):
    L = g.layout(4096, 14336)
    assert (L.K, L.N, L.n_groups, L.tile_n, L.n_tiles) == (4096, 14336, 112, 1024, 14)
    assert L.record_bytes == 8 * 128                      # the planes of one (row, tile) record
    assert L.packed_bytes == 4096 * 14 * (1024 + 32)       # planes, then 32 bytes of scale/zero per record
    L = g.layout(4, 4)
    assert (L.n_groups, L.n_tiles, L.record_bytes) == (1, 1, 1024)
    for K, N in ((0, 4), (4, 0), (-1, 5), (1 << 24 + 1, 1), (1 << 24, 1 << 24)):
        with pytest.raises(g.GrinqhError) as e:
            g.layout(K, N)
        assert e.value.code == 1


def test_maxent_matches_oracle(g, orc):
    for classes in ((0, 2, 3, 4, 8), (0, 2, 4, 6, 8), (1, 8), (3,)):
        lo, hi = classes[0], classes[-1]
        for t in np.linspace(lo, hi, 7):
            got = np.array(g.maxent_distribution(classes, t))
            ref = orc.maxent_distribution(np.array(classes, np.uint8), t)
            assert np.allclose(got, ref, rtol=0, atol=1e-12)
    with pytest.raises(g.GrinqhError):
        g.maxent_distribution((0, 2, 3, 4, 8), 8.5)
    with pytest.raises(g.GrinqhError):
        g.maxent_distribution((0, 3, 2), 2.0)
    with pytest.raises(g.GrinqhError):
        g.maxent_distribution((0, 2, 9), 2.0)


def _L(g, K, N):
    return ctypes.byref(g.layout(K, N))


def test_host_validation_rejects_before_launch(g):
    P = ctypes.c_void_p
    cl = (ctypes.c_uint8 * 5)(0, 2, 3, 4, 8)
    bad_cl = (ctypes.c_uint8 * 3)(0, 4, 4)
    ws = ctypes.c_size_t()
    # NULL layout / NULL pointers
    assert g._pack(None, P(0x1000), P(0x1000), None) == 1
    assert g._pack(_L(g, 8, 8), None, P(0x1000), None) == 1
    # layout that grinqh_layout_init would not produce
    L = g.layout(8, 8)
    L.tile_n = 512
    assert g._pack(ctypes.byref(L), P(0x1000), P(0x1000), None) == 1
    # misaligned packed buffer (alignment checked before launch)
    assert g._pack(_L(g, 8, 8), P(0x1000), P(0x1008), None) == 2
    # select: bad class sets, bad K, misaligned idx
    assert g._select(P(0x1000), 8, P(0x1000), ctypes.addressof(bad_cl), 3, P(0x1000), P(0x1000), P(0x1000), None) == 1
    assert g._select(P(0x1000), 8, P(0x1000), ctypes.addressof(cl), 10, P(0x1000), P(0x1000), P(0x1000), None) == 1
    assert g._select(P(0x1000), 0, P(0x1000), ctypes.addressof(cl), 5, P(0x1000), P(0x1000), P(0x1000), None) == 1
    # beyond 65536 channels the chunked count would read K^2/512 bytes: refused before any launch
    assert g._select(P(0x1000), 65537, P(0x1000), ctypes.addressof(cl), 5, P(0x1000), P(0x1000), P(0x1000), None) == 3
    assert g._select(P(0x1000), 8, P(0x1000), ctypes.addressof(cl), 5, P(0x1000), P(0x1002), P(0x1000), None) == 2
    assert g._select(None, 8, P(0x1000), ctypes.addressof(cl), 5, P(0x1000), P(0x1000), P(0x1000), None) == 1
    # vmm: workspace too small / missing, misaligned y
    L = g.layout(64, 1024)
    need = g.vmm_workspace_bytes(L)
    args = [ctypes.byref(L), P(0x1000), P(0x1000), P(0x1000), P(0x1000), ctypes.addressof(cl), 5, P(0x1000)]
    assert g._vmm(*args, None, need, None) == 4
    assert g._vmm(*args, P(0x1000), need - 1, None) == 4
    a2 = list(args)
    a2[7] = P(0x1002)                       # y not 4-byte aligned
    assert g._vmm(*a2, P(0x1000), need, None) == 2
    a3 = list(args)
    a3[3] = P(0x1002)                       # idx not 4-byte aligned
    assert g._vmm(*a3, P(0x1000), need, None) == 2
    a4 = list(args)
    a4[1] = P(0x1008)                       # packed not 16-byte aligned
    assert g._vmm(*a4, P(0x1000), need, None) == 2
    assert g._vmm(*args[:5], ctypes.addressof(bad_cl), 3, P(0x1000), P(0x1000), need, None) == 1
    # calibrate: bad P, missing workspace
    Pbad = (ctypes.c_double * 5)(0.5, 0.5, 0.5, 0.0, 0.0)
    assert g._calibrate(P(0x1000), 4, 16, ctypes.addressof(cl), 5, ctypes.addressof(Pbad), 0.0, P(0x1000),
                        P(0x1000), 1 << 20, None) == 1
    Pneg = (ctypes.c_double * 5)(-0.5, 0.5, 0.5, 0.5, 0.0)
    assert g._calibrate(P(0x1000), 4, 16, ctypes.addressof(cl), 5, ctypes.addressof(Pneg), 0.0, P(0x1000),
                        P(0x1000), 1 << 20, None) == 1
    assert g._calibrate(P(0x1000), 4, 16, ctypes.addressof(cl), 5, None, 9.0, P(0x1000), P(0x1000), 1 << 20,
                        None) == 1
    assert g._calibrate(P(0x1000), 4, 16, ctypes.addressof(cl), 5, None, 3.0, P(0x1000), None, 0, None) == 4
    assert g._calibrate(P(0x1000), 0, 16, ctypes.addressof(cl), 5, None, 3.0, P(0x1000), P(0x1000), 1 << 20,
                        None) == 1
    assert g._cal_ws(70000, 5, ctypes.byref(ws)) == 1
    assert g._cal_ws(128, 5, ctypes.byref(ws)) == 0 and ws.value >= 128 * 4 * 8


def test_layout_bmax(g):
    for bmax, rec in ((2, 256), (4, 512), (6, 768), (8, 1024)):
        L = g.layout(4096, 4096, bmax)
        assert (L.b_max, L.record_bytes, L.reserved) == (bmax, rec, 0)
        assert L.record_bytes == 128 * bmax and L.record_bytes % 128 == 0
        assert L.packed_bytes == 4096 * 4 * (rec + 32)
    assert g.layout(8, 8).b_max == 8
    for bad in (0, 1, 3, 5, 7, 9, 16, -2):
        with pytest.raises(g.GrinqhError) as e:
            g.layout(8, 8, bad)
        assert e.value.code == 1
    assert g._layout_init_bmax(8, 8, 4, None) == 1


def test_bmax_validation_rejects_before_launch(g):
    P = ctypes.c_void_p
    L = g.layout(64, 1024, 4)
    need = g.vmm_workspace_bytes(L)
    wide = (ctypes.c_uint8 * 4)(0, 2, 4, 6)      # a width above b_max = 4
    ok = (ctypes.c_uint8 * 3)(0, 2, 4)
    base = [ctypes.byref(L), P(0x1000), P(0x1000), P(0x1000), P(0x1000)]
    assert g._vmm(*base, ctypes.addressof(wide), 4, P(0x1000), P(0x1000), need, None) == 1
    assert g._vmm_noalloc(*base, ctypes.addressof(wide), 4, P(0x1000), None) == 1
    assert g._select_vmm(ctypes.byref(L), P(0x1000), P(0x1000), P(0x1000), ctypes.addressof(wide), 4, P(0x1000),
                         P(0x1000), need, None) == 1
    # the same call with classes that fit fails only on the workspace it lacks
    assert g._vmm(*base, ctypes.addressof(ok), 3, P(0x1000), None, need, None) == 4
    # a layout whose b_max field was edited is not one grinqh_layout_init_bmax makes
    L2 = g.layout(64, 1024, 4)
    L2.b_max = 6
    assert g._pack(ctypes.byref(L2), P(0x1000), P(0x1000), None) == 1
    L3 = g.layout(64, 1024, 4)
    L3.reserved = 1
    assert g._pack(ctypes.byref(L3), P(0x1000), P(0x1000), None) == 1


def test_batch_validation_rejects_before_launch(g):
    P = ctypes.c_void_p
    cl = (ctypes.c_uint8 * 5)(0, 2, 3, 4, 8)
    L = g.layout(64, 1024)
    ws = ctypes.c_size_t()
    assert g._batch_ws(ctypes.byref(L), 0, ctypes.byref(ws)) == 1
    assert g._batch_ws(ctypes.byref(L), 65536, ctypes.byref(ws)) == 1
    assert g._batch_ws(ctypes.byref(L), 3, ctypes.byref(ws)) == 0
    need3 = ws.value
    assert g._batch_ws(ctypes.byref(L), 1, ctypes.byref(ws)) == 0
    assert ws.value == g.vmm_workspace_bytes(L)
    assert need3 - 16 == 3 * (ws.value - 16)          # one set of partials per token
    base = [ctypes.byref(L), P(0x1000), P(0x1000)]
    rest = [P(0x1000), ctypes.addressof(cl), 5, P(0x1000)]
    assert g._select_vmm_batch(*base, 0, *rest, P(0x1000), need3, None) == 1            # no tokens
    assert g._select_vmm_batch(*base, 3, *rest, P(0x1000), need3 - 1, None) == 4        # workspace short
    assert g._select_vmm_batch(*base, 3, P(0x1000), ctypes.addressof(cl), 5, P(0x1002), P(0x1000), need3,
                               None) == 2                                                # Y misaligned
    Lbig = g.layout(20000, 64)
    assert g._select_vmm_batch(ctypes.byref(Lbig), P(0x1000), P(0x1000), 2, *rest, P(0x1000), 1 << 30,
                               None) == 3                                                # K above the fused limit


def test_prefill_validation_rejects_before_launch(g):
    P = ctypes.c_void_p
    L = g.layout(64, 1024)
    assert g._dequant(ctypes.byref(L), P(0x1000), None, None) == 1
    assert g._dequant(ctypes.byref(L), P(0x1000), P(0x1008), None) == 2        # W16 not 16-byte aligned
    assert g._prefill(ctypes.byref(L), P(0x1000), P(0x1000), 0, P(0x1000), P(0x1000), None) == 1   # T = 0
    assert g._prefill(ctypes.byref(L), P(0x1000), P(0x1001), 4, P(0x1000), P(0x1000), None) == 2  # X odd
    assert g._prefill(ctypes.byref(L), P(0x1000), P(0x1000), 4, P(0x1002), P(0x1000), None) == 2  # Y
    assert g._prefill(None, P(0x1000), P(0x1000), 4, P(0x1000), P(0x1000), None) == 1


def test_lut_validation_rejects_before_launch(g):
    P = ctypes.c_void_p
    cl = (ctypes.c_uint8 * 5)(0, 2, 3, 4, 8)
    cl6 = (ctypes.c_uint8 * 4)(0, 2, 4, 6)
    L = g.layout(64, 1024)
    L4 = g.layout(64, 1024, b_max=4)
    n = ctypes.c_size_t()
    assert g._lut_bytes(ctypes.byref(L), ctypes.byref(n)) == 0 and n.value == 64 * 1024
    assert g._lut_bytes(ctypes.byref(L4), ctypes.byref(n)) == 0 and n.value == 64 * 64
    assert g._lut_bytes(None, ctypes.byref(n)) == 1
    assert g._pack_codes(ctypes.byref(L), None, P(0x1000), None) == 1
    assert g._pack_codes(ctypes.byref(L), P(0x1001), P(0x1008), None) == 2     # packed not 16-byte aligned
    need = g.vmm_workspace_bytes(L)

    def vl(layout, lut=0x1000, x=0x1000, y=0x1000, classes=cl, nc=5, ws=0x1000, wsb=need):
        return g._vmm_lut(ctypes.byref(layout), P(0x1000), P(lut), P(x), P(0x1000), P(0x1000),
                          ctypes.addressof(classes), nc, P(y), P(ws), wsb, None)

    assert vl(L, lut=0) == 1                  # no tables
    assert vl(L, lut=0x1008) == 2             # tables not 16-byte aligned
    assert vl(L, x=0x1001) == 2
    assert vl(L, y=0x1002) == 2
    assert vl(L, wsb=need - 1) == 4
    assert vl(L4, classes=cl6, nc=4) == 1     # width 6 above b_max = 4
    Lbad = g.layout(64, 1024)
    Lbad.tile_n = 512
    assert vl(Lbad) == 1
