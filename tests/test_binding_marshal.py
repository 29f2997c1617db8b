"""Every call of the Python binding marshals its arguments into the C ABI and
turns a rejected call into GrinqhError. Runs without a GPU: stand-in tensors
carry plausible device addresses, and each call is given a layout or argument
that the library rejects on the host before anything could be launched."""
import ctypes
import os

import pytest
import torch


class FakeTensor:
    """The attributes the binding reads from a CUDA tensor; never dereferenced."""

    def __init__(self, shape, dtype, addr=0x10000):
        self.shape = tuple(shape)
        self.dtype = dtype
        self.is_cuda = True
        self.device = "cpu"
        self._addr = addr

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def element_size(self):
        return torch.empty(0, dtype=self.dtype).element_size()

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def data_ptr(self):
        return self._addr

    def view(self, *a):
        return self


class FakeStream:
    cuda_stream = 0


@pytest.fixture(scope="module")
def g():
    from activation_graded_bit_b200 import build
    build.build()
    from activation_graded_bit_b200 import grinqh
    return grinqh


def _bad_packed(g, K=64, N=1024):
    L = g.layout(K, N)
    L.tile_n = 512   # not a layout grinqh_layout_init makes: every call rejects it
    return g.PackedLayer(L, FakeTensor((int(L.packed_bytes),), torch.uint8))


def _expect_invalid(fn):
    from activation_graded_bit_b200 import grinqh
    with pytest.raises(grinqh.GrinqhError) as e:
        fn()
    assert e.value.code == 1


def test_every_call_marshals_and_reports(g):
    K, N, T = 64, 1024, 3
    cl = (0, 2, 3, 4, 8)
    st = FakeStream()
    p = _bad_packed(g, K, N)
    x = FakeTensor((K,), torch.int16)
    X = FakeTensor((T, K), torch.int16)
    th = FakeTensor((4,), torch.float32)
    y = FakeTensor((N,), torch.float32)
    Y = FakeTensor((T, N), torch.float32)
    ws = FakeTensor((1 << 20,), torch.uint8)
    sel = g.Selection(FakeTensor((K,), torch.uint8), FakeTensor((K,), torch.int32),
                      FakeTensor((len(cl) + 1,), torch.int32), cl)
    W = FakeTensor((K, N), torch.float32)
    W16 = FakeTensor((K, N), torch.float16)
    _expect_invalid(lambda: g.pack(W, out=p, stream=st))
    _expect_invalid(lambda: g.unpack_codes(p, stream=st))
    _expect_invalid(lambda: g.vmm(p, x, sel, ws, y=y, stream=st))
    _expect_invalid(lambda: g.select_vmm(p, x, th, cl, ws, y=y, stream=st))
    _expect_invalid(lambda: g.select_vmm_batch(p, X, th, cl, ws, Y=Y, stream=st))
    _expect_invalid(lambda: g.vmm_noalloc(p, x, sel, y, stream=st))
    _expect_invalid(lambda: g.dequant(p, out=W16, stream=st))
    _expect_invalid(lambda: g.prefill(p, X, Y=Y, W16=W16, stream=st))
    codes = FakeTensor((K, N), torch.uint8)
    lut = FakeTensor((K, 512), torch.int16)
    _expect_invalid(lambda: g.pack_codes(codes, out=p, stream=st))
    _expect_invalid(lambda: g.lut_bytes(p.layout))
    _expect_invalid(lambda: g.vmm_lut(p, lut, x, sel, ws, y=y, stream=st))
    # calls without a layout: invalid class sets
    _expect_invalid(lambda: g.select(x, th, (0, 4, 4), out=sel, stream=st))
    Xc = FakeTensor((8, K), torch.int16)
    _expect_invalid(lambda: g.calibrate(Xc, (0, 4, 4), target_bits=2.0, out=th, workspace=ws, stream=st))
    _expect_invalid(lambda: g.vmm_batch_workspace(g.layout(K, N), 0))


def test_short_or_mistyped_buffers_are_refused_before_the_call(g):
    # a valid layout: only the binding's size checks stand between these stand-in
    # buffers and the library, and each of them fails one
    K, N, T = 64, 1024, 3
    cl = (0, 2, 3, 4, 8)
    L = g.layout(K, N)
    p = g.PackedLayer(L, FakeTensor((int(L.packed_bytes),), torch.uint8))
    x = FakeTensor((K,), torch.int16)
    y = FakeTensor((N,), torch.float32)
    ws = FakeTensor((1 << 20,), torch.uint8)
    sel = g.Selection(FakeTensor((K,), torch.uint8), FakeTensor((K,), torch.int32),
                      FakeTensor((len(cl) + 1,), torch.int32), cl)
    short_sel = g.Selection(sel.bits, FakeTensor((K - 1,), torch.int32), sel.offsets, cl)
    th = FakeTensor((4,), torch.float32)
    cases = [
        lambda: g.vmm(p, FakeTensor((K - 1,), torch.int16), sel, ws, y=y),
        lambda: g.vmm(p, FakeTensor((K,), torch.float32), sel, ws, y=y),
        lambda: g.vmm(p, x, sel, ws, y=FakeTensor((N - 1,), torch.float32)),
        lambda: g.vmm(p, x, short_sel, ws, y=y),
        lambda: g.vmm_noalloc(p, x, sel, FakeTensor((N,), torch.float16)),
        lambda: g.select_vmm(p, x, FakeTensor((3,), torch.float32), cl, ws, y=y),
        lambda: g.select_vmm_batch(p, FakeTensor((T, K), torch.int16), th, cl, ws,
                                   Y=FakeTensor((T, N - 1), torch.float32)),
        lambda: g.dequant(p, out=FakeTensor((K, N - 1), torch.float16)),
        lambda: g.prefill(p, FakeTensor((T, K), torch.int16), Y=FakeTensor((T, N), torch.float32),
                          W16=FakeTensor((K - 1, N), torch.float16)),
        lambda: g.select(x, FakeTensor((2,), torch.float32), cl, out=sel),
        lambda: g.select(x, th, cl, out=short_sel),
        lambda: g.pack(FakeTensor((K, N - 1), torch.float32), out=p),
        lambda: g.pack_codes(FakeTensor((K, N - 1), torch.uint8), out=p),
        lambda: g.vmm_lut(p, FakeTensor((K, 512), torch.int16), x, short_sel, ws, y=y),
        lambda: g.calibrate(FakeTensor((8, K), torch.int16), cl, target_bits=3.0, out=FakeTensor((3,), torch.float32),
                            workspace=ws),
        lambda: g.calibrate(FakeTensor((8, K), torch.int16), cl, P=(0.5, 0.5), out=th, workspace=ws),
    ]
    for i, fn in enumerate(cases):
        with pytest.raises(ValueError):
            fn()


def test_binding_refuses_to_load_without_the_library(tmp_path):
    # a copy of the package without libgrinqh.so: importing the binding fails
    # loudly (no CPU or library fallback exists)
    import shutil
    import subprocess
    import sys
    src = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "activation_graded_bit_b200")
    dst = tmp_path / "activation_graded_bit_b200"
    dst.mkdir()
    for f in ("__init__.py", "grinqh.py", "workloads.py", "build.py"):
        shutil.copy(os.path.join(src, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import activation_graded_bit_b200.grinqh"], cwd=str(tmp_path),
                       capture_output=True, text=True, env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "libgrinqh.so is not built" in r.stderr
