"""Thin ctypes binding over libgrinqh.so (the C ABI in include/grinqh.h).

Argument marshalling only: every step of the graded VMM runs in the library's
CUDA kernels. torch is used for device memory and streams: tensors are passed as
raw device pointers and the current torch stream as the cudaStream_t. There is
no fallback: if the shared library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgrinqh.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libgrinqh.so is not built (expected at %s); run `python -m activation_graded_bit_b200.build` "
        "or __graft_entry__.build()" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "misaligned pointer", 3: "unsupported",
          4: "workspace missing or too small", 5: "CUDA error"}


class GrinqhError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s failed: %s (%d)" % (where, STATUS.get(code, "?"), code))
        self.code = code


class Layout(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("tile_n", ctypes.c_int32), ("n_tiles", ctypes.c_int32), ("record_bytes", ctypes.c_int32),
                ("b_max", ctypes.c_int32), ("reserved", ctypes.c_int32), ("packed_bytes", ctypes.c_int64)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_LP = ctypes.POINTER(Layout)


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_version = _sig("grinqh_version", [], ctypes.c_char_p)
_status_string = _sig("grinqh_status_string", [ctypes.c_int], ctypes.c_char_p)
_layout_init = _sig("grinqh_layout_init", [_I, _I, _LP])
_layout_init_bmax = _sig("grinqh_layout_init_bmax", [_I, _I, _I, _LP])
_pack = _sig("grinqh_pack", [_LP, _P, _P, _P])
_unpack = _sig("grinqh_unpack_codes", [_LP, _P, _P, _P, _P])
_maxent = _sig("grinqh_maxent_distribution", [_P, _I, ctypes.c_double, _P])
_cal_ws = _sig("grinqh_calibrate_workspace_bytes", [_I, _I, ctypes.POINTER(ctypes.c_size_t)])
_calibrate = _sig("grinqh_calibrate", [_P, _I, _I, _P, _I, _P, ctypes.c_double, _P, _P, ctypes.c_size_t, _P])
_select = _sig("grinqh_select", [_P, _I, _P, _P, _I, _P, _P, _P, _P])
_vmm_ws = _sig("grinqh_vmm_workspace_bytes", [_LP, ctypes.POINTER(ctypes.c_size_t)])
_vmm = _sig("grinqh_vmm", [_LP, _P, _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P])
_vmm_noalloc = _sig("grinqh_vmm_noalloc", [_LP, _P, _P, _P, _P, _P, _I, _P, _P])
_select_vmm = _sig("grinqh_select_vmm", [_LP, _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P])
_batch_ws = _sig("grinqh_vmm_batch_workspace_bytes", [_LP, _I, ctypes.POINTER(ctypes.c_size_t)])
_select_vmm_batch = _sig("grinqh_select_vmm_batch", [_LP, _P, _P, _I, _P, _P, _I, _P, _P, ctypes.c_size_t, _P])
_dequant = _sig("grinqh_dequant", [_LP, _P, _P, _P])
_prefill = _sig("grinqh_prefill", [_LP, _P, _P, _I, _P, _P, _P])
_prefill_tc = _sig("grinqh_prefill_tc", [_LP, _P, _P, _I, _P, _P, _P])
_select_vmm_batch_tc = _sig("grinqh_select_vmm_batch_tc", [_LP, _P, _P, _I, _P, _P, _I, _P, _P, _P])
_pack_codes = _sig("grinqh_pack_codes", [_LP, _P, _P, _P])
_lut_build = _sig("grinqh_lut_build", [_P, _I, _I, _I, _P, _P])
_lut_bytes = _sig("grinqh_lut_bytes", [_LP, ctypes.POINTER(ctypes.c_size_t)])
_vmm_lut = _sig("grinqh_vmm_lut", [_LP, _P, _P, _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t, _P])

# Every exported symbol of the C ABI, for the export check in the tests.
EXPORTS = ("grinqh_version", "grinqh_status_string", "grinqh_layout_init", "grinqh_layout_init_bmax", "grinqh_pack",
           "grinqh_unpack_codes", "grinqh_maxent_distribution", "grinqh_calibrate_workspace_bytes",
           "grinqh_calibrate", "grinqh_select", "grinqh_vmm_workspace_bytes", "grinqh_vmm",
           "grinqh_vmm_noalloc", "grinqh_select_vmm", "grinqh_vmm_batch_workspace_bytes",
           "grinqh_select_vmm_batch", "grinqh_dequant", "grinqh_prefill", "grinqh_prefill_tc", "grinqh_select_vmm_batch_tc", "grinqh_pack_codes",
           "grinqh_lut_bytes", "grinqh_vmm_lut", "grinqh_lut_build")


def version() -> str:
    return _version().decode()


def _check(rc: int, where: str):
    if rc != OK:
        raise GrinqhError(rc, where)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _classes_buf(classes: Sequence[int]):
    arr = (ctypes.c_uint8 * len(classes))(*[int(c) for c in classes])
    return arr, len(classes)


def _need(t, count: int, esize: int, what: str):
    """The library reads or writes `count` elements of `esize` bytes at t's address;
    the C ABI sees only the pointer, so a smaller buffer or another element size is
    refused here, before anything is launched."""
    if t is None:
        return
    if t.element_size() != esize or t.numel() < count:
        raise ValueError("%s: needs %d elements of %d bytes, got %d of %d" % (
            what, count, esize, t.numel(), t.element_size()))


def _need_selection(sel, K: int, what: str):
    _need(sel.idx, K, 4, what + " idx")
    _need(sel.offsets, len(sel.classes) + 1, 4, what + " offsets")


def layout(K: int, N: int, b_max: int = 8) -> Layout:
    L = Layout()
    if b_max == 8:
        _check(_layout_init(int(K), int(N), ctypes.byref(L)), "grinqh_layout_init")
    else:
        _check(_layout_init_bmax(int(K), int(N), int(b_max), ctypes.byref(L)), "grinqh_layout_init_bmax")
    return L


@dataclass
class PackedLayer:
    """Bit-plane packed K x N layer: one uint8 buffer holding the planes of every
    (row, tile) record, then the scale/zero words of every record."""
    layout: Layout
    packed: torch.Tensor

    @property
    def K(self):
        return self.layout.K

    @property
    def N(self):
        return self.layout.N

    @property
    def b_max(self):
        return self.layout.b_max

    @property
    def meta_offset(self) -> int:
        """Byte offset of the scale/zero words: after the planes of every record."""
        L = self.layout
        return L.K * L.n_tiles * L.record_bytes

    def planes(self) -> torch.Tensor:
        """uint8 view [K, n_tiles, record_bytes] of every record's planes (plane pair s in bytes 256 s .. 256 s + 255)."""
        L = self.layout
        return self.packed[: self.meta_offset].view(L.K, L.n_tiles, L.record_bytes)

    def meta_bytes(self) -> torch.Tensor:
        """uint8 view [K, n_tiles, 32] of every record's scale/zero words."""
        L = self.layout
        return self.packed[self.meta_offset: self.meta_offset + L.K * L.n_tiles * 32].view(L.K, L.n_tiles, 32)

    def meta_words(self) -> torch.Tensor:
        """int32 copy [K, n_tiles, 8] of the scale | zero << 16 words of every record."""
        L = self.layout
        return self.meta_bytes().contiguous().view(torch.int32).view(L.K, L.n_tiles, 8)


def empty_packed(K: int, N: int, device="cuda", b_max: int = 8) -> PackedLayer:
    L = layout(K, N, b_max)
    return PackedLayer(L, torch.empty(int(L.packed_bytes), dtype=torch.uint8, device=device))


def pack(W: torch.Tensor, out: Optional[PackedLayer] = None, stream=None, b_max: int = 8) -> PackedLayer:
    """grinqh_pack: W is a contiguous fp32 [K, N] CUDA tensor; codes of b_max bits
    (out, when given, fixes b_max through its layout)."""
    assert W.dtype == torch.float32 and W.is_cuda and W.is_contiguous() and W.dim() == 2
    K, N = W.shape
    p = out if out is not None else empty_packed(K, N, W.device, b_max)
    _need(W, p.K * p.N, 4, "grinqh_pack W")
    _check(_pack(ctypes.byref(p.layout), _ptr(W), _ptr(p.packed), _stream(stream)), "grinqh_pack")
    return p


def unpack_codes(p: PackedLayer, bits: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    codes = torch.empty((p.K, p.N), dtype=torch.uint8, device=p.packed.device)
    _check(_unpack(ctypes.byref(p.layout), _ptr(p.packed), _ptr(bits), _ptr(codes), _stream(stream)),
           "grinqh_unpack_codes")
    return codes


def maxent_distribution(classes: Sequence[int], target_bits: float):
    cb, n = _classes_buf(classes)
    P = (ctypes.c_double * n)()
    _check(_maxent(ctypes.addressof(cb), n, float(target_bits), ctypes.addressof(P)), "grinqh_maxent_distribution")
    return [P[i] for i in range(n)]


def calibrate_workspace_bytes(S: int, n_classes: int) -> int:
    v = ctypes.c_size_t()
    _check(_cal_ws(int(S), int(n_classes), ctypes.byref(v)), "grinqh_calibrate_workspace_bytes")
    return v.value


def calibrate(X: torch.Tensor, classes: Sequence[int], P: Optional[Sequence[float]] = None,
              target_bits: float = 0.0, out: Optional[torch.Tensor] = None,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_calibrate: X is a [S, K] CUDA tensor of fp16 (or its int16/uint16 bit view)."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.element_size() == 2
    S, K = X.shape
    cb, n = _classes_buf(classes)
    th = out if out is not None else torch.empty(max(n - 1, 1), dtype=torch.float32, device=X.device)
    _need(th, n - 1, 4, "grinqh_calibrate thresholds")
    if P is not None and len(P) != n:
        raise ValueError("grinqh_calibrate: P has %d entries for %d classes" % (len(P), n))
    ws_bytes = calibrate_workspace_bytes(S, n)
    ws = workspace if workspace is not None else torch.empty(ws_bytes, dtype=torch.uint8, device=X.device)
    Pbuf = None
    if P is not None:
        Pbuf = (ctypes.c_double * n)(*[float(v) for v in P])
    _check(_calibrate(_ptr(X), S, K, ctypes.addressof(cb), n,
                      ctypes.addressof(Pbuf) if Pbuf is not None else None, float(target_bits),
                      _ptr(th), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "grinqh_calibrate")
    return th[: n - 1]


@dataclass
class Selection:
    bits: torch.Tensor      # uint8 [K]
    idx: torch.Tensor       # int32 [K]
    offsets: torch.Tensor   # int32 [n_classes + 1]
    classes: tuple


def empty_selection(K: int, classes: Sequence[int], device="cuda") -> Selection:
    return Selection(torch.empty(K, dtype=torch.uint8, device=device),
                     torch.empty(K, dtype=torch.int32, device=device),
                     torch.empty(len(classes) + 1, dtype=torch.int32, device=device), tuple(classes))


def select(x: torch.Tensor, thresholds: torch.Tensor, classes: Sequence[int],
           out: Optional[Selection] = None, stream=None) -> Selection:
    """grinqh_select: x is a [K] CUDA tensor of fp16 (or its 16-bit bit view)."""
    assert x.is_cuda and x.dim() == 1 and x.is_contiguous() and x.element_size() == 2
    K = x.shape[0]
    sel = out if out is not None else empty_selection(K, classes, x.device)
    cb, n = _classes_buf(classes)
    _need(thresholds, n - 1, 4, "grinqh_select thresholds")
    _need(sel.bits, K, 1, "grinqh_select bits")
    _need(sel.idx, K, 4, "grinqh_select idx")
    _need(sel.offsets, n + 1, 4, "grinqh_select offsets")
    _check(_select(_ptr(x), K, _ptr(thresholds), ctypes.addressof(cb), n, _ptr(sel.bits), _ptr(sel.idx),
                   _ptr(sel.offsets), _stream(stream)), "grinqh_select")
    return sel


def vmm_workspace_bytes(L: Layout) -> int:
    v = ctypes.c_size_t()
    _check(_vmm_ws(ctypes.byref(L), ctypes.byref(v)), "grinqh_vmm_workspace_bytes")
    return v.value


def vmm_workspace(L: Layout, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for grinqh_vmm (reusable across calls on one stream)."""
    return torch.zeros(vmm_workspace_bytes(L), dtype=torch.uint8, device=device)


def vmm(p: PackedLayer, x: torch.Tensor, sel: Selection, workspace: torch.Tensor,
        y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_vmm: y[N] fp32 = x . W_hat over the graded bit planes."""
    if y is None:
        y = torch.empty(p.N, dtype=torch.float32, device=p.packed.device)
    _need(x, p.K, 2, "grinqh_vmm x")
    _need(y, p.N, 4, "grinqh_vmm y")
    _need_selection(sel, p.K, "grinqh_vmm")
    cb, n = _classes_buf(sel.classes)
    _check(_vmm(ctypes.byref(p.layout), _ptr(p.packed), _ptr(x), _ptr(sel.idx), _ptr(sel.offsets),
                ctypes.addressof(cb), n, _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                _stream(stream)), "grinqh_vmm")
    return y


def select_vmm(p: PackedLayer, x: torch.Tensor, thresholds: Optional[torch.Tensor], classes: Sequence[int],
               workspace: torch.Tensor, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_select_vmm: grading and the graded product in one call (K <= 16384)."""
    if y is None:
        y = torch.empty(p.N, dtype=torch.float32, device=p.packed.device)
    cb, n = _classes_buf(classes)
    _need(x, p.K, 2, "grinqh_select_vmm x")
    _need(y, p.N, 4, "grinqh_select_vmm y")
    _need(thresholds, n - 1, 4, "grinqh_select_vmm thresholds")
    _check(_select_vmm(ctypes.byref(p.layout), _ptr(p.packed), _ptr(x), _ptr(thresholds), ctypes.addressof(cb), n,
                       _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "grinqh_select_vmm")
    return y


def vmm_batch_workspace(L: Layout, tokens: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for grinqh_select_vmm_batch with this many tokens."""
    v = ctypes.c_size_t()
    _check(_batch_ws(ctypes.byref(L), int(tokens), ctypes.byref(v)), "grinqh_vmm_batch_workspace_bytes")
    return torch.zeros(v.value, dtype=torch.uint8, device=device)


def select_vmm_batch(p: PackedLayer, X: torch.Tensor, thresholds: Optional[torch.Tensor], classes: Sequence[int],
                     workspace: torch.Tensor, Y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_select_vmm_batch: X is a contiguous [T, K] CUDA tensor of fp16 (or its
    16-bit bit view); returns Y fp32 [T, N], row t as grinqh_select_vmm gives for X[t]."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.element_size() == 2 and X.shape[1] == p.K
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, p.N), dtype=torch.float32, device=X.device)
    cb, n = _classes_buf(classes)
    _need(Y, T * p.N, 4, "grinqh_select_vmm_batch Y")
    _need(thresholds, n - 1, 4, "grinqh_select_vmm_batch thresholds")
    _check(_select_vmm_batch(ctypes.byref(p.layout), _ptr(p.packed), _ptr(X), T, _ptr(thresholds),
                             ctypes.addressof(cb), n, _ptr(Y), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)),
           "grinqh_select_vmm_batch")
    return Y


def select_vmm_batch_tc(p: PackedLayer, X: torch.Tensor, thresholds: Optional[torch.Tensor],
                        classes: Sequence[int], status: torch.Tensor, Y: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """grinqh_select_vmm_batch_tc: the batched graded product on the tensor cores; X is a
    contiguous [T, K] CUDA tensor of fp16 (or its bit view), status a zero-filled
    16-byte CUDA tensor; returns Y fp32 [T, N]."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.element_size() == 2 and X.shape[1] == p.K
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, p.N), dtype=torch.float32, device=X.device)
    cb, n = _classes_buf(classes)
    _need(Y, T * p.N, 4, "grinqh_select_vmm_batch_tc Y")
    _need(thresholds, n - 1, 4, "grinqh_select_vmm_batch_tc thresholds")
    _need(status, 4, 4, "grinqh_select_vmm_batch_tc status")
    _check(_select_vmm_batch_tc(ctypes.byref(p.layout), _ptr(p.packed), _ptr(X), T, _ptr(thresholds),
                                ctypes.addressof(cb), n, _ptr(Y), _ptr(status), _stream(stream)),
           "grinqh_select_vmm_batch_tc")
    return Y


def dequant(p: PackedLayer, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_dequant: full-width w_hat as binary16 [K, N] (returned as float16)."""
    W16 = out if out is not None else torch.empty((p.K, p.N), dtype=torch.float16, device=p.packed.device)
    _need(W16, p.K * p.N, 2, "grinqh_dequant W16")
    _check(_dequant(ctypes.byref(p.layout), _ptr(p.packed), _ptr(W16), _stream(stream)), "grinqh_dequant")
    return W16


def prefill(p: PackedLayer, X: torch.Tensor, Y: Optional[torch.Tensor] = None, W16: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """grinqh_prefill: Y fp32 [T, N] = X [T, K] (fp16 or its bit view) . w_hat at full width."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.element_size() == 2 and X.shape[1] == p.K
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, p.N), dtype=torch.float32, device=X.device)
    if W16 is None:
        W16 = torch.empty((p.K, p.N), dtype=torch.float16, device=X.device)
    _need(Y, T * p.N, 4, "grinqh_prefill Y")
    _need(W16, p.K * p.N, 2, "grinqh_prefill W16")
    _check(_prefill(ctypes.byref(p.layout), _ptr(p.packed), _ptr(X), T, _ptr(Y), _ptr(W16), _stream(stream)),
           "grinqh_prefill")
    return Y


def prefill_tc(p: PackedLayer, X: torch.Tensor, status: torch.Tensor, Y: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """grinqh_prefill_tc: Y fp32 [T, N] = X [T, K] (fp16 or its bit view) . w_hat at full
    width, fused on the tensor cores; status is a zero-filled 16-byte CUDA tensor."""
    assert X.is_cuda and X.dim() == 2 and X.is_contiguous() and X.element_size() == 2 and X.shape[1] == p.K
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, p.N), dtype=torch.float32, device=X.device)
    _need(Y, T * p.N, 4, "grinqh_prefill_tc Y")
    _need(status, 4, 4, "grinqh_prefill_tc status")
    _check(_prefill_tc(ctypes.byref(p.layout), _ptr(p.packed), _ptr(X), T, _ptr(Y), _ptr(status), _stream(stream)),
           "grinqh_prefill_tc")
    return Y


def vmm_noalloc(p: PackedLayer, x: torch.Tensor, sel: Selection, y: torch.Tensor, stream=None) -> torch.Tensor:
    """grinqh_vmm_noalloc: as vmm, with the library's shared static scratch instead of a
    workspace; y (fp32 [N] CUDA tensor) must be given, since this call allocates nothing."""
    _need(x, p.K, 2, "grinqh_vmm_noalloc x")
    _need(y, p.N, 4, "grinqh_vmm_noalloc y")
    _need_selection(sel, p.K, "grinqh_vmm_noalloc")
    cb, n = _classes_buf(sel.classes)
    _check(_vmm_noalloc(ctypes.byref(p.layout), _ptr(p.packed), _ptr(x), _ptr(sel.idx), _ptr(sel.offsets),
                        ctypes.addressof(cb), n, _ptr(y), _stream(stream)), "grinqh_vmm_noalloc")
    return y

def pack_codes(codes: torch.Tensor, b_max: int = 8, out: Optional[PackedLayer] = None, stream=None) -> PackedLayer:
    """grinqh_pack_codes: bit planes of given b_max-bit codes (uint8 [K, N] CUDA
    tensor, e.g. nested look-up-table codes); the records' scale/zero words are zero."""
    assert codes.dtype == torch.uint8 and codes.is_cuda and codes.is_contiguous() and codes.dim() == 2
    K, N = codes.shape
    p = out if out is not None else empty_packed(K, N, codes.device, b_max)
    _need(codes, p.K * p.N, 1, "grinqh_pack_codes codes")
    _check(_pack_codes(ctypes.byref(p.layout), _ptr(codes), _ptr(p.packed), _stream(stream)), "grinqh_pack_codes")
    return p


def lut_bytes(L: Layout) -> int:
    """grinqh_lut_bytes: K * 2^(b_max+2) (binary16 tables in heap order per row)."""
    n = ctypes.c_size_t(0)
    _check(_lut_bytes(ctypes.byref(L), ctypes.byref(n)), "grinqh_lut_bytes")
    return n.value


def vmm_lut(p: PackedLayer, lut: torch.Tensor, x: torch.Tensor, sel: Selection, workspace: torch.Tensor,
            y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """grinqh_vmm_lut: y[N] fp32 = x . W_hat with w_hat[k][n] = lut[k][2^b_k + c_b]
    (lut: 16-bit [K, 2^(b_max+1)] CUDA tensor of binary16 bit patterns, heap order)."""
    assert lut.is_cuda and lut.is_contiguous() and lut.element_size() == 2
    assert lut.numel() * 2 == lut_bytes(p.layout), "table buffer size"
    if y is None:
        y = torch.empty(p.N, dtype=torch.float32, device=p.packed.device)
    _need(x, p.K, 2, "grinqh_vmm_lut x")
    _need(y, p.N, 4, "grinqh_vmm_lut y")
    _need_selection(sel, p.K, "grinqh_vmm_lut")
    cb, n = _classes_buf(sel.classes)
    _check(_vmm_lut(ctypes.byref(p.layout), _ptr(p.packed), _ptr(lut), _ptr(x), _ptr(sel.idx), _ptr(sel.offsets),
                    ctypes.addressof(cb), n, _ptr(y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                    _stream(stream)), "grinqh_vmm_lut")
    return y


def lut_build(W, b_max: int = 8):
    """grinqh_lut_build (host, offline): nested 2-means codes and binary16 tables of a
    fp32 [K, N] weight matrix (numpy array or CPU tensor). Returns CPU tensors
    (codes uint8 [K, N], tables int16 [K, 2^(b_max+1)] holding binary16 bit patterns)."""
    import numpy as np
    Wn = W.detach().cpu().numpy() if isinstance(W, torch.Tensor) else W
    Wn = np.ascontiguousarray(Wn, np.float32)
    assert Wn.ndim == 2
    K, N = Wn.shape
    codes = np.empty((K, N), np.uint8)
    lut = np.empty((K, 1 << (b_max + 1)), np.int16)
    _check(_lut_build(Wn.ctypes.data, K, N, b_max, codes.ctypes.data, lut.ctypes.data), "grinqh_lut_build")
    return torch.from_numpy(codes), torch.from_numpy(lut)
