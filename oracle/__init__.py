"""ctypes wrapper around the fp64 CPU oracle (oracle/grinqh_oracle.cpp).

TEST INFRASTRUCTURE ONLY. The CUDA library and its Python binding never import,
load or call anything in this directory; only the tests, the package smoke check
and the benchmark's CPU-baseline leg do. Each function states the passage of
"GRINQH: Graded Input-based Quantization Hierarchy for Efficient LLM Generation"
(arXiv 2606.23419) that it follows; the C++ source carries the full statement.

All arrays are numpy arrays. fp16 values are carried as uint16 bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f64_to_f16.argtypes = [ctypes.c_double]
        L.orc_f64_to_f16.restype = ctypes.c_uint16
        L.orc_rtn_quantize.argtypes = [P, i32, i32, P, P, P]
        L.orc_rtn_quantize_bmax.argtypes = [P, i32, i32, i32, P, P, P]
        L.orc_code.argtypes = [i32, i32]
        L.orc_code_bmax.argtypes = [i32, i32, i32]
        L.orc_grade.argtypes = [P, i32, P, i32, P, P]
        L.orc_compact.argtypes = [P, i32, P, i32, P, P]
        L.orc_vmm.argtypes = [P, P, P, P, P, i32, i32, P, P, i32]
        L.orc_vmm_bmax.argtypes = [P, P, P, P, P, i32, i32, i32, P, P, i32]
        L.orc_dequant_f16.argtypes = [P, P, P, i32, i32, P]
        L.orc_maxent_distribution.argtypes = [P, i32, ctypes.c_double, P]
        L.orc_thresholds.argtypes = [P, i32, i32, P, i32, P]
        L.orc_lut_build.argtypes = [P, i32, i32, i32, P, P, P]
        L.orc_vmm_lut.argtypes = [P, P, P, P, i32, i32, i32, P, P, i32]
        for f in ("orc_lut_build", "orc_vmm_lut", "orc_rtn_quantize", "orc_rtn_quantize_bmax", "orc_code", "orc_code_bmax", "orc_grade",
                  "orc_compact", "orc_vmm", "orc_vmm_bmax", "orc_dequant_f16",
                  "orc_maxent_distribution", "orc_thresholds"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def f16_to_f64(h):
    """binary16 bit pattern -> float (IEEE 754 definition)."""
    return lib().orc_f16_to_f64(int(h))


def f64_to_f16(v):
    """float -> binary16 bit pattern, round to nearest even, straight from fp64."""
    return lib().orc_f64_to_f16(float(v))


def rtn_quantize(W, bmax=8):
    """b_max-bit asymmetric RTN per (row, 128-column group): Section 3.3 and Section 4.

    Returns (q uint8 [K,N], scale uint16 [K,n_g], zero uint16 [K,n_g])."""
    W = _c(W, np.float32)
    K, N = W.shape
    ng = (N + 127) // 128
    q = np.empty((K, N), np.uint8)
    s = np.empty((K, ng), np.uint16)
    z = np.empty((K, ng), np.uint16)
    if bmax == 8:
        rc = lib().orc_rtn_quantize(_p(W), K, N, _p(q), _p(s), _p(z))
    else:
        rc = lib().orc_rtn_quantize_bmax(_p(W), K, N, int(bmax), _p(q), _p(s), _p(z))
    if rc != 0:
        raise ValueError("bad sizes or b_max")
    return q, s, z


def code(q, b, bmax=8):
    """Nested reconstruction code of the b_max-bit code q at width b (Section 3.3); -1 for b = 0."""
    if bmax == 8:
        return lib().orc_code(int(q), int(b))
    return lib().orc_code_bmax(int(q), int(b), int(bmax))


def grade(x_bits, theta, classes):
    """Per-channel bit width from |x| against the thresholds (Section 3.1)."""
    x_bits = _c(x_bits, np.uint16)
    theta = _c(theta, np.float32)
    classes = _c(classes, np.uint8)
    assert len(classes) == len(theta) + 1
    bits = np.empty(len(x_bits), np.uint8)
    if lib().orc_grade(_p(x_bits), len(x_bits), _p(theta), len(theta), _p(classes), _p(bits)) != 0:
        raise ValueError("bad sizes")
    return bits


def compact(bits, classes):
    """Class-major, ascending-k channel lists and class offsets."""
    bits = _c(bits, np.uint8)
    classes = _c(classes, np.uint8)
    idx = np.empty(len(bits), np.int32)
    off = np.empty(len(classes) + 1, np.int32)
    rc = lib().orc_compact(_p(bits), len(bits), _p(classes), len(classes), _p(idx), _p(off))
    if rc != 0:
        raise ValueError("compact failed (%d)" % rc)
    return idx, off


def vmm(x_bits, q, scale, zero, bits, nthreads=1, bmax=8):
    """fp64 graded product y and the tolerance scale bound = sum |x_k * w_hat_kn|
    (codes q of b_max bits, Section 3.3)."""
    x_bits = _c(x_bits, np.uint16)
    q = _c(q, np.uint8)
    scale = _c(scale, np.uint16)
    zero = _c(zero, np.uint16)
    bits = _c(bits, np.uint8)
    K, N = q.shape
    y = np.empty(N, np.float64)
    bound = np.empty(N, np.float64)
    if bmax == 8:
        rc = lib().orc_vmm(_p(x_bits), _p(q), _p(scale), _p(zero), _p(bits), K, N, _p(y), _p(bound),
                           int(nthreads))
    else:
        rc = lib().orc_vmm_bmax(_p(x_bits), _p(q), _p(scale), _p(zero), _p(bits), K, N, int(bmax), _p(y),
                                _p(bound), int(nthreads))
    if rc != 0:
        raise ValueError("bad sizes")
    return y, bound


def maxent_distribution(classes, target):
    """Maximum-entropy P with mean width = target (Appendix A.1 eq. (1) reading)."""
    classes = _c(classes, np.uint8)
    P = np.empty(len(classes), np.float64)
    if lib().orc_maxent_distribution(_p(classes), len(classes), float(target), _p(P)) != 0:
        raise ValueError("target outside the class range or bad class set")
    return P


def thresholds(X_bits, P):
    """Percentile-mapped, sample-averaged thresholds (Section 3.2, Appendix A.1 eq. (2))."""
    X_bits = _c(X_bits, np.uint16)
    if X_bits.ndim == 1:
        X_bits = X_bits[None, :]
    P = _c(P, np.float64)
    S, K = X_bits.shape
    th = np.empty(len(P) - 1, np.float32)
    if lib().orc_thresholds(_p(X_bits), S, K, _p(P), len(P), _p(th)) != 0:
        raise ValueError("bad arguments")
    return th


def select(x_bits, theta, classes):
    """Grade + compaction in one call: (bits, idx, offsets)."""
    bits = grade(x_bits, theta, classes)
    idx, off = compact(bits, classes)
    return bits, idx, off


def dequant_f16(q, scale, zero):
    """Full-width weights rounded once to binary16, w_hat = s (q - z) (Section 4,
    prefill at b_max; Section 3.3): uint16 bit patterns [K, N]."""
    q = _c(q, np.uint8)
    scale = _c(scale, np.uint16)
    zero = _c(zero, np.uint16)
    K, N = q.shape
    out = np.empty((K, N), np.uint16)
    if lib().orc_dequant_f16(_p(q), _p(scale), _p(zero), K, N, _p(out)) != 0:
        raise ValueError("bad sizes")
    return out


def prefill(X_bits, w16):
    """Dense prefill product in fp64: Y[t, n] = sum_k x[t, k] * w16[k, n] over the
    binary16 operands (a library matmul on their exact fp64 values), and the
    tolerance scale bound[t, n] = sum_k |x[t, k] * w16[k, n]|."""
    Xf = np.ascontiguousarray(X_bits, np.uint16).view(np.float16).astype(np.float64)
    Wf = np.ascontiguousarray(w16, np.uint16).view(np.float16).astype(np.float64)
    return Xf @ Wf, np.abs(Xf) @ np.abs(Wf)


def lut_build(W, bmax=8):
    """Nested look-up-table codes by incremental upscaling (Section 3.3 on nested
    non-uniform codes; Section 4 and Appendix E.2 on any-precision LLM weights).
    Each cluster of width b-1 of a row is split by the optimal 1-D 2-means cut.

    Returns (q uint8 [K,N] codes of bmax bits, lut uint16 [K, 2^(bmax+1)] binary16
    centroids in heap order (width b, code c at 2^b + c), cent float64 [K, 2^(bmax+1)]
    the same centroids before rounding)."""
    W = _c(W, np.float32)
    K, N = W.shape
    E = 1 << (bmax + 1)
    q = np.empty((K, N), np.uint8)
    lut = np.empty((K, E), np.uint16)
    cent = np.empty((K, E), np.float64)
    if lib().orc_lut_build(_p(W), K, N, int(bmax), _p(q), _p(lut), _p(cent)) != 0:
        raise ValueError("bad sizes or b_max")
    return q, lut, cent


def vmm_lut(x_bits, q, lut, bits, bmax=8, nthreads=1):
    """fp64 graded product over nested table codes: w_hat = lut[k][2^b + (q >> (bmax - b))]
    for b = b_k > 0 (no midpoint, no scale or zero point), and bound = sum |x_k w_hat_kn|."""
    x_bits = _c(x_bits, np.uint16)
    q = _c(q, np.uint8)
    lut = _c(lut, np.uint16)
    bits = _c(bits, np.uint8)
    K, N = q.shape
    assert lut.shape == (K, 1 << (bmax + 1))
    y = np.empty(N, np.float64)
    bound = np.empty(N, np.float64)
    if lib().orc_vmm_lut(_p(x_bits), _p(q), _p(lut), _p(bits), K, N, int(bmax), _p(y), _p(bound),
                         int(nthreads)) != 0:
        raise ValueError("bad sizes or a width above b_max")
    return y, bound
