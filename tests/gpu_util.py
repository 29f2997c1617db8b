"""Helpers for the GPU parity tests: canary-guarded device buffers, host<->device
conversion of fp16 bit patterns, and the parity tolerance.

Canaries stand in for a memory checker: every output buffer a test hands to the
library sits between two guard regions filled with a known byte pattern, and the
test checks after the call that the guards are untouched."""
import numpy as np
import torch

GUARD = 4096          # bytes on each side of a guarded buffer
PATTERN = 0xA5

# |y - y_ref| <= REL * sum_k |x_k w_hat_kn| + ABS, against the fp64 oracle
REL = 1e-4
ABS = 1e-6


class Guarded:
    """A device buffer of `count` elements of `dtype` with guard bytes around it."""

    def __init__(self, count, dtype, device="cuda"):
        esize = torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((2 * GUARD + count * esize,), PATTERN, dtype=torch.uint8, device=device)
        self.t = self.raw[GUARD:GUARD + count * esize].view(dtype)

    def check(self):
        head = self.raw[:GUARD]
        tail = self.raw[self.raw.numel() - GUARD:]
        assert bool((head == PATTERN).all()), "guard before the buffer was overwritten"
        assert bool((tail == PATTERN).all()), "guard after the buffer was overwritten"


def dev_u16(a):
    """numpy uint16 bit patterns -> CUDA int16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).cuda()


def host_u16(t):
    return t.cpu().numpy().view(np.uint16)


def assert_close(y_gpu, y_ref, bound, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    err = np.abs(y_gpu - y_ref)
    lim = REL * bound + ABS
    bad = np.nonzero(~(err <= lim))[0]
    assert bad.size == 0, "%s: %d of %d outside tolerance; first n=%d gpu=%r ref=%r bound=%r" % (
        what, bad.size, y_gpu.size, bad[0], y_gpu[bad[0]], y_ref[bad[0]], bound[bad[0]])
    return float((err / lim).max()) if err.size else 0.0


def meta_split(p):
    """PackedLayer -> (scale_bits, zero_bits) uint16 [K, n_groups] from the records' head words."""
    L = p.layout
    m = p.meta_words().cpu().numpy().view(np.uint32).reshape(L.K, L.n_tiles * 8)[:, :L.n_groups]
    return (m & 0xFFFF).astype(np.uint16), (m >> 16).astype(np.uint16)
