"""Seeded synthetic inputs for the graded bit-plane VMM.

This module only draws random numbers; it holds none of the method's arithmetic,
so that the CUDA path and the fp64 oracle can both be fed from it without sharing
any of the computation they are compared on.

Every draw comes from numpy's PCG64 seeded by a SeedSequence built from an
explicit key tuple, e.g. (config, layer, linear, stream, index), so a value is
reproducible from its key alone.

The shapes mirror the paper's evaluation models (Llama3-8B and Qwen3-8B decode
linears, "GRINQH" Section 4) and the isolated-kernel matrix of Section 4
"Setup for Kernel Benchmarking" (16384 x 4096). Trained weights and text corpora
are not used: weights and activations are synthetic with the distributions below.
"""
from __future__ import annotations

import numpy as np

# Class set used for every configuration: widths 0 (skip), 2, 3, 4 and 8 bits.
CLASSES = (0, 2, 3, 4, 8)

# (name, K inputs, N outputs) of one decoder layer's linears.
LLAMA3_8B = (
    ("q_proj", 4096, 4096),
    ("k_proj", 4096, 1024),
    ("v_proj", 4096, 1024),
    ("o_proj", 4096, 4096),
    ("gate_proj", 4096, 14336),
    ("up_proj", 4096, 14336),
    ("down_proj", 14336, 4096),
)
QWEN3_8B = (
    ("q_proj", 4096, 4096),
    ("k_proj", 4096, 1024),
    ("v_proj", 4096, 1024),
    ("o_proj", 4096, 4096),
    ("gate_proj", 4096, 12288),
    ("up_proj", 4096, 12288),
    ("down_proj", 12288, 4096),
)
# Which linears read the same input vector inside one decoder layer.
SHARED_INPUT = {"q_proj": "attn_in", "k_proj": "attn_in", "v_proj": "attn_in",
                "o_proj": "attn_out", "gate_proj": "mlp_in", "up_proj": "mlp_in",
                "down_proj": "mlp_mid"}


def rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def f16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE binary16 bit patterns (numpy's conversion, round to nearest even)."""
    return np.asarray(a, np.float32).astype(np.float16).view(np.uint16)


def weights_gaussian(K: int, N: int, key, std: float = 0.02) -> np.ndarray:
    """W ~ N(0, std^2), fp32, shape [K, N] (row k = input channel k)."""
    return (rng(*key).standard_normal((K, N), dtype=np.float32) * np.float32(std)).astype(np.float32)


def weights_rowstd_loguniform(K: int, N: int, key, lo: float = 0.005, hi: float = 0.05) -> np.ndarray:
    """W[k, :] ~ N(0, sigma_k^2) with sigma_k log-uniform in [lo, hi] per input row k."""
    g = rng(*key)
    sig = np.exp(g.uniform(np.log(lo), np.log(hi), size=(K, 1))).astype(np.float32)
    return (g.standard_normal((K, N), dtype=np.float32) * sig).astype(np.float32)


def outlier_channels(K: int, key, frac: float = 0.01) -> np.ndarray:
    """A fixed, seeded set of round(frac*K) channel indices (sorted)."""
    m = int(round(frac * K))
    return np.sort(rng(*key, 0x0071).choice(K, size=m, replace=False))


def activations_outlier(K: int, count: int, key, chan_key=None, frac: float = 0.01,
                        factor: float = 20.0) -> np.ndarray:
    """x ~ N(0,1) with a fixed 1% of channels scaled by `factor`, rounded to fp16.

    Returns uint16 bit patterns, shape [count, K]. `chan_key` fixes the outlier
    channels (one set per layer input, shared by its calibration and test draws)."""
    g = rng(*key)
    x = g.standard_normal((count, K), dtype=np.float32)
    ch = outlier_channels(K, chan_key if chan_key is not None else key, frac)
    x[:, ch] *= np.float32(factor)
    return f16_bits(x)


def activations_student_t(K: int, count: int, key, nu: float = 3.0) -> np.ndarray:
    """Student-t(nu) samples clamped to the fp16 range, rounded to fp16 (uint16 bits)."""
    x = rng(*key).standard_t(nu, size=(count, K)).astype(np.float32)
    x = np.clip(x, -65504.0, 65504.0)
    return f16_bits(x)


def activations_silu_gated(K: int, count: int, key) -> np.ndarray:
    """SiLU(a) * b with a, b ~ N(0,1), in fp32, rounded to fp16 (uint16 bits)."""
    g = rng(*key)
    a = g.standard_normal((count, K), dtype=np.float32)
    b = g.standard_normal((count, K), dtype=np.float32)
    x = (a / (np.float32(1.0) + np.exp(-a))) * b
    return f16_bits(x.astype(np.float32))


def activations_gaussian(K: int, count: int, key) -> np.ndarray:
    return f16_bits(rng(*key).standard_normal((count, K), dtype=np.float32))
