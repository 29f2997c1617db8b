"""The synthetic input recipe: draws are reproducible from their key alone, the
layer shapes are the Llama3-8B and Qwen3-8B decode linears, a fixed round(0.01 K)
channels of each layer input are scaled by exactly 20 before the one rounding to
binary16, Student-t draws are clamped to the binary16 range, and the weight
distributions have the stated spreads."""
import numpy as np

from activation_graded_bit_b200 import workloads as wl


def test_draws_depend_on_the_key_only():
    a = wl.weights_gaussian(64, 96, key=(1, 2, 3))
    b = wl.weights_gaussian(64, 96, key=(1, 2, 3))
    c = wl.weights_gaussian(64, 96, key=(1, 2, 4))
    assert a.dtype == np.float32 and np.array_equal(a, b) and not np.array_equal(a, c)
    x1 = wl.activations_outlier(300, 4, key=(5,), chan_key=(6,))
    x2 = wl.activations_outlier(300, 4, key=(5,), chan_key=(6,))
    assert x1.dtype == np.uint16 and x1.shape == (4, 300) and np.array_equal(x1, x2)


def test_layer_shapes():
    assert dict((n, (k, m)) for n, k, m in wl.LLAMA3_8B) == {
        "q_proj": (4096, 4096), "k_proj": (4096, 1024), "v_proj": (4096, 1024), "o_proj": (4096, 4096),
        "gate_proj": (4096, 14336), "up_proj": (4096, 14336), "down_proj": (14336, 4096)}
    assert dict((n, (k, m)) for n, k, m in wl.QWEN3_8B)["down_proj"] == (12288, 4096)
    assert wl.CLASSES == (0, 2, 3, 4, 8)


def test_outlier_channels_are_fixed_and_scaled_by_20():
    K = 4096
    ch = wl.outlier_channels(K, (7,))
    assert len(ch) == round(0.01 * K) and len(set(ch.tolist())) == len(ch)
    assert np.array_equal(ch, wl.outlier_channels(K, (7,)))
    # the same draw without scaling: the scaled channels are exactly 20 x the base
    # values before the one rounding to binary16
    x = wl.activations_outlier(K, 3, key=(8,), chan_key=(7,)).view(np.float16)
    base = wl.rng(8).standard_normal((3, K), dtype=np.float32)
    ref = base.copy()
    ref[:, ch] *= np.float32(20.0)
    assert np.array_equal(x, ref.astype(np.float16))
    mask = np.zeros(K, bool)
    mask[ch] = True
    assert np.abs(x[:, mask].astype(np.float64)).mean() > 10 * np.abs(x[:, ~mask].astype(np.float64)).mean()


def test_student_t_is_clamped_to_binary16():
    x = wl.activations_student_t(20000, 4, key=(9,), nu=0.3).view(np.float16)   # very heavy tails
    assert np.all(np.isfinite(x))
    assert np.abs(x.astype(np.float64)).max() <= 65504.0


def test_weight_spreads():
    W = wl.weights_gaussian(512, 512, key=(10,))
    assert abs(float(W.std()) - 0.02) < 0.0005
    V = wl.weights_rowstd_loguniform(2000, 400, key=(11,))
    s = V.std(axis=1)
    assert s.min() > 0.004 and s.max() < 0.056
    # log-uniform: the median row spread sits near the geometric mean of the range
    assert abs(np.log(np.median(s)) - 0.5 * (np.log(0.005) + np.log(0.05))) < 0.15
