"""The seeded input generator: determinism, counter independence, distribution and bf16 rounding."""
import math

import numpy as np
from scipy import stats

import synth


def test_deterministic_and_counter_based():
    a = synth.normal(7, 3, (1000,))
    b = synth.normal(7, 3, (1000,))
    np.testing.assert_array_equal(a, b)
    tail = synth.normal(7, 3, (400,), offset=600)
    np.testing.assert_array_equal(a[600:], tail)
    assert not np.array_equal(a, synth.normal(7, 4, (1000,)))
    assert not np.array_equal(a, synth.normal(8, 3, (1000,)))


def test_normal_distribution():
    a = synth.normal(1, 1, (200000,), 0.0, 1.0).astype(np.float64)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    assert stats.kstest(a, "norm").pvalue > 1e-3
    s = synth.normal(1, 2, (100000,), 0.5, 0.02).astype(np.float64)
    assert abs(s.mean() - 0.5) < 1e-3 and abs(s.std() - 0.02) < 1e-3


def test_bf16_is_rne_of_f32():
    f = synth.normal(3, 5, (50000,))
    b = synth.normal(3, 5, (50000,), dtype="bf16")
    np.testing.assert_array_equal(b, synth.to_storage(f, "bf16"))
    back = synth.bf16_bits_to_f32(b)
    # RNE: error at most half an ulp of bf16 (2^-8 relative)
    assert np.all(np.abs(back - f) <= np.abs(f) * 2.0 ** -8 + 1e-30)
    # exact tie case: 1 + 2^-8 rounds to even (1.0); 1 + 3*2^-8 rounds up to 1 + 2^-7 * 2
    t = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8], np.float32)
    assert synth.bf16_bits_to_f32(synth.to_storage(t, "bf16")).tolist() == [1.0, 1 + 2 ** -6]


def test_config_recipes():
    c = synth.CONFIGS["skew"]
    bg = synth.as_f64(synth.make_bg(c), "bf16")
    assert bg[0] == 0.0 and bg[1] < 0 and np.all(np.diff(bg) <= 0)
    assert abs(bg[63] - 1.5 * math.log(1 / 64)) < 0.02
    tiny = synth.make_inputs(synth.CONFIGS["tiny"])
    assert tiny.x.dtype == np.float32 and tiny.W1.shape == (4, 64, 256) and tiny.W2.shape == (4, 256, 64)
    assert abs(tiny.W1.std() - 1 / 8) < 0.01 and abs(tiny.W2.std() - 1 / 16) < 0.01
