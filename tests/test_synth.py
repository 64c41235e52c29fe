"""The seeded input generator: determinism, stated distributions, bf16 rounding."""
import numpy as np

from sparsity_step_b200 import synth


def test_deterministic_and_seed_dependent():
    a = synth.latent_weight(3, 16, 64)
    b = synth.latent_weight(3, 16, 64)
    c = synth.latent_weight(4, 16, 64)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    # chunking does not change the stream
    n = synth._CHUNK + 17
    full = synth.normal_f64(9, n)
    assert np.array_equal(full[-17:], synth.normal_f64(9, n)[-17:])


def test_splitmix64_known_value():
    # splitmix64 with state 0: first output of the published generator
    z = synth.splitmix64(0, 0, 0, 1)
    assert int(z[0]) == 0xE220A8397B1DCDAF


def test_normal_moments_and_outliers():
    v = synth.normal_f64(1, 1 << 20, std=0.02)
    assert abs(v.mean()) < 1e-4 and abs(v.std() - 0.02) < 1e-4
    f = synth.outlier_factor(1, 1 << 20)
    assert abs((f == 20).mean() - 0.01) < 5e-4


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.3], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    back = synth.bf16_bits_to_f32(bits)
    assert back[0] == 1.0                    # tie -> even mantissa
    assert back[1] == 1.0 + 4 * 2 ** -8      # tie -> even mantissa (up)
    assert back[2] == np.float32(-0.30078125)
