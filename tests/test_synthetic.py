"""The seeded input generator: reproducible, sliceable, with the stated moments."""
import numpy as np

import synthetic as syn


def test_slices_match_whole_tensor():
    full = syn.normal_bf16(7, syn.TENSOR_X, 300, 33)
    part = syn.normal_bf16(7, syn.TENSOR_X, 300, 33, row_begin=123, n_rows=50, threads=3)
    np.testing.assert_array_equal(part, full[123:173])
    again = syn.normal_bf16(7, syn.TENSOR_X, 300, 33, threads=5)
    np.testing.assert_array_equal(again, full)


def test_streams_differ_by_seed_and_tensor():
    a = syn.normal_bf16(0, 0, 4, 64)
    assert not np.array_equal(a, syn.normal_bf16(1, 0, 4, 64))
    assert not np.array_equal(a, syn.normal_bf16(0, 1, 4, 64))


def test_moments_and_scaling():
    v = syn.bf16_bits_to_f64(syn.normal_bf16(3, 2, 2000, 500, sigma=0.25))
    assert abs(v.mean()) < 0.002
    assert abs(v.std() - 0.25) < 0.002
    # 4th moment of a Gaussian is 3 sigma^4
    assert abs(np.mean(v ** 4) / 0.25 ** 4 - 3.0) < 0.05
    rows = syn.bf16_bits_to_f64(syn.normal_bf16(3, 0, 64, 2048, unit_rms_rows=True))
    np.testing.assert_allclose(np.sqrt(np.mean(rows ** 2, axis=1)), 1.0, atol=2e-3)


def test_first_draws_follow_the_published_definitions():
    # SplitMix64 of (key + GAMMA), uniform in (0, 1], Box-Muller cos/sin branch
    M64 = (1 << 64) - 1
    G = 0x9E3779B97F4A7C15

    def mix(z):
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        return z ^ (z >> 31)

    seed, tid = 5, 1
    key = mix(mix(seed) ^ (((tid + 1) * G) & M64))
    u = [((mix((key + (i + 1) * G) & M64) >> 11) + 1) * 2.0 ** -53 for i in range(4)]
    rho0 = np.sqrt(-2 * np.log(u[0]))
    rho1 = np.sqrt(-2 * np.log(u[2]))
    expect = [rho0 * np.cos(2 * np.pi * u[1]), rho0 * np.sin(2 * np.pi * u[1]),
              rho1 * np.cos(2 * np.pi * u[3]), rho1 * np.sin(2 * np.pi * u[3])]
    got = [syn.normal_at(seed, tid, j) for j in range(4)]
    np.testing.assert_allclose(got, expect, rtol=1e-14, atol=1e-14)


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0 - 2 ** -7, 3.0e-3], dtype=np.float32)
    bits = syn.f32_to_bf16_bits(f)
    back = syn.bf16_bits_to_f64(bits)
    # ties go to the even mantissa; others to the nearest representable value
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2 ** -6
    assert back[3] == -2.0
    assert abs(back[4] - 3.0e-3) <= 3.0e-3 * 2 ** -8
