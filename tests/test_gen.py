"""The seeded input generator: distribution, determinism and bf16 rounding."""
import numpy as np
import torch

import gen


def test_moments_and_determinism():
    z = gen.normal_f32(0, 123, 0, 1_000_000)
    assert abs(float(z.mean())) < 3e-3 and abs(float(z.std()) - 1.0) < 3e-3
    np.testing.assert_array_equal(z[1000:2000], gen.normal_f32(0, 123, 1000, 1000))
    idx = np.array([5, 999_999, 17], np.uint64)
    np.testing.assert_array_equal(gen.normal_f32(0, 123, 0, 0, idx=idx), z[[5, 999_999, 17]])
    assert not np.array_equal(z[:100], gen.normal_f32(1, 123, 0, 100))
    assert not np.array_equal(z[:100], gen.normal_f32(0, 124, 0, 100))


def test_values_are_exact_multiples():
    s = gen.irwin_hall_sum(0, 7, np.arange(1000, dtype=np.uint64))
    assert s.min() >= 0 and s.max() <= 12 * 1023
    z = gen.normal_f32(0, 7, 0, 1000)
    np.testing.assert_array_equal(z.astype(np.float64) * 1024, (s - 6138).astype(np.float64))
    w = gen.normal_f32(0, 7, 0, 1000, 0.02)
    np.testing.assert_array_equal(w, z * np.float32(0.02))


def test_bf16_rounding_matches_torch():
    v = gen.normal_f32(0, 8, 0, 100_000, 3.7)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(gen.f32_to_bf16_bits(v), want)


def test_permutation():
    p = gen.permutation(0, gen.TID_PERM, 256)
    assert sorted(p.tolist()) == list(range(256))
    np.testing.assert_array_equal(p, gen.permutation(0, gen.TID_PERM, 256))


def test_host_c_twin_matches_numpy():
    for tid, sigma in [(1, 1.0), (17, 0.02), (gen.tid_expert(200, 2), 0.02)]:
        a = gen.normal_f32(3, tid, 12345, 50_000, sigma)
        b = gen.fill_f32(3, tid, 50_000, sigma, start=12345)
        np.testing.assert_array_equal(a, b)
