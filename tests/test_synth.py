"""The seeded input generators: known-answer vectors and distribution checks."""
import numpy as np
import torch

from synth import configs, draws
from synth.philox import philox4x32_10


def test_philox_known_answers(golden):
    for row in golden("philox_kat.txt"):
        v = [int(h, 16) for h in row if h != "->"]
        out = philox4x32_10(*v[:6])
        assert [int(o) for o in out] == v[6:10]


def test_t4_moments_and_tail():
    t = draws.t4_draws(0, 5, 0, 1_000_000).astype(np.float64)
    assert abs(t.mean()) < 0.01
    assert abs(t.var() / 2.0 - 1.0) < 0.05               # nu / (nu - 2) = 2
    # closed-form t(4) CDF: F(t) = 1/2 + 3/8 s (1 - s^2 / 12), s = t / sqrt(1 + t^2 / 4)
    x = 6 * np.sqrt(2)                                    # 6 sigma of the scaled weights
    s = x / np.sqrt(1 + x * x / 4)
    tail = 2 * (0.5 - 0.375 * s * (1 - s * s / 12))
    frac = np.mean(np.abs(t) > x)
    assert abs(frac / tail - 1) < 0.15


def test_weights_slices_consistent():
    full = draws.expert_weights(0, 2, (3, 40, 64))
    part = draws.expert_weights(0, 2, (3, 40, 64), start_row=57, rows=20)
    assert np.array_equal(full[57:77], part)
    assert full.dtype == np.float32 and full.shape == (120, 64)
    assert abs(full.std() / 0.02 - 1) < 0.1


def test_planted_outliers():
    w = draws.expert_weights(0, 3, (200, 1000), outliers=(0.003, 10.0, 49.0))
    mask, vals = draws.planted_outliers(0, 3, 0, 200 * 1000, 0.003, 10.0, 49.0, 0.02)
    assert 0.0025 < mask.mean() < 0.0035
    assert np.array_equal(w.reshape(-1)[mask], vals[mask])
    m = np.abs(vals[mask])
    assert m.min() >= 10 * 0.02 * (1 - 1e-6) and m.max() <= 49 * 0.02 * (1 + 1e-6)
    assert 0.4 < np.mean(vals[mask] < 0) < 0.6


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32)
    bits = draws.f32_to_bf16_bits(x)
    t = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, t)


def test_configs_dims():
    c2 = configs.MOE_C2
    assert (c2.E, c2.H, c2.I, c2.k, c2.T) == (64, 2048, 768, 8, 16)
    c3 = configs.MOE_C3
    assert (c3.E, c3.H, c3.I, c3.k, c3.T, c3.fmt) == (256, 6144, 2048, 8, 64, "nvfp4")
    assert configs.MOE_C4.T == 8192 and configs.LINEAR_C1.N == 2048
    for c in configs.FULL.values():
        s = configs.small(c)
        assert s.fmt == c.fmt


def test_c_twin_equals_numpy():
    for o in (None, (0.00394, 6.0, 49.0)):
        a = draws.expert_weights(0, 3, (400, 384), start_row=33, rows=150, outliers=o, use_c=False)
        b = draws.expert_weights(0, 3, (400, 384), start_row=33, rows=150, outliers=o, use_c=True)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
