"""Checks of the seeded input generators (host only)."""
import numpy as np
import torch

from bit_gemv_rabit_b200 import inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    f = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 10000),
                        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, np.inf, -np.inf], np.float32)]).astype(np.float32)
    ours = inputs.bf16_bits(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(inputs.bf16_to_f32(ours), torch.from_numpy(f).to(torch.bfloat16).float().numpy())


def test_generators_are_seeded_and_shaped():
    W1 = inputs.weight(7, 64, 96, outlier_frac=0.01)
    W2 = inputs.weight(7, 64, 96, outlier_frac=0.01)
    np.testing.assert_array_equal(W1, W2)
    assert W1.dtype == np.float32 and W1.shape == (64, 96)
    # 1% of entries scaled by 20 -> visible in the max
    assert np.abs(W1).max() > 10 * 0.02
    a, b = inputs.scales(7, W1)
    assert a.shape == (2, 64) and b.shape == (2, 96)
    m = float(np.mean(np.abs(W1)))
    prod = np.outer(a[0], b[0])
    assert 0.5 * m < prod.mean() < 1.5 * m
    x = inputs.activations(7, 3, 96, channel_outlier_frac=0.05)
    assert x.dtype == np.uint16 and x.shape == (3, 96)
    xf = inputs.bf16_to_f32(x)
    big = np.abs(xf).max(axis=0) > 0
    assert big.all()


def test_calibration_stats_recipe():
    s_in, s_out = inputs.calibration_stats(3, 300, 4000)
    s_in2, s_out2 = inputs.calibration_stats(3, 300, 4000)
    np.testing.assert_array_equal(s_in, s_in2)
    np.testing.assert_array_equal(s_out, s_out2)
    assert s_in.dtype == np.float32 and s_in.shape == (4000,) and s_out.shape == (300,)
    assert np.all(s_in > 0) and np.all(s_out > 0)
    assert abs(float(s_in.mean(dtype=np.float64)) - 1.0) < 1e-5
    assert abs(float(s_out.mean(dtype=np.float64)) - 1.0) < 1e-5
    # 1% of the input channels are x10 outliers: they lift the top 1% far above the
    # log-normal tail alone (whose top 1% averages about 3.5x the median)
    s_in3, _ = inputs.calibration_stats(3, 300, 4000, outlier_frac=0.0)
    assert np.sort(s_in)[-40:].mean() > 6 * np.median(s_in)
    assert np.sort(s_in3)[-40:].mean() < 6 * np.median(s_in3)
