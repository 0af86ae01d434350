"""Pins of the distortion-calibration oracle (oracle/calibration.py) against
what the mathematics fixes: exact recovery of an exact exponential curve, the
textbook uniform-quantization noise of uniform data, the K/V grouping
identity under transposition, the R^2 fallback rule and the sensitivity cap."""

import numpy as np
import pytest

from oracle import calibration as cal
from oracle import quantize as qz


def _bf16(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)


def test_fit_recovers_an_exact_exponential():
    bits = [2, 3, 4, 8]
    alpha, beta = 0.37, 4.6
    d = alpha * beta ** -np.array(bits, dtype=np.float64)
    a, b, r2 = cal.fit_distortion(bits, d)
    assert abs(a - alpha) < 1e-12 * alpha and abs(b - beta) < 1e-12 * beta and abs(r2 - 1.0) < 1e-12


def test_fit_is_the_least_squares_line_in_log_space():
    bits = np.array([2.0, 3.0, 4.0])
    y = np.array([0.0, -1.0, -3.0])  # ln D: not collinear
    a, b, r2 = cal.fit_distortion(bits, np.exp(y))
    # normal equations by hand: slope = cov(b, y) / var(b) = (-1.5) / 1 over centred b = [-1, 0, 1]
    assert abs(-np.log(b) - (-1.5)) < 1e-12
    assert abs(np.log(a) - (np.mean(y) + 1.5 * 3.0)) < 1e-12
    res = y - (np.log(a) - np.log(b) * bits)
    assert abs(r2 - (1 - np.sum(res**2) / np.sum((y - y.mean()) ** 2))) < 1e-12


@pytest.mark.parametrize("b", [2, 3, 4])
def test_uniform_data_gives_the_textbook_noise(b):
    """x ~ U[0, 1): a group of n = 32 spans E[range^2] = n(n-1)/((n+1)(n+2));
    its two end points are exact and the other n - 2 carry the uniform noise
    Delta^2 / 12 with Delta = range / (2^b - 1)."""
    rng = np.random.default_rng(b)
    x = _bf16(rng.random((4096, 128), dtype=np.float32))
    n = 32
    e_range2 = n * (n - 1) / ((n + 1) * (n + 2))
    expect = (n - 2) / n * e_range2 / (12.0 * (2**b - 1) ** 2)
    got = cal.head_mse(x, b, "K")
    assert abs(got / expect - 1) < 0.03


def test_v_groups_are_k_groups_of_the_transpose():
    rng = np.random.default_rng(3)
    x = _bf16(rng.standard_normal((32, 32), dtype=np.float32))
    for b in (2, 3, 4, 8):
        assert cal.head_mse(x, b, "V") == cal.head_mse(np.ascontiguousarray(x.T), b, "K")


def test_gaussian_heads_follow_the_exponential_model():
    """The summary reports R^2 > 0.98 for most heads (W.10) and K/V decay
    rates near 5 (W.11); our quantizer on Gaussian data lands in that range."""
    rng = np.random.default_rng(5)
    bits = [2, 3, 4]
    x = _bf16(rng.standard_normal((2048, 128), dtype=np.float32))
    for role in ("K", "V"):
        _, beta, r2 = cal.fit_distortion(bits, [cal.head_mse(x, b, role) for b in bits])
        assert r2 > 0.98 and 3.0 < beta < 6.0


def test_fallback_takes_the_smaller_beta_for_poor_fits():
    bits = [2, 3, 4]
    good1 = 0.5 * 4.0 ** -np.array(bits, dtype=np.float64)
    good2 = 0.2 * 5.0 ** -np.array(bits, dtype=np.float64)
    bad = np.array([1.0, 0.05, 0.5])  # not monotone: R^2 well below 0.96
    alpha, beta, r2 = cal.calibrate(bits, [good1, good2, bad])
    assert r2[0] > 0.999 and r2[1] > 0.999 and r2[2] < 0.96
    beta_bar = (4.0 + 5.0) / 2
    _, b_fit, _ = cal.fit_distortion(bits, bad)
    assert abs(beta[0] - 4.0) < 1e-12 and abs(beta[1] - 5.0) < 1e-12
    assert beta[2] == min(b_fit, beta_bar)


def test_sensitivity_cap():
    w = np.array([1.0] * 9 + [491.0])  # mean 50: the outlier is capped at 250
    capped = cal.cap_weights(w)
    assert np.array_equal(capped, [1.0] * 9 + [250.0])
    assert np.array_equal(cal.cap_weights(np.ones(4)), np.ones(4))
