"""GPU parity of the distortion measurement (rq_measure_distortion) against the
oracle, and the whole calibration chain -- measure on the GPU, fit, cap the
sensitivities, allocate K and V jointly -- against the oracle's chain."""

import numpy as np
import pytest
import torch

from gpu_helpers import to_f32
from oracle import allocation as al
from oracle import calibration as cal
from quantized_decode_attention_head_b200 import (rq_allocate_bits, rq_cap_weights, rq_fit_distortion,
                                                  rq_measure_distortion)

pytestmark = pytest.mark.gpu

BITS = [2, 3, 4, 8]


def _samples(n_heads, n_tokens, d, k_sigma, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    f = torch.exp(torch.randn((n_heads, 1, d), generator=g, device="cuda") * k_sigma)
    return (torch.randn((n_heads, n_tokens, d), generator=g, device="cuda") * f).to(torch.bfloat16)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("role", ["K", "V"])
def test_measured_distortion_matches_oracle(d, role):
    x = _samples(3, 256, d, 1.5 if role == "K" else 0.0, seed=d + (role == "V"))
    got = rq_measure_distortion(x, role, BITS)
    xn = to_f32(x)
    for h in range(3):
        exp = [cal.head_mse(xn[h], b, role) for b in BITS]
        assert np.allclose(got[h], exp, rtol=1e-12, atol=0.0), (h, got[h], exp)


def test_calibration_chain_matches_oracle():
    n_heads, bits = 6, [2, 3, 4]
    k = _samples(n_heads, 512, 128, 1.5, seed=21)
    v = _samples(n_heads, 512, 128, 0.0, seed=22)
    mk, mv = rq_measure_distortion(k, "K", bits), rq_measure_distortion(v, "V", bits)
    ak, bk, _ = rq_fit_distortion(bits, mk)
    av, bv, _ = rq_fit_distortion(bits, mv)
    w = np.concatenate([np.linspace(0.5, 2.0, n_heads), np.linspace(0.2, 1.0, n_heads)])
    w[0] = 60.0  # an outlier sensitivity, capped at 5 * mean
    wc = rq_cap_weights(w)
    lib = rq_allocate_bits(wc, np.concatenate([ak, av]), np.concatenate([bk, bv]), 3.0, bits)["b_int"]
    kn, vn = to_f32(k), to_f32(v)
    ok_k = np.array([[cal.head_mse(kn[h], b, "K") for b in bits] for h in range(n_heads)])
    ok_v = np.array([[cal.head_mse(vn[h], b, "V") for b in bits] for h in range(n_heads)])
    oak, obk, _ = cal.calibrate(bits, ok_k)
    oav, obv, _ = cal.calibrate(bits, ok_v)
    orc = al.allocate(cal.cap_weights(w), np.concatenate([oak, oav]), np.concatenate([obk, obv]), 3.0, bits)["b_int"]
    assert np.array_equal(lib, orc)
    assert lib.sum() <= 3 * 2 * n_heads
