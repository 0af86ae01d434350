"""Pins for the fp64 attention oracle: library routine (torch SDPA in fp64 on
CPU) on unquantized inputs, closed forms (uniform scores, a dominant key),
token-permutation invariance and the grouped-query head mapping."""

import numpy as np
import pytest
import torch

from oracle import attention as at
from oracle import cache as ca


@pytest.mark.parametrize("g,d,t", [(1, 64, 7), (4, 128, 300), (8, 64, 33)])
def test_matches_torch_sdpa_fp64(g, d, t):
    rng = np.random.default_rng(g + d + t)
    q = rng.normal(size=(g, d))
    k = rng.normal(size=(t, d)) * np.exp(rng.normal(size=d))
    v = rng.normal(size=(t, d))
    ours = at.attend(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :],
        torch.from_numpy(k)[None, None].expand(1, g, t, d),
        torch.from_numpy(v)[None, None].expand(1, g, t, d),
    )[0, :, 0, :].numpy()
    assert np.allclose(ours, ref, rtol=0, atol=1e-12)
    ours2 = at.attend(q, k, v, scale=0.37)
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :],
        torch.from_numpy(k)[None, None].expand(1, g, t, d),
        torch.from_numpy(v)[None, None].expand(1, g, t, d),
        scale=0.37,
    )[0, :, 0, :].numpy()
    assert np.allclose(ours2, ref2, rtol=0, atol=1e-12)


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(1)
    k = rng.normal(size=(50, 64))
    v = rng.normal(size=(50, 64))
    out = at.attend(np.zeros((2, 64)), k, v)
    assert np.allclose(out, v.mean(axis=0), atol=1e-14)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(2)
    k = rng.normal(size=(40, 64)) * 0.01
    q = np.zeros((1, 64))
    q[0, 0] = 1.0
    k[17, 0] = 8000.0  # score gap ~ 1000 after 1/sqrt(64)
    v = rng.normal(size=(40, 64))
    assert np.allclose(at.attend(q, k, v)[0], v[17], atol=1e-12)


def test_token_order_invariance():
    rng = np.random.default_rng(3)
    q, k, v = rng.normal(size=(4, 64)), rng.normal(size=(90, 64)), rng.normal(size=(90, 64))
    perm = rng.permutation(90)
    assert np.allclose(at.attend(q, k, v), at.attend(q, k[perm], v[perm]), atol=1e-13)


def test_gqa_head_mapping():
    # kv head j has constant value rows equal to j: query head h must output floor(h/G)
    hkv, g, d = 4, 2, 64
    streams = []
    for j in range(hkv):
        st = ca.StreamCache(d, 8, 8, 4, 32)
        k = np.zeros((10, d), dtype=np.float32)
        v = np.full((10, d), float(j), dtype=np.float32)
        st.prefill(k, v)
        streams.append(st)
    out = at.decode_step(np.ones((hkv * g, d)), streams)
    for h in range(hkv * g):
        assert np.allclose(out[h], h // g)
