"""Pins for cache assembly: window/tile split of the five workloads, the
flush schedule of the 64-step append run, prefill-vs-append equivalence and
the short-context edge cases."""

import numpy as np
import pytest

from oracle import cache as ca
from oracle import quantize as qz


@pytest.mark.parametrize(
    "T,S,R,expect",
    [
        (512, 4, 32, (4, 448, 60)),  # tiny
        (4096, 4, 128, (4, 3936, 156)),  # llama3_8b
        (8192, 4, 128, (4, 8032, 156)),  # qwen3_8b
        (131072, 4, 128, (4, 130912, 156)),  # long_128k
        (32768, 4, 128, (4, 32608, 156)),  # mistral_7b_b64
        (3, 4, 32, (3, 0, 0)),
        (20, 4, 32, (4, 0, 16)),
        (36, 4, 32, (4, 0, 32)),
        (67, 4, 32, (4, 0, 63)),
        (68, 4, 32, (4, 32, 32)),
        (0, 4, 32, (0, 0, 0)),
        (40, 0, 0, (0, 32, 8)),
    ],
)
def test_split_lengths(T, S, R, expect):
    assert ca.split_lengths(T, S, R) == expect
    s, tq, r = expect
    if T >= S + R:
        assert R <= r < R + 32


def test_flush_schedule_of_append_run():
    # 4096-token prefill, S=4, R=128: r = 156 -> flushes when r reaches 160, i.e.
    # at appended steps 4 and 36 (1-based) of a 64-step run.
    st = ca.StreamCache(64, 2, 2, 4, 128)
    rng = np.random.default_rng(0)
    k = rng.normal(size=(4096, 64)).astype(np.float32)
    st.T = 4096
    st.recent = [(p, k[0], k[0]) for p in range(4096 - 156, 4096)]
    st.sink_k = [k[0]] * 4
    st.sink_v = [k[0]] * 4
    flushed = [step for step in range(1, 65) if st.append(k[1], k[1])]
    assert flushed == [4, 36]


@pytest.mark.parametrize("hybrid", [False, True])
@pytest.mark.parametrize("T0,T1,S,R", [(100, 230, 4, 32), (36, 99, 4, 32), (0, 80, 4, 32), (2, 70, 4, 0), (40, 200, 0, 16)])
def test_prefill_then_append_equals_prefill(T0, T1, S, R, hybrid):
    rng = np.random.default_rng(T0 + T1)
    d = 64
    k = qz.bf16_bits_to_f32(rng.integers(0x3C00, 0x4100, size=(T1, d), dtype=np.uint16) ^ rng.integers(0, 2, size=(T1, d), dtype=np.uint16) << 15)
    v = qz.bf16_bits_to_f32(rng.integers(0x3C00, 0x4100, size=(T1, d), dtype=np.uint16))
    a = ca.StreamCache(d, 3, 2, S, R, hybrid=hybrid)
    a.prefill(k[:T0], v[:T0])
    for t in range(T0, T1):
        a.append(k[t], v[t])
    b = ca.StreamCache(d, 3, 2, S, R, hybrid=hybrid)
    b.prefill(k, v)
    assert a.T == b.T == T1 and a.n_tiles == b.n_tiles
    for i in range(a.n_tiles):
        assert np.array_equal(a.record(i), b.record(i))
    assert a.window_rows().keys() == b.window_rows().keys()
    for key, val in a.window_rows().items():
        assert np.array_equal(val, b.window_rows()[key])
    ka, va = a.dequantized()
    assert ka.shape == (T1, d)
    # sink and recent tokens are returned unchanged
    s, tq, r = ca.split_lengths(T1, S, R)
    assert np.array_equal(ka[:s], k[:s]) and np.array_equal(ka[s + tq :], k[s + tq :])
    assert np.array_equal(va[:s], v[:s]) and np.array_equal(va[s + tq :], v[s + tq :])


def test_ring_slots_never_collide_with_live_tokens():
    S, R = 4, 32
    for T in range(S, 400):
        s, tq, r = ca.split_lengths(T, S, R)
        slots = [ca.ring_slot(p, S, R) for p in range(S + tq, T)]
        assert len(set(slots)) == len(slots)


@pytest.mark.parametrize("kb,vb,d", [(2, 2, 128), (3, 8, 64), (4, 3, 128), (8, 4, 64)])
def test_batched_records_equal_single_tile_records(kb, vb, d):
    rng = np.random.default_rng(kb * 100 + vb + d)
    T = 4 + 32 * 5 + 32 + 9
    k = qz.bf16_bits_to_f32(rng.integers(0x3C00, 0x4100, size=(T, d), dtype=np.uint16))
    v = qz.bf16_bits_to_f32(rng.integers(0xBC00, 0xC100, size=(T, d), dtype=np.uint16))
    st = ca.StreamCache(d, kb, vb, 4, 32)
    st.prefill(k, v)
    recs = st.records()
    assert recs.shape == (st.n_tiles, qz.record_bytes(kb, vb, d)) and st.n_tiles == 5
    for i in range(st.n_tiles):
        assert np.array_equal(recs[i], st.record(i))
        # and each record decodes back to the tile's own quantization
        back = qz.unpack_record(recs[i], kb, vb, d)
        a = 4 + 32 * i
        ref = qz.quantize_tile(k[a : a + 32], v[a : a + 32], kb, vb)
        for key in ref:
            assert np.array_equal(back[key], ref[key]), key


# ------------------------------------------------ per-channel K normalization
def _bf16(x):
    """Round float32 to the nearest bf16 value (ties to even)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32).view(np.float32)


def test_channel_norm_closed_forms():
    k = np.zeros((3, 5), dtype=np.float32)
    k[:, 0] = [0.5, -3.0, 1.0]   # max 3 -> 4
    k[:, 1] = [4.0, -1.0, 0.0]   # max 4 -> 4 (already a power of two)
    k[:, 2] = [0.3, 0.1, -0.2]   # max 0.3 -> 0.5
    k[:, 3] = 0.0                # zero channel -> 1
    k[:, 4] = [-1e-3, 0.0, 0.0]  # smallest power of two >= 1e-3 is 2^-9
    n = ca.channel_norm(k)
    assert n.tolist() == [4.0, 4.0, 0.5, 1.0, 2.0**-9]


def test_k_norm_is_invariant_to_power_of_two_channel_scaling():
    """With normalization, scaling a K channel by 2^j leaves every tile record
    unchanged and scales the dequantized channel by exactly 2^j."""
    rng = np.random.default_rng(9)
    T, d = 4 + 32 * 3 + 40, 64
    k = _bf16(rng.standard_normal((T, d), dtype=np.float32))
    v = _bf16(rng.standard_normal((T, d), dtype=np.float32))
    k2 = k.copy()
    k2[:, 5] *= np.float32(8.0)
    k2[:, 17] *= np.float32(0.25)
    a = ca.StreamCache(d, 2, 3, 4, 32, k_norm=True)
    b = ca.StreamCache(d, 2, 3, 4, 32, k_norm=True)
    a.prefill(k, v)
    b.prefill(k2, v)
    assert np.array_equal(a.records(), b.records())
    ka, _ = a.dequantized()
    kb, _ = b.dequantized()
    scale = np.ones(d)
    scale[5], scale[17] = 8.0, 0.25
    assert np.array_equal(ka * scale, kb)


def test_k_norm_reduces_error_on_outlier_channels():
    rng = np.random.default_rng(4)
    T, d = 4 + 32 * 40 + 32, 128
    f = np.exp(rng.standard_normal(d) * 1.5).astype(np.float32)
    k = _bf16(rng.standard_normal((T, d), dtype=np.float32) * f)
    v = _bf16(rng.standard_normal((T, d), dtype=np.float32))
    err = {}
    for norm in (False, True):
        st = ca.StreamCache(d, 2, 2, 4, 32, k_norm=norm)
        st.prefill(k, v)
        kh, _ = st.dequantized()
        # relative error per channel, averaged: outlier channels no longer
        # coarsen the groups they share with small channels
        err[norm] = np.mean(np.abs(kh - k) / (np.abs(k).max(axis=0) + 1e-30))
    assert err[True] < 0.8 * err[False]


def test_k_norm_without_prefill_is_the_identity():
    rng = np.random.default_rng(5)
    d = 64
    a = ca.StreamCache(d, 2, 2, 2, 0, k_norm=True)
    b = ca.StreamCache(d, 2, 2, 2, 0, k_norm=False)
    for _ in range(40):
        kk = _bf16(rng.standard_normal(d, dtype=np.float32) * 5)
        vv = _bf16(rng.standard_normal(d, dtype=np.float32))
        a.append(kk, vv)
        b.append(kk, vv)
    assert np.array_equal(a.records(), b.records())
