"""Pins for the quantizer and packed-format oracle.

Against: the error bound of round-to-nearest with the stored fp16 scale, exact
grid round trips, the half-to-even rounding of the rule, hand-derived code
positions of the format (tests/golden/pack_positions.json) and bijectivity of
the format tables.
"""

import json
import os

import numpy as np
import pytest

from oracle import quantize as qz

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = (2, 3, 4, 8)


def _bf16(x):
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even to bf16
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def _tile(rng, d, sigma=1.0):
    f = np.exp(rng.normal(0, sigma, d)).astype(np.float32)
    k = _bf16(rng.normal(size=(32, d)).astype(np.float32) * f)
    v = _bf16(rng.normal(size=(32, d)).astype(np.float32))
    return k, v


@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("d", [64, 128])
def test_code_range_and_half_step_error(b, d):
    rng = np.random.default_rng(b * 7 + d)
    for _ in range(20):
        k, v = _tile(rng, d, sigma=1.5)
        q = qz.quantize_tile(k, v, b, b)
        assert q["k_codes"].max() <= (1 << b) - 1 and q["v_codes"].max() <= (1 << b) - 1
        kh, vh = qz.dequantize_tile(q)
        ks = np.repeat(q["k_s"].astype(np.float64), 32, axis=1)
        vs = q["v_s"].astype(np.float64)[None, :]
        assert np.all(np.abs(kh - k) <= ks * 0.5 * (1 + 2**-10))
        assert np.all(np.abs(vh - v) <= vs * 0.5 * (1 + 2**-10))
        # the group's minimum is reproduced exactly (code 0, x_hat = z)
        assert np.all(kh.reshape(32, d // 32, 32).min(axis=2) == k.reshape(32, d // 32, 32).min(axis=2))


@pytest.mark.parametrize("b", BITS)
def test_grid_round_trip_is_exact(b):
    # x = z + c*s with s a power of two and every code used: the rule must give
    # back c, s, z and x_hat == x exactly.
    rng = np.random.default_rng(b)
    qmax = (1 << b) - 1
    s = np.float32(2.0**-3)
    z = np.float32(-1.0)
    codes = rng.integers(0, qmax + 1, size=(32, 64))
    codes[:, 0] = 0
    codes[:, 31] = qmax
    codes[:, 32] = 0
    codes[:, 63] = qmax
    k = (z + codes.astype(np.float32) * s).astype(np.float32)
    assert np.array_equal(_bf16(k), k)
    vcodes = rng.integers(0, qmax + 1, size=(32, 64))  # [32 tokens, 64 channels]
    vcodes[0, :] = 0
    vcodes[31, :] = qmax
    v = (z + vcodes.astype(np.float32) * s).astype(np.float32)
    q = qz.quantize_tile(k, v, b, b)
    assert np.array_equal(q["k_codes"], codes)
    assert np.array_equal(q["v_codes"], vcodes)
    assert np.all(q["k_s"] == np.float16(s)) and np.all(q["v_s"] == np.float16(s))
    assert np.all(q["k_z"] == z) and np.all(q["v_z"] == z)
    kh, vh = qz.dequantize_tile(q)
    assert np.array_equal(kh, k) and np.array_equal(vh, v)


def test_round_half_to_even():
    # group min 0, max 3, b = 2 -> s = 1; 0.5 -> 0, 1.5 -> 2, 2.5 -> 2 (ties to even)
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, :5] = [0.0, 3.0, 0.5, 1.5, 2.5]
    c, s, z = qz.quantize_groups(x, 2, axis=1)
    assert s[0] == 1.0 and z[0] == 0.0
    assert c[0, :5].tolist() == [0, 3, 0, 2, 2]


def test_scale_is_fp16_rounded_and_used_for_codes():
    # range 1.0 at 3 bits: s32 = 1/7 is not an fp16; the stored scale is its
    # nearest fp16 and codes are computed with that rounded scale.
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 1] = 1.0
    x[0, 2] = np.float32(0.5)  # 0.5 / fp16(1/7) = 3.5004.. -> 4 (not a tie)
    c, s, z = qz.quantize_groups(x, 3, axis=1)
    assert s[0] == np.float16(1.0 / 7.0)
    assert float(s[0]) != np.float32(1.0) / np.float32(7.0)
    assert c[0, 1] == 7 and c[0, 2] == 4


def test_constant_group_is_exact():
    x = np.full((4, 32), np.float32(-2.375), dtype=np.float32)
    for b in BITS:
        c, s, z = qz.quantize_groups(x, b, axis=1)
        assert np.all(c == 0) and np.all(s == 0) and np.all(z == np.float32(-2.375))


@pytest.mark.parametrize("role", ["K", "V"])
@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("d", [64, 128])
def test_pack_table_is_a_bijection(role, b, d):
    rows, cols, wbyte, bit = qz.pack_table(role, b, d)
    shape = (32, d) if role == "K" else (d, 32)
    seen = np.zeros(shape, dtype=np.int64)
    np.add.at(seen, (rows, cols), 1)
    assert np.all(seen == 1)
    # no two codes share bits of a word
    occ = set()
    for wb, bt in zip(wbyte.tolist(), bit.tolist()):
        for k in range(b):
            key = (wb, bt + k)
            assert key not in occ
            occ.add(key)
        assert (bt % 16) + b <= 16
    assert wbyte.max() < qz.blob_bytes(b, d)
    # slots of one quad share one class (4 pairs = 8 codes per quad per lane)
    cls = qz.SLOT_CLASS[b]
    per_lane = d  # codes per lane
    for lane in range(32):
        sl = slice(lane * per_lane, (lane + 1) * per_lane)
        p = (bit[sl] % 16) // b
        for qd in range(per_lane // 8):
            assert len({cls[x] for x in p[qd * 8 : (qd + 1) * 8]}) == 1


def test_pack_positions_golden():
    spec = json.load(open(os.path.join(GOLDEN, "pack_positions.json")))
    for c in spec["cases"]:
        rows, cols, wbyte, bit = qz.pack_table(c["role"], c["bits"], c["head_dim"])
        idx = np.nonzero((rows == c["row"]) & (cols == c["col"]))[0]
        assert idx.size == 1
        assert (int(wbyte[idx[0]]), int(bit[idx[0]])) == (c["byte"], c["bit"]), c["why"]


def test_meta_permutations():
    assert sorted(qz.k_meta_token(np.arange(32)).tolist()) == list(range(32))
    assert qz.k_meta_token(5) == 9 and qz.k_meta_token(6) == 17 and qz.k_meta_token(31) == 31
    for d in (64, 128):
        assert sorted(qz.v_meta_channel(np.arange(d), d).tolist()) == list(range(d))
    assert qz.v_meta_channel(17, 128) == 9
    assert qz.v_meta_channel(1, 64) == 8


@pytest.mark.parametrize("kb,vb", [(2, 2), (3, 2), (4, 8), (8, 3)])
@pytest.mark.parametrize("d", [64, 128])
def test_record_round_trip(kb, vb, d):
    rng = np.random.default_rng(kb * 10 + vb + d)
    k, v = _tile(rng, d)
    q = qz.quantize_tile(k, v, kb, vb)
    rec = qz.pack_record(q, kb, vb)
    assert rec.size == qz.record_bytes(kb, vb, d) and rec.size % 16 == 0
    back = qz.unpack_record(rec, kb, vb, d)
    for key in q:
        assert np.array_equal(back[key], q[key]), key


def test_record_sizes():
    # W(b, D) = ceil(D / codes-per-word); metadata 4 bytes per group
    assert qz.record_bytes(2, 2, 128) == 1024 + 512 + 1024 + 512
    assert qz.record_bytes(3, 3, 128) == 13 * 128 * 2 + 1024
    assert qz.record_bytes(8, 8, 128) == 4096 * 2 + 1024
    assert qz.record_bytes(3, 2, 64) == 7 * 128 + 256 + 4 * 128 + 256
