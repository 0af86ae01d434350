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
    # no two code bits share a bit of a word; every bit stays inside the blob
    keys = set(zip(wbyte.reshape(-1).tolist(), bit.reshape(-1).tolist()))
    assert len(keys) == wbyte.size
    assert wbyte.max() < qz.blob_bytes(b, d) and bit.min() >= 0 and bit.max() < 32
    # the blob has no more room than its codes need, up to the 3-bit padding
    assert qz.blob_bytes(b, d) * 8 - 32 * d * b == (0 if b != 3 else 32 * (32 * qz.words_per_lane(3, d) - 3 * d))


def _extract_registers(blob, b, d):
    """Model of the decode-side unpacking: for every lane and register
    (rho, kh), mask the source word to the class bits of each byte (3-bit top
    sources are first assembled from the top bits of three words).  Returns
    uint8 [32, D/8, 2, 4] byte values."""
    words = np.asarray(blob, dtype=np.uint8).view(np.uint32).astype(np.int64)
    nw = qz.words_per_lane(b, d)
    c = qz.CLASSES[b]
    out = np.zeros((32, d // 8, 2, 4), dtype=np.int64)
    for lane in range(32):
        wl = [int(words[qz.word_byte(nw, lane, w) // 4]) for w in range(nw)]
        for rho in range(d // 8):
            for kh in range(2):
                j, sigma = rho % c, 2 * (rho // c) + kh
                if b == 3 and sigma >= nw:
                    q = sigma - nw
                    src = ((wl[3 * q] >> 6) & 0x03030303) | ((wl[3 * q + 1] >> 4) & 0x0C0C0C0C) | (
                        (wl[3 * q + 2] >> 2) & 0x30303030)
                else:
                    src = wl[sigma]
                mask = (((1 << b) - 1) * 0x01010101) & 0xFFFFFFFF
                reg = src & ((mask << (b * j)) & 0xFFFFFFFF)
                for e in range(4):
                    out[lane, rho, kh, e] = (reg >> (8 * e)) & 0xFF
    return out


@pytest.mark.parametrize("role", ["K", "V"])
@pytest.mark.parametrize("b", BITS)
@pytest.mark.parametrize("d", [64, 128])
def test_masked_registers_read_code_times_class_factor(role, b, d):
    """Each byte of a masked register equals code * 2^(b*j) of the code the
    table places there (fits a u8), and every row group's two registers share
    one class -- the property the integer tensor-core path relies on."""
    rng = np.random.default_rng(b * 1000 + d + (role == "V"))
    shape = (32, d) if role == "K" else (d, 32)
    codes = rng.integers(0, 1 << b, size=shape, dtype=np.uint8)
    regs = _extract_registers(qz.pack_blob(codes, role, b), b, d)
    c = qz.CLASSES[b]
    for lane in range(32):
        for rho in range(d // 8):
            f = 1 << (b * (rho % c))
            for kh in range(2):
                for e in range(4):
                    r, col = qz.fragment_coords(role, d, lane, rho, kh, e)
                    assert regs[lane, rho, kh, e] == int(codes[r, col]) * f
                    assert regs[lane, rho, kh, e] <= 255


def test_fragment_products_reproduce_the_dot_products():
    """Integer model of one tile's two MMAs built from the registers alone:
    sum over fragments of (register byte / class factor) * operand equals the
    plain q.K^T and P.V products of the codes (K: token x channel, V: channel
    x token, P in the V token order of the format)."""
    rng = np.random.default_rng(7)
    d, b = 128, 2
    kc = rng.integers(0, 4, size=(32, d), dtype=np.uint8)
    vc = rng.integers(0, 4, size=(d, 32), dtype=np.uint8)
    q = rng.integers(-127, 128, size=d).astype(np.int64)
    p = rng.integers(0, 256, size=32).astype(np.int64)
    kr = _extract_registers(qz.pack_blob(kc, "K", b), b, d)
    vr = _extract_registers(qz.pack_blob(vc, "V", b), b, d)
    c = qz.CLASSES[b]
    s_k = np.zeros(32, dtype=np.int64)
    o_v = np.zeros(d, dtype=np.int64)
    for lane in range(32):
        gid, tig = lane >> 2, lane & 3
        for rho in range(d // 8):
            f = 1 << (b * (rho % c))
            for kh in range(2):
                for e in range(4):
                    # K: B operand of byte e of a k32 fragment is channel 32g + 16kh + 4tig + e
                    g = rho % (d // 32)
                    s_k[gid + 8 * (rho // (d // 32))] += (kr[lane, rho, kh, e] // f) * q[32 * g + 16 * kh + 4 * tig + e]
                    # V: B operand k = 16kh + 4tig + e holds token 4kh + tig + 8e
                    o_v[16 * (rho // 2) + 8 * (rho % 2) + gid] += (vr[lane, rho, kh, e] // f) * p[4 * kh + tig + 8 * e]
    assert np.array_equal(s_k, kc.astype(np.int64) @ q)
    assert np.array_equal(o_v, vc.astype(np.int64) @ p)


def test_pack_positions_golden():
    spec = json.load(open(os.path.join(GOLDEN, "pack_positions.json")))
    for c in spec["cases"]:
        rows, cols, wbyte, bit = qz.pack_table(c["role"], c["bits"], c["head_dim"])
        idx = np.nonzero((rows == c["row"]) & (cols == c["col"]))[0]
        assert idx.size == 1
        got = [[int(a), int(t)] for a, t in zip(wbyte[idx[0]], bit[idx[0]])]
        assert got == c["positions"], c["why"]


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
