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


def _signed_zero_groups():
    """Groups of 32 whose extremes are zeros of either sign: all +0, all -0,
    mixed zeros, a -0 minimum under positives, a -0 maximum over negatives."""
    rows = [np.zeros(32), -np.zeros(32), np.where(np.arange(32) % 3 == 0, -0.0, 0.0)]
    r = np.linspace(0.25, 8.0, 32)
    r[[0, 17]] = [-0.0, 0.0]
    rows.append(r)
    r = -np.linspace(0.5, 3.0, 32)
    r[[5, 30]] = [0.0, -0.0]
    rows.append(r)
    return np.asarray(rows, dtype=np.float32)


def test_signed_zero_extremes_are_order_free():
    """min and max are taken as real numbers, so the stored zero and scale of
    a group do not depend on the order of its elements (a group's extremes
    are a property of the set); a zero extreme is stored as +0.0 and an
    all-zero group dequantizes to exactly zero."""
    x = _signed_zero_groups()
    rng = np.random.default_rng(5)
    for b in BITS:
        c0, s0, z0 = qz.quantize_groups(x, b, axis=1)
        assert not np.any(np.signbit(z0)[:4]) and not np.any(np.signbit(s0))
        assert np.all(c0[:3] == 0) and np.all(s0[:3] == 0) and np.all(z0[:3] == 0)
        assert z0[3] == 0 and s0[3] == np.float16(np.float32(8.0) / np.float32((1 << b) - 1))
        assert z0[4] == np.float32(-3.0)
        for _ in range(8):
            perm = rng.permutation(32)
            c, s, z = qz.quantize_groups(x[:, perm], b, axis=1)
            assert np.array_equal(c, c0[:, perm])
            assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
            assert np.array_equal(z.view(np.uint32), z0.view(np.uint32))
        xh = c0.astype(np.float64) * s0.astype(np.float64)[:, None] + z0.astype(np.float64)[:, None]
        assert np.all(xh[:3] == 0)


def _centred_and_offset_groups(rng, n=64):
    """Groups of 32 bf16 values: the first half centred on zero (a symmetric
    law), the second half shifted well away from zero."""
    x = rng.normal(size=(n, 32)).astype(np.float32) * np.exp(rng.normal(size=(n, 1))).astype(np.float32)
    x[n // 2:] += (3.0 * np.abs(x[n // 2:]).max(axis=1, keepdims=True)).astype(np.float32)
    return _bf16(x)


@pytest.mark.parametrize("b", BITS)
def test_hybrid_chooses_by_centring(b):
    """Hybrid rule (InnerQ technique (i), reading: centred groups are quantized
    on the symmetric interval [-M, M]): a group with |max + min| <= (max - min)/8
    gets z = -M and s = fp16(2M / (2^b - 1)); any other group is quantized
    exactly as without the option."""
    rng = np.random.default_rng(100 + b)
    x = _centred_and_offset_groups(rng)
    c_a, s_a, z_a = qz.quantize_groups(x, b, axis=1)
    c_h, s_h, z_h = qz.quantize_groups(x, b, axis=1, hybrid=True)
    mn, mx = x.min(axis=1), x.max(axis=1)
    sym = np.abs(mx.astype(np.float64) + mn) <= (mx.astype(np.float64) - mn) / 8
    assert sym[:32].sum() >= 8 and not sym[32:].any()  # the generator gives both kinds
    m = np.maximum(np.abs(mn), np.abs(mx))
    assert np.array_equal(z_h[sym], -m[sym])
    assert np.array_equal(s_h[sym], (np.float32(2.0) * m[sym] / np.float32((1 << b) - 1)).astype(np.float16))
    for arr_h, arr_a in ((c_h, c_a), (s_h, s_a), (z_h, z_a)):
        assert np.array_equal(arr_h[~sym], arr_a[~sym])
    # the half-step bound holds on either interval
    xh = c_h * s_h.astype(np.float64)[:, None] + z_h.astype(np.float64)[:, None]
    assert np.all(np.abs(xh - x) <= s_h.astype(np.float64)[:, None] * 0.5 * (1 + 2**-10))


@pytest.mark.parametrize("b", BITS)
def test_hybrid_symmetric_group_equals_the_group_widened_to_plus_minus_m(b):
    """A symmetric group is quantized as the asymmetric rule quantizes the same
    group with -M and +M added to it (its extremes become exactly -M, M): an
    independent statement of 'the interval is [-M, M]'."""
    rng = np.random.default_rng(200 + b)
    x = _centred_and_offset_groups(rng)[:32]
    c_h, s_h, z_h = qz.quantize_groups(x, b, axis=1, hybrid=True)
    m = np.maximum(np.abs(x.min(axis=1)), np.abs(x.max(axis=1)))
    sym = qz.symmetric_groups(x.min(axis=1), x.max(axis=1))
    wide = np.concatenate([x, -m[:, None], m[:, None]], axis=1)
    c_w, s_w, z_w = qz.quantize_groups(wide, b, axis=1)
    assert sym.sum() >= 8
    assert np.array_equal(c_h[sym], c_w[sym, :32])
    assert np.array_equal(s_h[sym], s_w[sym]) and np.array_equal(z_h[sym], z_w[sym])


def test_hybrid_threshold_is_inclusive():
    """|max + min| = (max - min) / 8 exactly is centred; a hair more is not."""
    g_on = np.full((1, 32), 1.0, dtype=np.float32)
    g_on[0, 0], g_on[0, 1] = -7.0, 9.0          # |2| = 16 / 8
    g_off = g_on.copy()
    g_off[0, 1] = 9.0625                       # |2.0625| > 16.0625 / 8 (bf16 value)
    assert qz.symmetric_groups(g_on.min(axis=1), g_on.max(axis=1))[0]
    assert not qz.symmetric_groups(g_off.min(axis=1), g_off.max(axis=1))[0]
    _, s, z = qz.quantize_groups(g_on, 2, axis=1, hybrid=True)
    assert z[0] == -9.0 and s[0] == np.float16(6.0)
    _, s, z = qz.quantize_groups(g_off, 2, axis=1, hybrid=True)
    assert z[0] == -7.0


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
