"""Group-wise asymmetric KV quantizer and packed tile format (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Sources
-------
"InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language
Models" (pith.science page for arXiv 2602.23200), abstract and "Core claim":
the cache matrices are grouped along the *inner* dimension of the decode
vector-matrix product -- keys per token along head_dim, values per channel along
tokens -- so each group's scale factors out of the inner sum; asymmetric
quantization is one of the per-group options; recent and sink tokens stay in
high precision.

The rounding rule (every step IEEE fp32, round-to-nearest-even, no FMA):

    x  = bf16 input widened to fp32 (exact)
    mn, mx = min, max over the group
    s32 = (mx - mn) / (2**b - 1)             fp32 subtract, fp32 divide
    s16 = fp16_rne(min(s32, 65504))           stored scale (fp16)
    s   = fp32(s16)
    z   = mn                                 stored zero (bf16, exact)
    r   = 1 / s  (fp32 divide) if s > 0 else 0
    c   = clamp(rint((x - z) * r), 0, 2**b - 1)
    x_hat = c * s + z                         (dequantized, fp64 here)

Packed tile record (one per 32-token tile of one (layer, batch, kv-head)
stream), byte layout:

    [K code blob][K meta][V code blob][V meta]

Code blobs.  Each of the 32 lanes of a blob owns D/2 *pairs* of codes; a pair
is two codes that share a 32-bit word, the first at bit b*p, the second at bit
16 + b*p (slot p of the word).  The pairs a lane owns are the elements of the
16x16 "A" operand fragments of an m16n8k16 tensor-core multiply-accumulate:

    lane = 4*gid + tig;   pair (mb, kb, r), r in 0..3
    row = 16*mb + 8*(r & 1) + gid
    col = 16*kb + 8*(r >> 1) + 2*tig + h    (h = 0 first code, h = 1 second)

    K blob: row = token (mb in 0..1),  col = channel (kb in 0..D/16-1)
    V blob: row = channel (mb in 0..D/16-1), col = token (kb in 0..1)

Pairs are grouped in quads of four.  K quad Q = (mb*2 + rr)*(D/32) + grp holds
the pairs (mb, 2grp + kk, rr + 2ch) for u = 2kk + ch; V quad Q = mb*2 + rr
holds (mb, kb, rr + 2ch) for u = 2kb + ch.  Quad Q occupies entries
4Q .. 4Q+3 of the lane's slot list, which orders the W = ceil(D / cpw) words'
slots by (class, word, slot) with the per-slot class

    b = 2: [0,1,2,3,4,0,1,2]   b = 4: [0,1,0,1]   b = 3, 8: all 0

(cpw = codes per word = 16, 10, 8, 4 for b = 2, 3, 4, 8).  The class is the
number of b-bit steps a code sits above the lowest position it can be read
from in place inside an fp16 mantissa; grouping equal classes into a quad lets
one scale factor per quad undo the position.  Unused slots (b = 3) are zero.
Word w of lane L is stored at byte ((w // 4) * 32 + L) * 16 + (w % 4) * 4 for
w < 4*floor(W/4), else at floor(W/4)*512 + ((w - 4*floor(W/4)) * 32 + L) * 4.

Metadata entries are u32 = fp16 bits of s | bf16 bits of z << 16.
    K meta: D/32 groups x 32 entries; entry i of group grp is token
            t = 16*((i >> 1) & 1) + 8*(i & 1) + (i >> 2).
    V meta: D entries; entry i is channel d = 16*mb + 8*rr + gid with
            gid = i // (D/8), mb = (i % (D/8)) // 2, rr = i % 2.
"""

from __future__ import annotations

from functools import lru_cache

import numpy as np

TILE = 32  # tokens per quantized tile == group size g
CPW = {2: 16, 3: 10, 4: 8, 8: 4}
SLOT_CLASS = {2: [0, 1, 2, 3, 4, 0, 1, 2], 3: [0] * 5, 4: [0, 1, 0, 1], 8: [0, 0]}


# ---------------------------------------------------------------- bf16 helpers
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 values that are exactly bf16 -> uint16 bit patterns."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value is not exactly representable in bf16")
    return (u >> 16).astype(np.uint16)


# ------------------------------------------------------------------ quantizer
def quantize_groups(x: np.ndarray, b: int, axis: int):
    """Quantize float32 (bf16-valued) data in groups that run along ``axis``.

    Returns (codes uint8 same shape as x, s16 float16, z float32) where s16 and
    z have ``axis`` removed.
    """
    if b not in CPW:
        raise ValueError(f"unsupported bit width {b}")
    x = np.asarray(x, dtype=np.float32)
    qmax = np.float32((1 << b) - 1)
    mn = np.min(x, axis=axis)
    mx = np.max(x, axis=axis)
    with np.errstate(over="ignore", invalid="ignore"):
        s32 = (mx - mn).astype(np.float32) / qmax
    s32 = np.minimum(s32, np.float32(65504.0)).astype(np.float32)
    s16 = s32.astype(np.float16)
    s = s16.astype(np.float32)
    r = np.zeros_like(s)
    pos = s > 0
    r[pos] = np.float32(1.0) / s[pos]
    zb = np.expand_dims(mn, axis)
    rb = np.expand_dims(r, axis)
    diff = (x - zb).astype(np.float32)
    y = (diff * rb).astype(np.float32)
    c = np.clip(np.rint(y), 0, qmax).astype(np.uint8)
    return c, s16, mn.astype(np.float32)


def quantize_tile(k_tile: np.ndarray, v_tile: np.ndarray, kb: int, vb: int):
    """Quantize one 32-token tile.  k_tile, v_tile: float32 [32, D] (bf16 values).

    K groups: per token, 32 consecutive channels.  V groups: per channel, the
    tile's 32 tokens.  Returns dict with codes [32, D] (token-major) for K and
    V, K scale/zero [32, D/32], V scale/zero [D].
    """
    q = quantize_tiles(k_tile[None], v_tile[None], kb, vb)
    return {key: val[0] for key, val in q.items()}


def quantize_tiles(k_tiles: np.ndarray, v_tiles: np.ndarray, kb: int, vb: int):
    """The same rule applied to n tiles at once: inputs [n, 32, D]; outputs
    carry a leading tile axis."""
    n, t, d = k_tiles.shape
    assert t == TILE and d % 32 == 0
    kx = np.asarray(k_tiles, dtype=np.float32).reshape(n, TILE, d // 32, 32)
    kc, ks, kz = quantize_groups(kx, kb, axis=3)
    vc, vs, vz = quantize_groups(np.asarray(v_tiles, dtype=np.float32), vb, axis=1)
    return {
        "k_codes": kc.reshape(n, TILE, d),
        "k_s": ks,  # [n, 32 tokens, D/32 groups]
        "k_z": kz,
        "v_codes": vc,  # [n, 32 tokens, D]
        "v_s": vs,  # [n, D]
        "v_z": vz,
    }


def dequantize_tile(q: dict) -> tuple[np.ndarray, np.ndarray]:
    """fp64 x_hat = c * s + z for K and V of one tile (or of n tiles with a
    leading tile axis)."""
    kc = q["k_codes"].astype(np.float64)
    ks = np.repeat(q["k_s"].astype(np.float64), 32, axis=-1)
    kz = np.repeat(q["k_z"].astype(np.float64), 32, axis=-1)
    vc = q["v_codes"].astype(np.float64)
    vs = q["v_s"].astype(np.float64)[..., None, :]
    vz = q["v_z"].astype(np.float64)[..., None, :]
    return kc * ks + kz, vc * vs + vz


# --------------------------------------------------------------- pack format
def words_per_lane(b: int, head_dim: int) -> int:
    return -(-head_dim // CPW[b])


def _sorted_slots(b: int, n_words: int):
    slots = [(SLOT_CLASS[b][p], w, p) for w in range(n_words) for p in range(CPW[b] // 2)]
    slots.sort()
    return [(w, p) for _, w, p in slots]


def _lane_pairs(role: str, head_dim: int):
    """The lane-independent list of (mb, kb, r) in quad order (quad-major)."""
    out = []
    if role == "K":
        for mb in range(2):
            for rr in range(2):
                for grp in range(head_dim // 32):
                    for kk in range(2):
                        for ch in range(2):
                            out.append((mb, 2 * grp + kk, rr + 2 * ch))
    elif role == "V":
        for mb in range(head_dim // 16):
            for rr in range(2):
                for kb in range(2):
                    for ch in range(2):
                        out.append((mb, kb, rr + 2 * ch))
    else:
        raise ValueError(role)
    return out


@lru_cache(maxsize=None)
def pack_table(role: str, b: int, head_dim: int):
    """Scatter table for one code blob.

    Returns (rows, cols, word_byte, bit) arrays of length 32 * head_dim * 32 / 32
    = 32 * D: for every code of the tile, the fragment row/col it holds, the
    byte offset of its 32-bit word inside the blob and its bit offset.
    """
    n_words = words_per_lane(b, head_dim)
    slots = _sorted_slots(b, n_words)
    pairs = _lane_pairs(role, head_dim)
    assert len(pairs) == head_dim // 2 and len(slots) >= len(pairs)
    full4 = 4 * (n_words // 4)
    rows, cols, wbyte, bit = [], [], [], []
    for lane in range(32):
        gid, tig = lane >> 2, lane & 3
        for j, (mb, kb, r) in enumerate(pairs):
            w, p = slots[j]
            if w < full4:
                off = ((w // 4) * 32 + lane) * 16 + (w % 4) * 4
            else:
                off = (n_words // 4) * 512 + ((w - full4) * 32 + lane) * 4
            row = 16 * mb + 8 * (r & 1) + gid
            for h in range(2):
                col = 16 * kb + 8 * (r >> 1) + 2 * tig + h
                rows.append(row)
                cols.append(col)
                wbyte.append(off)
                bit.append(16 * h + b * p)
    return (np.array(rows), np.array(cols), np.array(wbyte), np.array(bit))


def blob_bytes(b: int, head_dim: int) -> int:
    return words_per_lane(b, head_dim) * 32 * 4


def pack_blob(codes_rc: np.ndarray, role: str, b: int) -> np.ndarray:
    """codes_rc: uint8 [rows, cols] (or [n, rows, cols]) in fragment
    coordinates (K: [token, channel]; V: [channel, token]).  Returns the blob
    bytes (uint8 [blob] or [n, blob])."""
    single = codes_rc.ndim == 2
    c = codes_rc[None] if single else codes_rc
    head_dim = c.shape[2] if role == "K" else c.shape[1]
    rows, cols, wbyte, bit = pack_table(role, b, head_dim)
    n_words = blob_bytes(b, head_dim) // 4
    # codes never overlap inside a word, so OR == sum over the codes of a word
    vals = c[:, rows, cols].astype(np.uint64) << bit.astype(np.uint64)
    words = np.zeros((c.shape[0], n_words), dtype=np.uint64)
    order = np.argsort(wbyte, kind="stable")
    w_sorted = wbyte[order] // 4
    starts = np.searchsorted(w_sorted, np.arange(n_words))
    present = np.unique(w_sorted)
    sums = np.add.reduceat(vals[:, order], starts[present], axis=1)
    words[:, present] = sums
    out = words.astype(np.uint32).view(np.uint8)
    return out[0] if single else out


def unpack_blob(blob: np.ndarray, role: str, b: int, head_dim: int) -> np.ndarray:
    """Inverse of pack_blob: returns codes in fragment coordinates."""
    rows, cols, wbyte, bit = pack_table(role, b, head_dim)
    words = np.asarray(blob, dtype=np.uint8).view(np.uint32)
    shape = (TILE, head_dim) if role == "K" else (head_dim, TILE)
    out = np.zeros(shape, dtype=np.uint8)
    out[rows, cols] = ((words[wbyte // 4] >> bit.astype(np.uint32)) & ((1 << b) - 1)).astype(np.uint8)
    return out


def k_meta_token(i):
    i = np.asarray(i)
    return 16 * ((i >> 1) & 1) + 8 * (i & 1) + (i >> 2)


def v_meta_channel(i, head_dim):
    i = np.asarray(i)
    per = head_dim // 8
    gid, rem = i // per, i % per
    return 16 * (rem // 2) + 8 * (rem % 2) + gid


def meta_word(s16: np.ndarray, z: np.ndarray) -> np.ndarray:
    sb = np.asarray(s16, dtype=np.float16).view(np.uint16).astype(np.uint32)
    zb = f32_to_bf16_bits(z).astype(np.uint32)
    return sb | (zb << 16)


def record_bytes(kb: int, vb: int, head_dim: int) -> int:
    return blob_bytes(kb, head_dim) + head_dim * 4 + blob_bytes(vb, head_dim) + head_dim * 4


def pack_record(q: dict, kb: int, vb: int) -> np.ndarray:
    """Serialize one quantized tile into its record bytes."""
    return pack_records({k: v[None] for k, v in q.items()}, kb, vb)[0]


def pack_records(q: dict, kb: int, vb: int) -> np.ndarray:
    """Serialize n quantized tiles (leading tile axis) -> uint8 [n, record]."""
    n, _, d = q["k_codes"].shape
    kblob = pack_blob(q["k_codes"], "K", kb)
    t_of_i = k_meta_token(np.arange(32))
    kmeta = np.concatenate(
        [meta_word(q["k_s"][:, t_of_i, g], q["k_z"][:, t_of_i, g]) for g in range(d // 32)], axis=1
    )
    vblob = pack_blob(np.ascontiguousarray(np.swapaxes(q["v_codes"], 1, 2)), "V", vb)
    d_of_i = v_meta_channel(np.arange(d), d)
    vmeta = meta_word(q["v_s"][:, d_of_i], q["v_z"][:, d_of_i])
    kmeta = np.ascontiguousarray(kmeta, dtype=np.uint32)
    vmeta = np.ascontiguousarray(vmeta, dtype=np.uint32)
    out = np.concatenate(
        [kblob, kmeta.view(np.uint8).reshape(n, -1), vblob, vmeta.view(np.uint8).reshape(n, -1)], axis=1
    )
    assert out.shape[1] == record_bytes(kb, vb, d)
    return out


def unpack_record(rec: np.ndarray, kb: int, vb: int, head_dim: int) -> dict:
    """Parse record bytes back into codes / scales / zeros (token-major)."""
    rec = np.asarray(rec, dtype=np.uint8)
    o = 0
    kbl = blob_bytes(kb, head_dim)
    kc = unpack_blob(rec[o : o + kbl], "K", kb, head_dim)
    o += kbl
    kmeta = rec[o : o + head_dim * 4].view(np.uint32).reshape(head_dim // 32, 32)
    o += head_dim * 4
    vbl = blob_bytes(vb, head_dim)
    vc = unpack_blob(rec[o : o + vbl], "V", vb, head_dim).T
    o += vbl
    vmeta = rec[o : o + head_dim * 4].view(np.uint32)
    t_of_i = k_meta_token(np.arange(32))
    k_s = np.zeros((32, head_dim // 32), dtype=np.float16)
    k_z = np.zeros((32, head_dim // 32), dtype=np.float32)
    for g in range(head_dim // 32):
        k_s[t_of_i, g] = (kmeta[g] & 0xFFFF).astype(np.uint16).view(np.float16)
        k_z[t_of_i, g] = bf16_bits_to_f32((kmeta[g] >> 16).astype(np.uint16))
    d_of_i = v_meta_channel(np.arange(head_dim), head_dim)
    v_s = np.zeros(head_dim, dtype=np.float16)
    v_z = np.zeros(head_dim, dtype=np.float32)
    v_s[d_of_i] = (vmeta & 0xFFFF).astype(np.uint16).view(np.float16)
    v_z[d_of_i] = bf16_bits_to_f32((vmeta >> 16).astype(np.uint16))
    return {"k_codes": kc, "k_s": k_s, "k_z": k_z, "v_codes": np.ascontiguousarray(vc), "v_s": v_s, "v_z": v_z}
