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
    mn, mx = min, max over the group, each + 0.0 (a -0.0 extreme is stored
             as +0.0: the pages fix no sign for a zero extreme)
    hybrid option only (InnerQ technique (i), a symmetric or asymmetric
    quantizer per group chosen from the group's own statistics; the page
    prints no rule, this is the reading): a group that is nearly centred on
    zero, |mx + mn| <= TAU * (mx - mn) in fp32 with TAU = 1/8, is quantized
    on the symmetric interval [-M, M], M = max(|mn|, |mx|):
               mn, mx = -M, M     (exact: M is a bf16 value)
    and every other group on [mn, mx]; the rest of the rule is the same
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

Code blobs.  Each of the 32 lanes (lane = 4*gid + tig) of a blob owns D/4
registers of four byte lanes e = 0..3, laid out as the 8-bit "A" operand
fragments of the m16n8k32 integer tensor-core multiply-accumulate.  Register
(rho, kh) -- row group rho in 0..D/8-1, half kh in 0..1 -- holds in byte e:

    K blob: rho = i*(D/32) + g            code of token t = gid + 8*i,
                                          channel d = 32*g + 16*kh + 4*tig + e
    V blob: rho = 2*mb + rh               code of channel d = 16*mb + 8*rh + gid,
                                          token t = 4*kh + tig + 8*e

(the V token order is the order in which the softmax probabilities of a tile
arrive in the "B" fragment of the P.V product).  Row group rho has class
j = rho mod C and both its registers come from source sigma = 2*(rho // C) + kh,
with C = 4, 2, 2, 1 classes for b = 2, 3, 4, 8.  A register of class j is the
source word masked to the bits [b*j, b*j + b) of each of its four bytes, so
every byte reads as code * 2^(b*j) and one factor 2^(-b*j) per row group
undoes the position.

    b = 2, 4, 8: source sigma is word sigma; the code of byte e occupies bits
                 8e + b*j .. 8e + b*j + b - 1.
    b = 3:       W = ceil(D/10) words (ten codes per word, as dense as 10 per
                 u32).  Source sigma < W is word sigma, code at bits
                 8e + 3j .. 8e + 3j + 2.  Source sigma = W + q is assembled
                 from the two top bits (6, 7) of each byte of words 3q, 3q+1,
                 3q+2: bit k of the class-j code of byte e is bit
                 8e + 6 + (f mod 2) of word 3q + f // 2, f = 3j + k.  The top
                 bits of the remaining words are zero.

A blob has W = ceil(D / cpw) words per lane (cpw = 16, 10, 8, 4 codes per word
for b = 2, 3, 4, 8).  Word w of lane L is stored at byte
((w // 4) * 32 + L) * 16 + (w % 4) * 4 for w < 4*floor(W/4), else at
floor(W/4)*512 + ((w - 4*floor(W/4)) * 32 + L) * 4.

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
# hybrid option: a group with |max + min| <= TAU * (max - min) is quantized on
# the symmetric interval [-M, M] (power of two, so TAU * w is exact in fp32)
TAU = np.float32(0.125)


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
def symmetric_groups(mn: np.ndarray, mx: np.ndarray) -> np.ndarray:
    """Hybrid rule: True where a group with extremes (mn, mx) is nearly
    centred on zero, |mx + mn| <= TAU * (mx - mn), each side one fp32
    operation rounded to nearest even."""
    mn = np.asarray(mn, dtype=np.float32)
    mx = np.asarray(mx, dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        centre = np.abs((mx + mn).astype(np.float32))
        width = ((mx - mn).astype(np.float32) * TAU).astype(np.float32)
    return centre <= width


def quantize_groups(x: np.ndarray, b: int, axis: int, hybrid: bool = False):
    """Quantize float32 (bf16-valued) data in groups that run along ``axis``.

    Returns (codes uint8 same shape as x, s16 float16, z float32) where s16 and
    z have ``axis`` removed.  hybrid: centred groups on [-M, M] (see above).
    """
    if b not in CPW:
        raise ValueError(f"unsupported bit width {b}")
    x = np.asarray(x, dtype=np.float32)
    qmax = np.float32((1 << b) - 1)
    # min and max as real numbers: a -0.0 extreme becomes +0.0 (x + 0 in IEEE
    # round-to-nearest), so which of two equal zeros a reduction returns does
    # not matter
    mn = (np.min(x, axis=axis) + np.float32(0.0)).astype(np.float32)
    mx = (np.max(x, axis=axis) + np.float32(0.0)).astype(np.float32)
    if hybrid:
        sym = symmetric_groups(mn, mx)
        m = np.maximum(np.abs(mn), np.abs(mx)).astype(np.float32)
        mn = np.where(sym, (-m + np.float32(0.0)).astype(np.float32), mn).astype(np.float32)
        mx = np.where(sym, m, mx).astype(np.float32)
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


def quantize_tile(k_tile: np.ndarray, v_tile: np.ndarray, kb: int, vb: int, hybrid: bool = False):
    """Quantize one 32-token tile.  k_tile, v_tile: float32 [32, D] (bf16 values).

    K groups: per token, 32 consecutive channels.  V groups: per channel, the
    tile's 32 tokens.  Returns dict with codes [32, D] (token-major) for K and
    V, K scale/zero [32, D/32], V scale/zero [D].
    """
    q = quantize_tiles(k_tile[None], v_tile[None], kb, vb, hybrid)
    return {key: val[0] for key, val in q.items()}


def quantize_tiles(k_tiles: np.ndarray, v_tiles: np.ndarray, kb: int, vb: int, hybrid: bool = False):
    """The same rule applied to n tiles at once: inputs [n, 32, D]; outputs
    carry a leading tile axis."""
    n, t, d = k_tiles.shape
    assert t == TILE and d % 32 == 0
    kx = np.asarray(k_tiles, dtype=np.float32).reshape(n, TILE, d // 32, 32)
    kc, ks, kz = quantize_groups(kx, kb, axis=3, hybrid=hybrid)
    vc, vs, vz = quantize_groups(np.asarray(v_tiles, dtype=np.float32), vb, axis=1, hybrid=hybrid)
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
CLASSES = {2: 4, 3: 2, 4: 2, 8: 1}


def words_per_lane(b: int, head_dim: int) -> int:
    return -(-head_dim // CPW[b])


def word_byte(n_words: int, lane: int, w: int) -> int:
    full4 = 4 * (n_words // 4)
    if w < full4:
        return ((w // 4) * 32 + lane) * 16 + (w % 4) * 4
    return (n_words // 4) * 512 + ((w - full4) * 32 + lane) * 4


def code_bit_positions(b: int, head_dim: int, rho: int, kh: int, e: int):
    """(word, bit) of bits 0..b-1 of the code in byte e of register (rho, kh)."""
    n_words = words_per_lane(b, head_dim)
    c = CLASSES[b]
    j, sigma = rho % c, 2 * (rho // c) + kh
    if b != 3 or sigma < n_words:
        return [(sigma, 8 * e + b * j + k) for k in range(b)]
    q = sigma - n_words
    out = []
    for k in range(3):
        f = 3 * j + k
        out.append((3 * q + f // 2, 8 * e + 6 + f % 2))
    return out


def fragment_coords(role: str, head_dim: int, lane: int, rho: int, kh: int, e: int):
    """(row, col) of the code in byte e of register (rho, kh) of a lane.
    K: (token, channel); V: (channel, token)."""
    gid, tig = lane >> 2, lane & 3
    if role == "K":
        ng = head_dim // 32
        i, g = rho // ng, rho % ng
        return gid + 8 * i, 32 * g + 16 * kh + 4 * tig + e
    if role == "V":
        mb, rh = rho // 2, rho % 2
        return 16 * mb + 8 * rh + gid, 4 * kh + tig + 8 * e
    raise ValueError(role)


@lru_cache(maxsize=None)
def pack_table(role: str, b: int, head_dim: int):
    """Scatter table for one code blob.

    Returns (rows, cols, word_byte, bit): rows/cols [32 * D] give the fragment
    coordinates of every code of the tile; word_byte/bit [32 * D, b] give, for
    each bit k of that code, the byte offset of its 32-bit word inside the
    blob and the bit offset inside the word.
    """
    n_words = words_per_lane(b, head_dim)
    rows, cols, wbyte, bit = [], [], [], []
    for lane in range(32):
        for rho in range(head_dim // 8):
            for kh in range(2):
                for e in range(4):
                    r, c = fragment_coords(role, head_dim, lane, rho, kh, e)
                    pos = code_bit_positions(b, head_dim, rho, kh, e)
                    rows.append(r)
                    cols.append(c)
                    wbyte.append([word_byte(n_words, lane, w) for w, _ in pos])
                    bit.append([bt for _, bt in pos])
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
    codes = c[:, rows, cols].astype(np.uint64)  # [n, codes]
    # every code bit lands on its own (word, bit): OR == sum over a word
    ks = np.arange(b, dtype=np.uint64)
    vals = ((codes[:, :, None] >> ks) & np.uint64(1)) << bit.astype(np.uint64)[None]  # [n, codes, b]
    widx = (wbyte // 4).reshape(-1)
    vals = vals.reshape(c.shape[0], -1)
    order = np.argsort(widx, kind="stable")
    w_sorted = widx[order]
    present = np.unique(w_sorted)
    starts = np.searchsorted(w_sorted, present)
    words = np.zeros((c.shape[0], n_words), dtype=np.uint64)
    words[:, present] = np.add.reduceat(vals[:, order], starts, axis=1)
    out = words.astype(np.uint32).view(np.uint8)
    return out[0] if single else out


def unpack_blob(blob: np.ndarray, role: str, b: int, head_dim: int) -> np.ndarray:
    """Inverse of pack_blob: returns codes in fragment coordinates."""
    rows, cols, wbyte, bit = pack_table(role, b, head_dim)
    words = np.asarray(blob, dtype=np.uint8).view(np.uint32)
    bits = (words[wbyte // 4] >> bit.astype(np.uint32)) & np.uint32(1)  # [codes, b]
    vals = (bits << np.arange(b, dtype=np.uint32)[None]).sum(axis=1)
    shape = (TILE, head_dim) if role == "K" else (head_dim, TILE)
    out = np.zeros(shape, dtype=np.uint8)
    out[rows, cols] = vals.astype(np.uint8)
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
