"""Per-stream cache assembly and the append rule (oracle; test infrastructure).

A *stream* is one (layer, batch element, kv-head).  Its T cached tokens are

    sink   tokens [0, S)                      bf16, never quantized
    tiles  tokens [S, S + Tq)                 quantized, 32 tokens per tile
    recent tokens [S + Tq, T)                 bf16 ring

Sources: InnerQ (pith.science page for arXiv 2602.23200), abstract: high
precision windows for the most recent tokens and for the attention-sink tokens;
NOVA-KV review page ("Spend Bits Where Queries Look"), assumptions list: sink
and recent bands kept apart from the quantized body.

Readings where the pages are silent:

* Tq = 32 * floor((T - S - R) / 32) when T >= S + R, else 0, so the recent
  window length r = T - S - Tq lies in [R, R + 32) (InnerQ gives no rule for a
  remainder that is not a multiple of the group size).
* Append: the token joins the recent window; when r reaches R + 32 the oldest
  32 recent tokens are quantized (same rule, same order) into the next tile.
  While T < S the token fills the sink.
* The recent ring stores token position P at slot (P - S) mod (R + 32).
* Per-channel K normalization (optional; InnerQ abstract: "per-channel
  normalization of the key cache, computed once during prefill and folded
  into the model parameters"): n_d = the smallest power of two >= the
  absolute maximum of channel d of K over the prefill tokens (1 when that
  maximum is 0 or nothing was prefilled).  Quantized tiles hold K / n (exact:
  a power-of-two scaling) and dequantize to n * K_hat; the sink and recent
  windows keep K as is; queries are multiplied by n (the folding) for the
  quantized tokens only.  The statistic and the power-of-two rounding are this
  library's reading; the page gives neither.
"""

from __future__ import annotations

import numpy as np

from . import quantize as qz

TILE = qz.TILE


def split_lengths(n_tokens: int, n_sink: int, n_recent: int):
    """(sink length, quantized length Tq, recent length r) for T tokens."""
    s = min(n_tokens, n_sink)
    if n_tokens >= n_sink + n_recent:
        tq = ((n_tokens - n_sink - n_recent) // TILE) * TILE
    else:
        tq = 0
    return s, tq, n_tokens - s - tq


def channel_norm(k: np.ndarray) -> np.ndarray:
    """Smallest power of two >= max_t |k[t, d]| per channel (1 for a zero
    channel), float32 [D]."""
    m = np.max(np.abs(np.asarray(k, dtype=np.float32)), axis=0).astype(np.float64)
    frac, e = np.frexp(m)  # m = frac * 2^e, frac in [0.5, 1)
    e = np.where(frac == 0.5, e - 1, e)
    return np.where(m > 0, np.ldexp(1.0, e), 1.0).astype(np.float32)


def ring_slot(pos: int, n_sink: int, n_recent: int) -> int:
    return (pos - n_sink) % (n_recent + TILE)


class StreamCache:
    """Quantized cache of one stream, built token by token or by prefill."""

    def __init__(self, head_dim, k_bits, v_bits, n_sink, n_recent, k_norm=False, hybrid=False):
        self.d = head_dim
        self.k_norm = k_norm
        self.hybrid = hybrid  # per-group symmetric / asymmetric choice (quantize.quantize_groups)
        self.nrm = np.ones(head_dim, dtype=np.float32)  # per-channel K normalization n_d
        self.kb = k_bits
        self.vb = v_bits
        self.S = n_sink
        self.R = n_recent
        self.tiles = []  # list of quantized-tile dicts
        self.sink_k = []
        self.sink_v = []
        self.recent = []  # list of (pos, k, v) in position order
        self.T = 0

    # -- building ------------------------------------------------------------
    def prefill(self, k: np.ndarray, v: np.ndarray):
        """k, v: float32 [T, D] holding bf16 values."""
        T = k.shape[0]
        self.nrm = channel_norm(k) if (self.k_norm and T > 0) else np.ones(self.d, dtype=np.float32)
        kn = (k / self.nrm).astype(np.float32)
        s, tq, r = split_lengths(T, self.S, self.R)
        self.sink_k = [k[i].copy() for i in range(s)]
        self.sink_v = [v[i].copy() for i in range(s)]
        self.tiles = []
        n = tq // TILE
        if n:
            d = self.d
            qb = qz.quantize_tiles(kn[s : s + tq].reshape(n, TILE, d), v[s : s + tq].reshape(n, TILE, d), self.kb, self.vb,
                                   self.hybrid)
            self.tiles = [{key: val[i] for key, val in qb.items()} for i in range(n)]
        self.recent = [(p, k[p].copy(), v[p].copy()) for p in range(s + tq, T)]
        self.T = T

    def append(self, k_new: np.ndarray, v_new: np.ndarray) -> bool:
        """Add one token; returns True when a tile was flushed."""
        pos = self.T
        self.T += 1
        if pos < self.S:
            self.sink_k.append(k_new.copy())
            self.sink_v.append(v_new.copy())
            return False
        self.recent.append((pos, k_new.copy(), v_new.copy()))
        if len(self.recent) == self.R + TILE:
            old = self.recent[:TILE]
            self.recent = self.recent[TILE:]
            kt = (np.stack([o[1] for o in old]) / self.nrm).astype(np.float32)
            vt = np.stack([o[2] for o in old])
            self.tiles.append(qz.quantize_tile(kt, vt, self.kb, self.vb, self.hybrid))
            return True
        return False

    # -- views -----------------------------------------------------------------
    @property
    def n_tiles(self):
        return len(self.tiles)

    def dequantized(self):
        """fp64 K_hat, V_hat [T, D] in token order."""
        parts_k, parts_v = [], []
        if self.sink_k:
            parts_k.append(np.stack(self.sink_k).astype(np.float64))
            parts_v.append(np.stack(self.sink_v).astype(np.float64))
        if self.tiles:
            kh, vh = qz.dequantize_tile({key: np.stack([t[key] for t in self.tiles]) for key in self.tiles[0]})
            parts_k.append(kh.reshape(-1, self.d) * self.nrm.astype(np.float64))
            parts_v.append(vh.reshape(-1, self.d))
        if self.recent:
            parts_k.append(np.stack([r[1] for r in self.recent]).astype(np.float64))
            parts_v.append(np.stack([r[2] for r in self.recent]).astype(np.float64))
        if not parts_k:
            return np.zeros((0, self.d)), np.zeros((0, self.d))
        return np.concatenate(parts_k), np.concatenate(parts_v)

    def record(self, i: int) -> np.ndarray:
        return qz.pack_record(self.tiles[i], self.kb, self.vb)

    def records(self) -> np.ndarray:
        """All tile records, uint8 [n_tiles, record_bytes]."""
        if not self.tiles:
            return np.zeros((0, qz.record_bytes(self.kb, self.vb, self.d)), dtype=np.uint8)
        qb = {key: np.stack([t[key] for t in self.tiles]) for key in self.tiles[0]}
        return qz.pack_records(qb, self.kb, self.vb)

    def window_rows(self):
        """Expected window content as {('sink'|'ring', 'k'|'v', slot): bf16 bits}."""
        out = {}
        for i, (kk, vv) in enumerate(zip(self.sink_k, self.sink_v)):
            out[("sink", "k", i)] = qz.f32_to_bf16_bits(kk)
            out[("sink", "v", i)] = qz.f32_to_bf16_bits(vv)
        for pos, kk, vv in self.recent:
            sl = ring_slot(pos, self.S, self.R)
            out[("ring", "k", sl)] = qz.f32_to_bf16_bits(kk)
            out[("ring", "v", sl)] = qz.f32_to_bf16_bits(vv)
        return out
