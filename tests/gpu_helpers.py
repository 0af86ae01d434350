"""Shared plumbing of the GPU parity tests: build the same cache on the GPU
(through the C ABI) and in the oracle, and compare them.

Inputs come from quantized_decode_attention_head_b200.workloads (seeded);
bit widths come from the library's allocator for the GPU side and from the
oracle's allocator for the oracle side, and are asserted equal.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import allocation as al
from oracle import attention as at
from oracle import cache as ca
from oracle import quantize as qz
from quantized_decode_attention_head_b200 import QuantizedKVCache, rq_allocate_bits, workloads

MAX_ABS = 2e-3
REL_L2 = 1e-3


def to_f32(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor (any device) -> float32 numpy with the same values."""
    return qz.bf16_bits_to_f32(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def workload_bits(wl):
    """Per-(layer, kv-head) K and V bits: (library, oracle) pairs, asserted equal."""
    inp = workloads.allocation_inputs(wl)
    n = wl.n_layers * wl.n_kv_heads

    def both(w, a, b, avg):
        lib_bits = rq_allocate_bits(w, a, b, avg, wl.allowed)["b_int"]
        orc_bits = al.allocate(w, a, b, avg, wl.allowed)["b_int"]
        assert np.array_equal(lib_bits, orc_bits)
        return lib_bits.reshape(wl.n_layers, wl.n_kv_heads), orc_bits.reshape(wl.n_layers, wl.n_kv_heads)

    if "kv" in inp:
        lb, ob = both(*inp["kv"])
        return (lb, lb), (ob, ob)
    lk, ok = both(*inp["k"])
    lv, ov = both(*inp["v"])
    assert lk.size == n
    return (lk, lv), (ok, ov)


def make_cache(wl, k_bits, v_bits, max_tokens, k_norm=False, hybrid=False):
    return QuantizedKVCache(wl.n_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n_sink,
                            wl.n_recent, max_tokens, k_bits, v_bits, k_norm=k_norm, hybrid=hybrid)


def oracle_streams(wl, k_bits, v_bits, k_np, v_np, which, k_norm=False, hybrid=False):
    """Oracle StreamCache for each (l, b, h) in ``which`` from float32 inputs
    [L, B, H, T, D]."""
    out = {}
    for (l, b, h) in which:
        st = ca.StreamCache(wl.head_dim, int(k_bits[l, h]), int(v_bits[l, h]), wl.n_sink, wl.n_recent, k_norm=k_norm,
                            hybrid=hybrid)
        st.prefill(k_np[l, b, h], v_np[l, b, h])
        out[(l, b, h)] = st
    return out


def all_streams(wl):
    return [(l, b, h) for l in range(wl.n_layers) for b in range(wl.batch) for h in range(wl.n_kv_heads)]


def check_stream_bytes(cache: QuantizedKVCache, st: ca.StreamCache, l, b, h, tiles=None):
    """Tile records (all, or the given indices) and window rows must match bit for bit."""
    lay = cache.stream_layout(l, b, h)
    n, rb = lay["n_tiles"], lay["record_bytes"]
    assert n == st.n_tiles, (n, st.n_tiles)
    assert rb == qz.record_bytes(st.kb, st.vb, st.d)
    if n:
        if tiles is None:
            got = cache.buffer[lay["tile_offset"] : lay["tile_offset"] + n * rb].cpu().numpy().reshape(n, rb)
            exp = st.records()
            idx = np.arange(n)
        else:
            idx = np.asarray(sorted(set(int(i) for i in tiles if 0 <= i < n)))
            blk = cache.buffer[lay["tile_offset"] : lay["tile_offset"] + n * rb].view(-1, rb)
            got = blk[torch.as_tensor(idx, device=blk.device)].cpu().numpy()
            exp = np.stack([st.record(int(i)) for i in idx])
        bad = np.nonzero(np.any(got != exp, axis=1))[0]
        assert bad.size == 0, f"stream {(l, b, h)}: {bad.size} tile records differ, first tile {idx[bad[0]]}, " \
                              f"first byte {np.nonzero(got[bad[0]] != exp[bad[0]])[0][:8]}"
    d, S, ring = st.d, st.S, st.R + 32
    wb = (2 * S + 2 * ring) * d * 2
    win = cache.buffer[lay["window_offset"] : lay["window_offset"] + wb].cpu().numpy().view(np.uint16)
    for (kind, kv, slot), bits in st.window_rows().items():
        row = (slot + (S if kv == "v" else 0)) if kind == "sink" else (2 * S + slot + (ring if kv == "v" else 0))
        assert np.array_equal(win[row * d : (row + 1) * d], bits), (kind, kv, slot)
    assert np.array_equal(cache.k_norm_factors(l, b, h).cpu().numpy(), st.nrm)


def oracle_decode(wl, streams, q_np, which_lb):
    """fp64 oracle outputs {(l, b): [Hq, D]} for the (layer, batch) pairs given."""
    out = {}
    for (l, b) in which_lb:
        sts = [streams[(l, b, h)] for h in range(wl.n_kv_heads)]
        out[(l, b)] = at.decode_step(q_np[l, b], sts)
    return out


def assert_close(got: np.ndarray, exp: np.ndarray, what=""):
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    err = np.abs(got - exp)
    rel = np.linalg.norm(got - exp) / max(np.linalg.norm(exp), 1e-30)
    assert np.all(np.isfinite(got)), what
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)
