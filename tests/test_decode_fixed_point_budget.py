"""Error budget of the decode kernel's arithmetic (CPU model, no GPU).

The decode kernel multiplies integer codes on the tensor cores, so it rounds
two things the fp64 oracle keeps exact: the query, to 16-bit fixed point per
head (q_int = rint(q * 32639 / max|q_h|), the same q_int in the code and the
zero-point terms), and each tile probability, to p_int = rint(65535 * p) with
p taken relative to the running maximum of the work item's warp; every
product and tile sum after that is an exact integer.  This module models
exactly those two roundings -- with the kernel's split of the tiles into
contiguous ranges and of each range over four warps, each warp with its own
running maximum, and an exact log-sum-exp merge -- on a full-length
long-context stream, and checks that they alone stay well inside the parity
tolerance (max-abs 2e-3, rel-L2 1e-3) against the fp64 oracle.  The kernel's
fp32 epilogues add rounding several orders of magnitude smaller.
"""

import numpy as np
import torch

from oracle import attention as at
from oracle import cache as ca
from oracle import quantize as qz
from quantized_decode_attention_head_b200 import workloads

QMAX = 32639.0        # 16-bit query (two s8 terms)
QMAX3 = 8323072.0     # 24-bit query of K-normalized caches (three s8 terms)
PSCALE = 65535.0
LOG2E = 1.4426950408889634


def _bf16_to_f64(t):
    return qz.bf16_bits_to_f32(t.contiguous().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)


def _emulated_decode(q, kh, vh, S, Tq, n_splits, n_warps=4, rounding=True, nrm=None, qmax=QMAX):
    """Output [G, D] of the kernel's arithmetic model for one stream
    (rounding=False: q_int and p_int left unrounded).  nrm: the K
    normalization factors of a normalized cache -- the tiles hold K / n and
    the tile products use q * n (exact: powers of two), whose fixed point
    then spans the channels' whole range."""
    rint = np.rint if rounding else (lambda x: x)
    G, D = q.shape
    scale = 1.0 / np.sqrt(D)
    n = np.ones(D) if nrm is None else np.asarray(nrm, dtype=np.float64)
    q32 = (q * n).astype(np.float32)
    mx = np.abs(q32).max(axis=1, keepdims=True)
    inv = np.where(mx > 0, np.float32(qmax) / mx, np.float32(0)).astype(np.float32)
    q_int = np.clip(rint((q32 * inv).astype(np.float64)), -qmax, qmax)
    sq = (mx.astype(np.float64) / qmax)[:, 0]
    n_tiles = Tq // 32
    x_tiles = ((kh[S:S + Tq] / n) @ q_int.T) * sq * scale * LOG2E  # base-2 logits [Tq, G]
    parts = []  # (m [G], l [G], o [G, D])
    for item in range(n_splits):
        t0, t1 = item * n_tiles // n_splits, (item + 1) * n_tiles // n_splits
        for w in range(n_warps):
            m = np.full(G, -np.inf)
            l = np.zeros(G)
            o = np.zeros((G, D))
            for t in range(t0 + w, t1, n_warps):
                x = x_tiles[32 * t:32 * t + 32]  # [32, G]
                m_new = np.maximum(m, x.max(axis=0))
                a = np.where(np.isfinite(m), np.exp2(m - m_new), 0.0)
                o *= a[:, None]
                l *= a
                m = m_new
                p_int = rint(np.exp2(x - m) * PSCALE)  # [32, G]
                o += p_int.T @ vh[S + 32 * t:S + 32 * t + 32]
                l += p_int.sum(axis=0)
            parts.append((m, l / PSCALE, o / PSCALE))
    # bf16 sink + recent window: exact (the kernel uses fp32 FMAs on bf16 values)
    win = np.r_[0:S, S + Tq:kh.shape[0]]
    xw = (kh[win] @ q.T) * scale * LOG2E
    mw = xw.max(axis=0)
    pw = np.exp2(xw - mw)
    parts.append((mw, pw.sum(axis=0), pw.T @ vh[win]))
    M = np.max([p[0] for p in parts], axis=0)
    L = sum(p[1] * np.exp2(p[0] - M) for p in parts)
    O = sum(p[2] * np.exp2(p[0] - M)[:, None] for p in parts)
    return O / L[:, None]


def _stream(name, bits, k_norm=False, **over):
    wl = workloads.CONFIGS[name].with_(**over)
    one = wl.with_(n_layers=1, batch=1, n_kv_heads=1, n_q_heads=wl.group)
    k, v, f = workloads.kv_inputs(one, "cpu")
    q, _, _ = workloads.step_inputs(one, 1, f, "cpu")
    st = ca.StreamCache(wl.head_dim, bits, bits, wl.n_sink, wl.n_recent, k_norm=k_norm)
    st.prefill(_bf16_to_f64(k)[0, 0, 0].astype(np.float32), _bf16_to_f64(v)[0, 0, 0].astype(np.float32))
    kh, vh = st.dequantized()
    return wl, _bf16_to_f64(q)[0, 0, 0], kh, vh, st


def test_long_context_fixed_point_error_budget():
    """131072 tokens, K outlier channels lognormal(1.5), 2-bit K and V, 4
    query heads, 73 tile items as the automatic plan takes on a B200 (74
    resident CTAs per stream, one of them for the window)."""
    wl, q, kh, vh, st = _stream("long_128k", 2)
    S, Tq = wl.n_sink, st.n_tiles * 32
    got = _emulated_decode(q, kh, vh, S, Tq, n_splits=73)
    exp = at.attend(q, kh, vh)
    err = np.abs(got - exp).max()
    rel = np.linalg.norm(got - exp) / np.linalg.norm(exp)
    assert err < 1e-3 and rel < 5e-4, (err, rel)  # at most half of the parity tolerance


def test_fixed_point_model_is_exact_without_rounding():
    """Sanity of the model itself: with the two roundings removed the
    split/warp/merge structure reproduces the oracle up to the fp32 scaling
    of q (relative 1e-7), so the budget above measures the roundings."""
    wl, q, kh, vh, st = _stream("llama3_8b", 4)
    S, Tq = wl.n_sink, st.n_tiles * 32
    got = _emulated_decode(q, kh, vh, S, Tq, n_splits=6, rounding=False)
    exp = at.attend(q, kh, vh)
    assert np.abs(got - exp).max() < 1e-6
    # and the roundings are what moves it: rounded, the error is orders larger
    err = np.abs(_emulated_decode(q, kh, vh, S, Tq, n_splits=6) - exp).max()
    assert 1e-6 < err < 1e-3


def test_k_norm_fixed_point_error_budget():
    """A normalized cache (K / n in the tiles, q * n in the tile products) on
    the long-context workload itself (outlier sigma = 1.5): the query's fixed
    point now spans every channel's magnitude.  With the 24-bit query the
    kernel uses for normalized caches the error stays far under half the
    tolerance; a 16-bit query would lose more than ten times as much (the
    reason normalized caches take the three-term query).  54 tile items:
    the 24-bit kernel holds three CTAs per SM."""
    wl, q, kh, vh, st = _stream("long_128k", 2, k_norm=True)
    assert wl.k_sigma == 1.5
    exp = at.attend(q, kh, vh)
    got = _emulated_decode(q, kh, vh, wl.n_sink, st.n_tiles * 32, n_splits=54, nrm=st.nrm, qmax=QMAX3)
    err = np.abs(got - exp).max()
    rel = np.linalg.norm(got - exp) / np.linalg.norm(exp)
    assert err < 1e-3 and rel < 5e-4, (err, rel)
    got16 = _emulated_decode(q, kh, vh, wl.n_sink, st.n_tiles * 32, n_splits=54, nrm=st.nrm, qmax=QMAX)
    err16 = np.abs(got16 - exp).max()
    assert err16 > 10 * err, (err16, err)
