"""fp64 decode attention over a (dequantized) KV cache (oracle; test infra).

One decode step of multi-head attention with grouped KV heads: query head h
reads kv head floor(h / G), G = n_q_heads / n_kv_heads.  For each query head

    s_t = tau * (q . k_hat_t),   p = softmax(s),   out = sum_t p_t v_hat_t

over every cached token (sink, dequantized tiles, recent window -- including
the token appended this step).

Sources: InnerQ (pith.science page for arXiv 2602.23200): its Algorithm 1
("multi-head attention with quantized cache in the decode phase") is cut off
on the page after its "Require" lines, so the standard scaled dot-product
decode step is taken, with tau = 1 / sqrt(head_dim) unless a scale is given;
the grouped-query layout follows the GQA reference the InnerQ page cites.
q is bf16 (widened exactly), the output is reported in fp32 by the library and
computed here in fp64.
"""

from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray, scale: float | None = None) -> np.ndarray:
    """q [G, D], k_hat/v_hat [T, D] (any float) -> out [G, D] fp64."""
    q = np.asarray(q, dtype=np.float64)
    k_hat = np.asarray(k_hat, dtype=np.float64)
    v_hat = np.asarray(v_hat, dtype=np.float64)
    d = q.shape[-1]
    tau = (1.0 / np.sqrt(d)) if not scale else float(scale)
    if k_hat.shape[0] == 0:
        return np.zeros_like(q)
    s = (q @ k_hat.T) * tau  # [G, T]
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v_hat


def decode_step(q_bh: np.ndarray, streams, scale: float | None = None) -> np.ndarray:
    """q_bh: [Hq, D] for one batch element of one layer; streams: the Hkv
    StreamCache objects of that (layer, batch).  Returns [Hq, D] fp64."""
    hq = q_bh.shape[0]
    hkv = len(streams)
    g = hq // hkv
    out = np.zeros((hq, q_bh.shape[1]))
    for kvh, st in enumerate(streams):
        kh, vh = st.dequantized()
        out[kvh * g : (kvh + 1) * g] = attend(q_bh[kvh * g : (kvh + 1) * g], kh, vh, scale)
    return out
