"""Synthetic workloads: shapes of the five benchmark caches and seeded inputs.

This module holds no arithmetic of the method.  It only fixes shapes and
draws random numbers; the CUDA library and the CPU oracle both receive what it
returns.  No model weights or datasets are used: the caches are shaped like
the attention layers of Llama-3-8B, Qwen3-8B and Mistral-7B and filled with
seeded random values.

Value laws (all drawn in fp32, then rounded to bf16):
  K[l,b,h,t,d] = N(0,1) * f[l,h,d],  f ~ lognormal(0, k_sigma) per (layer,
                 kv-head, channel), shared by batch elements and tokens
                 (outlier channels);
  V, q         = N(0,1);
  w (head sensitivity) ~ lognormal(0, 0.5); alpha = 1; beta per workload.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int
    n_sink: int
    n_recent: int
    k_sigma: float
    allowed: tuple
    avg_bits: float | None = None  # one budget shared by K and V
    k_avg_bits: float | None = None  # separate K / V budgets
    v_avg_bits: float | None = None
    beta: float = 4.4
    beta_range: tuple | None = None  # beta_h ~ U[lo, hi] per head
    beta_k: float | None = None
    beta_v: float | None = None
    w_sigma: float = 0.5
    decode_steps: int = 1
    seed: int = 0
    splits: tuple = field(default_factory=tuple)

    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads

    def with_(self, **kw):
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Workload(
        "tiny", n_layers=1, batch=1, n_q_heads=8, n_kv_heads=4, head_dim=64, context=512,
        n_sink=4, n_recent=32, k_sigma=1.0, allowed=(2, 3, 4, 8), avg_bits=2.5,
        beta=4.4, decode_steps=1, seed=0),
    "llama3_8b": Workload(
        "llama3_8b", n_layers=1, batch=8, n_q_heads=32, n_kv_heads=8, head_dim=128,
        context=4096, n_sink=4, n_recent=128, k_sigma=1.0, allowed=(2, 3, 4, 8),
        avg_bits=2.5, beta_range=(3.6, 5.3), decode_steps=64, seed=1),
    "qwen3_8b": Workload(
        "qwen3_8b", n_layers=36, batch=16, n_q_heads=32, n_kv_heads=8, head_dim=128,
        context=8192, n_sink=4, n_recent=128, k_sigma=1.0, allowed=(2, 3, 4, 8),
        k_avg_bits=3.0, v_avg_bits=2.0, beta_k=5.28, beta_v=4.92, decode_steps=1, seed=2),
    "long_128k": Workload(
        "long_128k", n_layers=1, batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
        context=131072, n_sink=4, n_recent=128, k_sigma=1.5, allowed=(2, 3, 4),
        avg_bits=2.0, beta=4.4, decode_steps=1, seed=3, splits=(64, 128, 256)),
    "mistral_7b_b64": Workload(
        "mistral_7b_b64", n_layers=1, batch=64, n_q_heads=32, n_kv_heads=8, head_dim=128,
        context=32768, n_sink=4, n_recent=128, k_sigma=1.0, allowed=(2, 4, 8),
        avg_bits=4.0, beta=4.4, decode_steps=1, seed=4),
}


def allocation_inputs(wl: Workload):
    """Seeded allocation inputs.

    Returns a dict with one entry per budget: {"kv": (w, alpha, beta, avg)} for
    a shared budget over the L*Hkv kv heads, or {"k": ..., "v": ...} for
    separate key / value budgets.  Arrays are float64 numpy.
    """
    rng = np.random.default_rng(1000 + wl.seed)
    n = wl.n_layers * wl.n_kv_heads
    out = {}
    if wl.avg_bits is not None:
        w = rng.lognormal(0.0, wl.w_sigma, n)
        if wl.beta_range is not None:
            beta = rng.uniform(wl.beta_range[0], wl.beta_range[1], n)
        else:
            beta = np.full(n, wl.beta)
        out["kv"] = (w, np.ones(n), beta, float(wl.avg_bits))
    else:
        wk = rng.lognormal(0.0, wl.w_sigma, n)
        wv = rng.lognormal(0.0, wl.w_sigma, n)
        out["k"] = (wk, np.ones(n), np.full(n, wl.beta_k), float(wl.k_avg_bits))
        out["v"] = (wv, np.ones(n), np.full(n, wl.beta_v), float(wl.v_avg_bits))
    return out


def kv_inputs(wl: Workload, device="cpu", n_tokens: int | None = None, seed: int | None = None):
    """Seeded bf16 prefill K, V [L, B, Hkv, T, D] and the per-(layer, kv-head,
    channel) outlier factors used for K.  Generated on ``device``."""
    import torch

    T = wl.context if n_tokens is None else n_tokens
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else seed)
    L, B, H, D = wl.n_layers, wl.batch, wl.n_kv_heads, wl.head_dim
    f = torch.exp(torch.randn((L, 1, H, 1, D), generator=g, device=device) * wl.k_sigma)
    k = torch.empty((L, B, H, T, D), dtype=torch.bfloat16, device=device)
    v = torch.empty((L, B, H, T, D), dtype=torch.bfloat16, device=device)
    for l in range(L):  # per layer keeps the fp32 temporaries small
        k[l] = (torch.randn((B, H, T, D), generator=g, device=device) * f[l]).to(torch.bfloat16)
        v[l] = torch.randn((B, H, T, D), generator=g, device=device).to(torch.bfloat16)
    return k, v, f


def step_inputs(wl: Workload, steps: int, f, device="cpu", seed: int | None = None):
    """Seeded per-step decode inputs: q [S, L, B, Hq, D], k_new/v_new
    [S, L, B, Hkv, D] (bf16).  ``f`` is the K outlier factor tensor of
    kv_inputs, so appended keys follow the same law."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(10_000 + (wl.seed if seed is None else seed))
    L, B, H, Hq, D = wl.n_layers, wl.batch, wl.n_kv_heads, wl.n_q_heads, wl.head_dim
    q = torch.randn((steps, L, B, Hq, D), generator=g, device=device).to(torch.bfloat16)
    fk = f.reshape(1, L, 1, H, D)
    kn = (torch.randn((steps, L, B, H, D), generator=g, device=device) * fk).to(torch.bfloat16)
    vn = torch.randn((steps, L, B, H, D), generator=g, device=device).to(torch.bfloat16)
    return q, kn, vn
