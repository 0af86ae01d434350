"""Per-quantizer distortion calibration (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "RateQuant: Optimal Mixed-Precision KV Cache Quantization via
Rate-Distortion Theory" (paperlayer.ai summary of arXiv 2605.06675v2):

- §1 "Method" and §3.4: a distortion model D(b) = alpha * beta^-b is fitted
  per quantizer from a small calibration set (here: per head, on that head's
  own K or V samples, with this library's group-wise quantizer), and K and V
  get separate curves;
- W.10: the exponential model fits most heads with R^2 > 0.98; a head whose
  fit has R^2 < 0.96 falls back to beta = min(beta_fitted, beta_bar);
- W.14: sensitivities are capped as w_i <- min(w_i, 5 * w_bar) before the
  allocation.

Readings (the summary gives no formulas for these): the fit is an ordinary
least-squares line through (b, ln D(b)), ln D = ln alpha - b ln beta, and R^2
is that line's coefficient of determination; beta_bar is the mean fitted beta
of the heads whose fit passes the R^2 threshold (all heads when none does);
w_bar is the mean of the uncapped sensitivities.  The distortion of a head at
b bits is the mean squared error of its samples after quantizing and
dequantizing them with this library's rule (oracle/quantize.py), in fp64.
"""

from __future__ import annotations

import numpy as np

from .quantize import TILE, quantize_groups


def head_mse(x: np.ndarray, b: int, role: str) -> float:
    """Mean squared quantization error of one head's samples x (float32
    [T, D], bf16 values; T a multiple of 32 for V) at b bits.  K groups: 32
    consecutive channels of a token; V groups: one channel over 32
    consecutive tokens."""
    x = np.asarray(x, dtype=np.float32)
    t, d = x.shape
    if role == "K":
        g = x.reshape(t, d // 32, 32)
        c, s, z = quantize_groups(g, b, axis=2)
        xh = c.astype(np.float64) * s.astype(np.float64)[..., None] + z.astype(np.float64)[..., None]
    elif role == "V":
        assert t % TILE == 0
        g = x.reshape(t // TILE, TILE, d)
        c, s, z = quantize_groups(g, b, axis=1)
        xh = c.astype(np.float64) * s.astype(np.float64)[:, None, :] + z.astype(np.float64)[:, None, :]
    else:
        raise ValueError(role)
    return float(np.mean((g.astype(np.float64) - xh) ** 2))


def fit_distortion(bits, mse):
    """Least-squares fit of ln D = ln alpha - b ln beta.  Returns (alpha,
    beta, r2).  Points with D <= 0 carry no information on a log scale and are
    left out; with fewer than two usable points the fit is undefined (nan)."""
    b = np.asarray(bits, dtype=np.float64)
    dv = np.asarray(mse, dtype=np.float64)
    ok = dv > 0
    if ok.sum() < 2:
        return float("nan"), float("nan"), float("nan")
    b, y = b[ok], np.log(dv[ok])
    bm, ym = b.mean(), y.mean()
    sxx = np.sum((b - bm) ** 2)
    slope = np.sum((b - bm) * (y - ym)) / sxx
    icpt = ym - slope * bm
    ss_res = np.sum((y - (icpt + slope * b)) ** 2)
    ss_tot = np.sum((y - ym) ** 2)
    r2 = 1.0 - ss_res / ss_tot if ss_tot > 0 else 1.0
    return float(np.exp(icpt)), float(np.exp(-slope)), float(r2)


def calibrate(bits, mse_table, r2_min: float = 0.96):
    """Per-head (alpha, beta, r2) from an [n_heads, n_bits] table of measured
    distortions, with the W.10 fallback beta = min(beta_fitted, beta_bar) for
    heads whose R^2 is below r2_min."""
    fits = [fit_distortion(bits, row) for row in np.asarray(mse_table, dtype=np.float64)]
    alpha = np.array([f[0] for f in fits])
    beta = np.array([f[1] for f in fits])
    r2 = np.array([f[2] for f in fits])
    good = r2 >= r2_min
    pool = beta[good] if good.any() else beta
    beta_bar = float(np.mean(pool))
    beta_out = np.where(good, beta, np.minimum(beta, beta_bar))
    return alpha, beta_out, r2


def cap_weights(w, factor: float = 5.0):
    """W.14: w_i <- min(w_i, factor * mean(w))."""
    w = np.asarray(w, dtype=np.float64)
    return np.minimum(w, factor * float(np.mean(w)))
