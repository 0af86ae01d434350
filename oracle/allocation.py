"""RateQuant per-head bit allocation (oracle; test infrastructure only).

Source: "RateQuant: Optimal Mixed-Precision KV Cache Quantization via
Rate-Distortion Theory" (paperlayer.ai summary of arXiv 2605.06675v2).

* §3.1 -- per-head distortion D_h(b) = alpha_h * beta_h**(-b), alpha > 0,
  beta > 1; minimise sum_h w_h D_h(b_h) subject to an average-bit budget;
  reverse waterfilling: allocation grows with log(sensitivity).
* App. B.1 -- free heads get the stationary allocation, heads outside the bit
  bounds are clipped, repeat (at most N rounds).
* App. B.2 (Thm 3) -- D_uniform / D_opt >= 1 (AM-GM).
* §3.3, App. B.3, App. U, W.7 -- integer allocation: start every head at
  b_min, repeatedly give one bit to the head with the largest weighted
  marginal gain (max-heap), optimal because the gains decrease in b.

Readings taken where the page is silent:

* The stationary point of the Lagrangian of sum w a beta^-b + lambda*(sum b)
  gives b_h(lambda) = log_beta_h(w_h alpha_h ln(beta_h) / lambda); it is
  clipped to [b_min, b_max] = [min S, max S] of the allowed set S.
* W.7 prints the marginal gain with a natural exponent (alpha e^{-beta b}
  (1 - e^{-beta})), which contradicts §3.1's D = alpha beta^-b; §3.1 is
  followed: Delta D_h(b) = alpha_h beta_h^-b (1 - 1/beta_h).
* For a non-contiguous allowed set (e.g. {2,3,4,8}) unit steps do not exist;
  the integer problem "minimise sum w D(b_h), b_h in S, sum b_h <= floor(N B)"
  is solved exactly by a multiple-choice knapsack DP.  Among allocations whose
  distortion is equal within a relative 1e-12 the lexicographically largest
  bit vector (in head order) is returned.
* An average budget outside [min S, max S] is infeasible (error).
"""

from __future__ import annotations

import heapq
import itertools
import math

import numpy as np


class InfeasibleBudget(ValueError):
    """avg_bits outside [min(S), max(S)]."""


def _as_arrays(w, alpha, beta):
    w = np.asarray(w, dtype=np.float64)
    alpha = np.broadcast_to(np.asarray(alpha, dtype=np.float64), w.shape).copy()
    beta = np.broadcast_to(np.asarray(beta, dtype=np.float64), w.shape).copy()
    if w.ndim != 1 or w.size == 0:
        raise ValueError("need a non-empty 1-D vector of head sensitivities")
    if np.any(w <= 0) or np.any(alpha <= 0) or np.any(beta <= 1):
        raise ValueError("need w > 0, alpha > 0, beta > 1 (RateQuant §3.1)")
    return w, alpha, beta


def distortion(w, alpha, beta, bits) -> float:
    """Weighted total distortion sum_h w_h alpha_h beta_h^-b_h (§3.1)."""
    w, alpha, beta = _as_arrays(w, alpha, beta)
    bits = np.asarray(bits, dtype=np.float64)
    return float(np.sum(w * alpha * np.power(beta, -bits)))


def stationary_bits(w, alpha, beta, log_lambda, b_min, b_max):
    """b_h(lambda) = clip(log_beta(w alpha ln beta / lambda), b_min, b_max)."""
    w, alpha, beta = _as_arrays(w, alpha, beta)
    ln_beta = np.log(beta)
    c = np.log(w * alpha * ln_beta)
    return np.clip((c - log_lambda) / ln_beta, b_min, b_max)


def waterfill_continuous(w, alpha, beta, avg_bits, b_min, b_max):
    """Exact continuous reverse waterfilling (§3.1, App. B.1).

    Sum_h b_h(nu) with nu = ln(lambda) is continuous, non-increasing and
    piecewise linear with breakpoints where a head hits b_max or b_min.  The
    breakpoints are sorted, the segment holding the budget N * avg_bits is
    found, and nu is solved in closed form on that segment's free set.

    Returns (bits[N] float64, nu = ln(lambda)).
    """
    w, alpha, beta = _as_arrays(w, alpha, beta)
    n = w.size
    if not (b_min <= avg_bits <= b_max):
        raise InfeasibleBudget(f"avg_bits {avg_bits} outside [{b_min}, {b_max}]")
    budget = n * float(avg_bits)
    ln_beta = np.log(beta)
    c = np.log(w * alpha * ln_beta)
    nu_hi = c - b_max * ln_beta  # nu <= nu_hi  -> head at b_max
    nu_lo = c - b_min * ln_beta  # nu >= nu_lo  -> head at b_min

    def total(nu):
        return float(np.sum(np.clip((c - nu) / ln_beta, b_min, b_max)))

    if b_min == b_max:
        return np.full(n, float(b_min)), float(np.max(nu_lo))
    points = np.sort(np.concatenate([nu_hi, nu_lo]))
    if budget >= n * b_max:
        return np.full(n, float(b_max)), float(points[0])
    if budget <= n * b_min:
        return np.full(n, float(b_min)), float(points[-1])
    # total() at the breakpoints is non-increasing; binary-search the first
    # breakpoint whose total is <= budget.  The solution lies between it and
    # the previous one.  total(points[0]) = N*b_max > budget and
    # total(points[-1]) = N*b_min < budget.
    lo_i, hi_i = 0, points.size - 1
    while hi_i - lo_i > 1:
        m = (lo_i + hi_i) // 2
        if total(points[m]) <= budget:
            hi_i = m
        else:
            lo_i = m
    k = hi_i
    lo_nu, hi_nu = points[k - 1], points[k]
    mid = 0.5 * (lo_nu + hi_nu)
    free = (nu_hi < mid) & (mid < nu_lo)
    at_max = nu_hi >= mid
    at_min = nu_lo <= mid
    clipped_bits = b_max * np.count_nonzero(at_max) + b_min * np.count_nonzero(at_min)
    inv = np.sum(1.0 / ln_beta[free])
    nu = (np.sum(c[free] / ln_beta[free]) - (budget - clipped_bits)) / inv
    bits = np.clip((c - nu) / ln_beta, b_min, b_max)
    return bits, float(nu)


def waterfill_bisection(w, alpha, beta, avg_bits, b_min, b_max, iters=200):
    """Cross-check: bisection on nu = ln(lambda) until sum b_h(nu) = budget."""
    w, alpha, beta = _as_arrays(w, alpha, beta)
    n = w.size
    if not (b_min <= avg_bits <= b_max):
        raise InfeasibleBudget(f"avg_bits {avg_bits} outside [{b_min}, {b_max}]")
    budget = n * float(avg_bits)
    ln_beta = np.log(beta)
    c = np.log(w * alpha * ln_beta)
    lo = float(np.min(c - b_max * ln_beta)) - 1.0
    hi = float(np.max(c - b_min * ln_beta)) + 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        s = float(np.sum(np.clip((c - mid) / ln_beta, b_min, b_max)))
        if s > budget:
            lo = mid
        else:
            hi = mid
    nu = 0.5 * (lo + hi)
    return np.clip((c - nu) / ln_beta, b_min, b_max), nu


def marginal_gain(w_h, alpha_h, beta_h, b):
    """Weighted distortion reduction of one more bit at b (W.7, §3.1 form)."""
    return w_h * alpha_h * beta_h ** (-b) * (1.0 - 1.0 / beta_h)


def greedy_heap(w, alpha, beta, b_min, b_max, budget_bits):
    """App. U: all heads start at b_min; pop the head with the largest
    marginal gain, give it one bit, push its next gain; stop when the
    remaining budget R reaches zero (or every head is at b_max).

    Valid for a contiguous allowed set {b_min, ..., b_max} (App. B.3).
    Equal gains are broken towards the lower head index.
    """
    w, alpha, beta = _as_arrays(w, alpha, beta)
    n = w.size
    bits = np.full(n, int(b_min), dtype=np.int64)
    remaining = int(budget_bits) - n * int(b_min)
    if remaining < 0:
        raise InfeasibleBudget("budget below N * b_min")
    heap = [(-marginal_gain(w[h], alpha[h], beta[h], b_min), h) for h in range(n)]
    heapq.heapify(heap)
    while remaining > 0 and heap:
        _, h = heapq.heappop(heap)
        bits[h] += 1
        remaining -= 1
        if bits[h] < b_max:
            heapq.heappush(heap, (-marginal_gain(w[h], alpha[h], beta[h], bits[h]), h))
    return bits


def integer_allocation_dp(w, alpha, beta, allowed, budget_bits, rel_tie=1e-12):
    """Exact integer allocation onto an arbitrary allowed set S.

    Minimise sum_h w_h alpha_h beta_h^-b_h over b_h in S with
    sum_h b_h <= budget_bits (multiple-choice knapsack, solved by dynamic
    programming over heads).  Near-ties (relative 1e-12) go to the
    lexicographically largest bit vector.
    """
    w, alpha, beta = _as_arrays(w, alpha, beta)
    S = sorted(set(int(b) for b in allowed))
    n = w.size
    budget = int(budget_bits)
    if budget < n * S[0]:
        raise InfeasibleBudget("budget below N * min(S)")
    budget = min(budget, n * S[-1])
    cost = np.array([[w[h] * alpha[h] * beta[h] ** (-b) for b in S] for h in range(n)])
    inf = np.inf
    # f[h][u]: min cost of heads h..n-1 using at most u bits.
    f = np.full((n + 1, budget + 1), inf)
    f[n, :] = 0.0
    for h in range(n - 1, -1, -1):
        best = np.full(budget + 1, inf)
        for j, b in enumerate(S):
            if b > budget:
                continue
            cand = np.full(budget + 1, inf)
            cand[b:] = f[h + 1, : budget + 1 - b] + cost[h, j]
            best = np.minimum(best, cand)
        f[h] = best
    bits = np.zeros(n, dtype=np.int64)
    u = budget
    for h in range(n):
        target = f[h, u]
        for j in range(len(S) - 1, -1, -1):  # largest bit width first
            b = S[j]
            if b > u:
                continue
            val = cost[h, j] + f[h + 1, u - b]
            if val <= target * (1.0 + rel_tie) + 1e-300:
                bits[h] = b
                u -= b
                break
        else:  # pragma: no cover - DP table guarantees a choice exists
            raise RuntimeError("DP backtrack failed")
    return bits


def brute_force(w, alpha, beta, allowed, budget_bits):
    """Enumerate all |S|^N allocations (tiny N only); return the minimum
    distortion and every optimal vector (within relative 1e-12)."""
    w, alpha, beta = _as_arrays(w, alpha, beta)
    S = sorted(set(int(b) for b in allowed))
    n = w.size
    if len(S) ** n > 2_000_000:
        raise ValueError("brute force too large")
    best = math.inf
    vecs = []
    for combo in itertools.product(S, repeat=n):
        if sum(combo) > budget_bits:
            continue
        d = float(np.sum(w * alpha * np.power(beta, -np.asarray(combo, dtype=np.float64))))
        if d < best * (1 - 1e-12):
            best, vecs = d, [combo]
        elif d <= best * (1 + 1e-12):
            vecs.append(combo)
    return best, [np.asarray(v, dtype=np.int64) for v in vecs]


def allocate(w, alpha, beta, avg_bits, allowed):
    """Full a1 step: continuous waterfilling on [min S, max S] plus the exact
    integer allocation with budget floor(N * avg_bits).

    Returns dict(b_cont, b_int, log_lambda, budget).
    """
    S = sorted(set(int(b) for b in allowed))
    w, alpha, beta = _as_arrays(w, alpha, beta)
    b_cont, nu = waterfill_continuous(w, alpha, beta, avg_bits, S[0], S[-1])
    budget = int(math.floor(w.size * avg_bits + 1e-9))
    b_int = integer_allocation_dp(w, alpha, beta, S, budget)
    return {"b_cont": b_cont, "b_int": b_int, "log_lambda": nu, "budget": budget}


def gain_ratio(w, alpha, beta, avg_bits, bits):
    """Thm 3 ratio D_uniform / D(bits) with D_uniform at b_h = avg_bits."""
    return distortion(w, alpha, beta, np.full(len(w), float(avg_bits))) / distortion(
        w, alpha, beta, bits
    )


def code_bytes(n_layers, n_kv_heads, head_dim, n_tokens, avg_bits, kv=2):
    """KV-cache size counting code bits only (RateQuant App. L / W.12 accounting:
    metadata excluded).  bf16 when avg_bits == 16."""
    return n_layers * n_kv_heads * head_dim * kv * n_tokens * avg_bits / 8.0
