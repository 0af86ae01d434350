"""Pins for the allocation oracle (RateQuant §3.1, App. B.1-B.3, App. U, App. L).

Each test checks the oracle against something other than itself: the KKT
conditions of the constrained problem, a general-purpose convex solver, the
AM-GM closed form of Thm 3, brute-force enumeration, and the memory figures the
page prints.
"""

import json
import math
import os

import numpy as np
import pytest
from scipy.optimize import minimize

from oracle import allocation as al

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _instance(rng, n, per_head_beta=True):
    w = rng.lognormal(0.0, 0.8, n)
    alpha = rng.uniform(0.5, 2.0, n)
    beta = rng.uniform(3.6, 5.3, n) if per_head_beta else np.full(n, 4.4)
    return w, alpha, beta


@pytest.mark.parametrize("n", [2, 4, 8, 64, 288])
@pytest.mark.parametrize("avg", [2.1, 2.5, 3.0, 3.5, 5.0, 7.9])
def test_waterfill_budget_and_kkt(n, avg):
    rng = np.random.default_rng(n * 100 + int(avg * 10))
    w, a, be = _instance(rng, n)
    bits, nu = al.waterfill_continuous(w, a, be, avg, 2, 8)
    lam = math.exp(nu)
    assert abs(bits.sum() - n * avg) < 1e-9 * n
    # KKT of min sum w a be^-b + lam (sum b - budget), 2 <= b <= 8:
    # marginal m_h = w a ln(be) be^-b equals lam on free heads, >= lam at the
    # upper bound, <= lam at the lower bound.
    m = w * a * np.log(be) * be ** (-bits)
    free = (bits > 2 + 1e-9) & (bits < 8 - 1e-9)
    assert np.allclose(m[free], lam, rtol=1e-9)
    assert np.all(m[bits >= 8 - 1e-9] >= lam * (1 - 1e-9))
    assert np.all(m[bits <= 2 + 1e-9] <= lam * (1 + 1e-9))


@pytest.mark.parametrize("seed", range(5))
def test_waterfill_matches_generic_convex_solver(seed):
    rng = np.random.default_rng(seed)
    n = 8
    w, a, be = _instance(rng, n)
    avg = 2.5 + seed * 0.3
    bits, _ = al.waterfill_continuous(w, a, be, avg, 2, 8)
    res = minimize(
        lambda b: float(np.sum(w * a * be ** (-b))),
        x0=np.full(n, avg),
        jac=lambda b: -w * a * np.log(be) * be ** (-b),
        bounds=[(2, 8)] * n,
        constraints=[{"type": "eq", "fun": lambda b: b.sum() - n * avg, "jac": lambda b: np.ones(n)}],
        method="SLSQP",
        options={"ftol": 1e-15, "maxiter": 1000},
    )
    assert res.success
    d_ours = al.distortion(w, a, be, bits)
    assert d_ours <= res.fun * (1 + 1e-9)
    assert np.allclose(bits, res.x, atol=1e-4)


@pytest.mark.parametrize("seed", range(4))
def test_waterfill_bisection_agrees(seed):
    rng = np.random.default_rng(10 + seed)
    w, a, be = _instance(rng, 33)
    b1, nu1 = al.waterfill_continuous(w, a, be, 3.3, 2, 8)
    b2, nu2 = al.waterfill_bisection(w, a, be, 3.3, 2, 8)
    assert np.allclose(b1, b2, atol=1e-9)


def test_gain_ratio_equals_am_over_gm_when_unclipped():
    # Thm 3 (App. B.2): equal alpha, beta and no clipping give
    # D_uniform / D_opt = AM(w) / GM(w) exactly.
    rng = np.random.default_rng(7)
    w = rng.lognormal(0.0, 0.7, 50)
    bits, _ = al.waterfill_continuous(w, 1.0, 4.4, 3.0, -100, 100)
    ratio = al.gain_ratio(w, 1.0, 4.4, 3.0, bits)
    am, gm = w.mean(), math.exp(np.log(w).mean())
    assert abs(ratio - am / gm) < 1e-12 * ratio
    # and the optimum spreads bits by log_beta of the sensitivity (§3.1)
    assert np.allclose(np.diff(bits), np.diff(np.log(w) / math.log(4.4)), atol=1e-12)


def test_gain_ratio_lognormal_limit():
    # For ln w ~ N(0, sigma^2) the AM/GM ratio tends to exp(sigma^2 / 2).
    rng = np.random.default_rng(11)
    sigma = 0.5
    w = rng.lognormal(0.0, sigma, 400_000)
    bits, _ = al.waterfill_continuous(w, 1.0, 4.4, 3.0, -100, 100)
    ratio = al.gain_ratio(w, 1.0, 4.4, 3.0, bits)
    assert abs(ratio - math.exp(sigma**2 / 2)) < 0.01


def test_gain_ratio_is_one_when_floor_binds():
    # App. M.3: when the minimum-bit constraint floors all heads the gain ratio is exactly 1.
    rng = np.random.default_rng(3)
    w, a, be = _instance(rng, 8, per_head_beta=False)
    bits, _ = al.waterfill_continuous(w, a, be, 2.0, 2, 4)
    assert np.all(bits == 2.0)
    assert al.gain_ratio(w, a, be, 2.0, bits) == 1.0
    assert np.all(al.integer_allocation_dp(w, a, be, (2, 3, 4), 16) == 2)


def test_gain_ratio_at_least_one():
    rng = np.random.default_rng(5)
    for _ in range(20):
        w, a, be = _instance(rng, 16, per_head_beta=False)
        bits, _ = al.waterfill_continuous(w, a, be, 3.0, 2, 8)
        assert al.gain_ratio(w, a, be, 3.0, bits) >= 1.0 - 1e-12


@pytest.mark.parametrize("allowed", [(2, 3, 4, 8), (2, 4, 8), (2, 3, 4), (1, 2, 3, 4, 5, 6)])
@pytest.mark.parametrize("n", [1, 2, 3, 4])
def test_integer_dp_equals_brute_force(allowed, n):
    rng = np.random.default_rng(hash((allowed, n)) % 2**32)
    for trial in range(6):
        w, a, be = _instance(rng, n)
        lo, hi = min(allowed) * n, max(allowed) * n
        budget = int(rng.integers(lo, hi + 1))
        best, vecs = al.brute_force(w, a, be, allowed, budget)
        got = al.integer_allocation_dp(w, a, be, allowed, budget)
        d = al.distortion(w, a, be, got)
        assert abs(d - best) <= 1e-12 * best
        assert got.sum() <= budget
        assert set(got.tolist()) <= set(allowed)
        # tie-break: lexicographically largest optimal vector
        lex = max(tuple(v.tolist()) for v in vecs)
        assert tuple(got.tolist()) == lex


@pytest.mark.parametrize("seed", range(6))
def test_greedy_heap_optimal_for_contiguous_sets(seed):
    # App. B.3 / U: greedy by weighted marginal gain is optimal for contiguous S.
    rng = np.random.default_rng(100 + seed)
    n = [4, 8, 36, 64, 288, 17][seed]
    w, a, be = _instance(rng, n)
    for lo, hi in [(2, 4), (2, 8), (1, 6)]:
        budget = int(rng.integers(lo * n, hi * n + 1))
        g = al.greedy_heap(w, a, be, lo, hi, budget)
        dp = al.integer_allocation_dp(w, a, be, range(lo, hi + 1), budget)
        assert al.distortion(w, a, be, g) == pytest.approx(al.distortion(w, a, be, dp), rel=1e-12)
        assert g.sum() == min(budget, hi * n)


def test_integer_relaxation_bounds():
    rng = np.random.default_rng(9)
    for allowed in [(2, 3, 4, 8), (2, 4, 8), (2, 3, 4)]:
        for avg in [2.0, 2.5, 3.0, 4.0]:
            if avg > max(allowed):
                continue
            w, a, be = _instance(rng, 12)
            res = al.allocate(w, a, be, avg, allowed)
            d_int = al.distortion(w, a, be, res["b_int"])
            d_cont = al.distortion(w, a, be, res["b_cont"])
            assert d_int >= d_cont * (1 - 1e-12)
            if avg in allowed:
                d_uni = al.distortion(w, a, be, np.full(12, avg))
                assert d_int <= d_uni * (1 + 1e-12)


def test_infeasible_budget():
    w = np.ones(4)
    with pytest.raises(al.InfeasibleBudget):
        al.waterfill_continuous(w, 1.0, 4.4, 1.5, 2, 8)
    with pytest.raises(al.InfeasibleBudget):
        al.waterfill_continuous(w, 1.0, 4.4, 8.5, 2, 8)
    with pytest.raises(al.InfeasibleBudget):
        al.integer_allocation_dp(w, 1.0, 4.4, (2, 3), 7)


def test_memory_footprint_golden():
    spec = json.load(open(os.path.join(GOLDEN, "memory_footprint.json")))
    for c in spec["cases"]:
        got = al.code_bytes(c["n_layers"], c["n_kv_heads"], c["head_dim"], c["n_tokens"], c["bits"])
        assert got / 2**20 == pytest.approx(c["mib"], rel=1e-12), c["model"]
