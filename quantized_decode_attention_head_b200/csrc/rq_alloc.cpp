// RateQuant per-head bit allocation (host only).
//
// RateQuant (arXiv 2605.06675v2), §3.1: D_h(b) = alpha_h beta_h^-b; minimise
// sum_h w_h D_h(b_h) under an average-bit budget.  The stationary point of the
// Lagrangian gives b_h(nu) = (ln(w_h alpha_h ln beta_h) - nu) / ln beta_h with
// nu = ln(lambda) -- reverse waterfilling.
//
// Continuous solution: App. B.1's procedure -- give every free head its
// stationary allocation for the remaining budget, clip heads that leave
// [b_min, b_max], repeat (at most N rounds).  When heads leave on both sides
// in the same round, only the side with the larger total excess is clipped
// (variable fixing), which keeps every clip final.
//
// Integer solution: §3.3 / App. U greedy max-heap (one bit at a time to the
// largest weighted marginal gain w alpha beta^-b (1 - 1/beta), App. B.3 / W.7)
// when the allowed set is contiguous; an exact multiple-choice-knapsack
// dynamic programme otherwise.
#include <algorithm>
#include <cmath>
#include <queue>
#include <vector>

#include "rq.h"

namespace {

bool continuous(int n, const double* w, const double* alpha, const double* beta, double avg, double bmin,
                double bmax, std::vector<double>& bits, double& nu_out) {
  std::vector<double> c(n), lb(n);
  for (int h = 0; h < n; ++h) {
    lb[h] = std::log(beta[h]);
    c[h] = std::log(w[h] * alpha[h] * lb[h]);
  }
  std::vector<int> state(n, 0);  // 0 free, +1 at b_max, -1 at b_min
  bits.assign(n, 0.0);
  const double budget = n * avg;
  double nu = 0.0;
  for (int round = 0; round <= n; ++round) {
    double fixed = 0.0, num = 0.0, den = 0.0;
    int n_free = 0;
    for (int h = 0; h < n; ++h) {
      if (state[h] > 0) fixed += bmax;
      else if (state[h] < 0) fixed += bmin;
      else {
        num += c[h] / lb[h];
        den += 1.0 / lb[h];
        ++n_free;
      }
    }
    if (n_free == 0) break;
    nu = (num - (budget - fixed)) / den;
    double over = 0.0, under = 0.0;
    for (int h = 0; h < n; ++h) {
      if (state[h] != 0) continue;
      const double b = (c[h] - nu) / lb[h];
      if (b > bmax) over += b - bmax;
      if (b < bmin) under += bmin - b;
    }
    if (over == 0.0 && under == 0.0) break;
    const bool clip_high = over >= under;
    for (int h = 0; h < n; ++h) {
      if (state[h] != 0) continue;
      const double b = (c[h] - nu) / lb[h];
      if (clip_high && b > bmax) state[h] = 1;
      if (!clip_high && b < bmin) state[h] = -1;
    }
  }
  for (int h = 0; h < n; ++h) {
    if (state[h] > 0) bits[h] = bmax;
    else if (state[h] < 0) bits[h] = bmin;
    else bits[h] = std::min(bmax, std::max(bmin, (c[h] - nu) / lb[h]));
  }
  nu_out = nu;
  return true;
}

double gain(double w, double a, double be, int b) { return w * a * std::pow(be, -b) * (1.0 - 1.0 / be); }

void greedy(int n, const double* w, const double* alpha, const double* beta, int bmin, int bmax, long budget,
            int* out) {
  struct Item {
    double g;
    int h;
    bool operator<(const Item& o) const { return g < o.g || (g == o.g && h > o.h); }
  };
  std::priority_queue<Item> heap;
  long remaining = budget - (long)n * bmin;
  for (int h = 0; h < n; ++h) {
    out[h] = bmin;
    if (bmin < bmax) heap.push({gain(w[h], alpha[h], beta[h], bmin), h});
  }
  while (remaining > 0 && !heap.empty()) {
    const Item it = heap.top();
    heap.pop();
    ++out[it.h];
    --remaining;
    if (out[it.h] < bmax) heap.push({gain(w[it.h], alpha[it.h], beta[it.h], out[it.h]), it.h});
  }
}

void knapsack(int n, const double* w, const double* alpha, const double* beta, const std::vector<int>& S,
              long budget, int* out) {
  const long cap = std::min(budget, (long)n * S.back());
  const double inf = HUGE_VAL;
  // g[h][u]: least distortion of heads h..n-1 using at most u bits
  std::vector<double> g((size_t)(n + 1) * (cap + 1), inf);
  auto G = [&](int h, long u) -> double& { return g[(size_t)h * (cap + 1) + u]; };
  // distortion of head h at width S[j], computed once per (h, j)
  const int ns = (int)S.size();
  std::vector<double> dist((size_t)n * ns);
  for (int h = 0; h < n; ++h)
    for (int j = 0; j < ns; ++j) dist[(size_t)h * ns + j] = w[h] * alpha[h] * std::pow(beta[h], -S[j]);
  for (long u = 0; u <= cap; ++u) G(n, u) = 0.0;
  for (int h = n - 1; h >= 0; --h)
    for (long u = 0; u <= cap; ++u) {
      double best = inf;
      for (int j = 0; j < ns; ++j) {
        const int b = S[j];
        if (b > u) continue;
        const double v = G(h + 1, u - b) + dist[(size_t)h * ns + j];
        if (v < best) best = v;
      }
      G(h, u) = best;
    }
  long u = cap;
  for (int h = 0; h < n; ++h) {
    const double target = G(h, u);
    for (int j = (int)S.size() - 1; j >= 0; --j) {
      const int b = S[j];
      if (b > u) continue;
      const double v = G(h + 1, u - b) + dist[(size_t)h * ns + j];
      if (v <= target * (1.0 + 1e-12) + 1e-300) {
        out[h] = b;
        u -= b;
        break;
      }
    }
  }
}

}  // namespace

extern "C" rq_status rq_allocate_bits(int n, const double* w, const double* alpha, const double* beta,
                                      double avg_bits, const int* allowed, int n_allowed, double* b_cont,
                                      int* b_int, double* log_lambda) {
  if (n < 1 || !w || !alpha || !beta || !allowed || n_allowed < 1 || !b_int || !std::isfinite(avg_bits))
    return RQ_ERR_INVALID_ARG;
  for (int h = 0; h < n; ++h)
    if (!(w[h] > 0) || !(alpha[h] > 0) || !(beta[h] > 1) || !std::isfinite(w[h]) || !std::isfinite(alpha[h]) ||
        !std::isfinite(beta[h]))
      return RQ_ERR_INVALID_ARG;
  std::vector<int> S(allowed, allowed + n_allowed);
  std::sort(S.begin(), S.end());
  for (size_t i = 0; i < S.size(); ++i)
    if (S[i] < 1 || S[i] > 16 || (i > 0 && S[i] == S[i - 1])) return RQ_ERR_INVALID_ARG;
  const double bmin = S.front(), bmax = S.back();
  if (avg_bits < bmin || avg_bits > bmax) return RQ_ERR_INFEASIBLE_BUDGET;
  std::vector<double> bc;
  double nu = 0.0;
  if (bmin == bmax) {
    bc.assign(n, bmin);
  } else {
    continuous(n, w, alpha, beta, avg_bits, bmin, bmax, bc, nu);
  }
  const long budget = (long)std::floor(n * avg_bits + 1e-9);
  std::vector<int> bi(n);
  bool contiguous = true;
  for (size_t i = 1; i < S.size(); ++i) contiguous = contiguous && (S[i] == S[i - 1] + 1);
  if (contiguous)
    greedy(n, w, alpha, beta, S.front(), S.back(), budget, bi.data());
  else
    knapsack(n, w, alpha, beta, S, budget, bi.data());
  for (int h = 0; h < n; ++h) b_int[h] = bi[h];
  if (b_cont)
    for (int h = 0; h < n; ++h) b_cont[h] = bc[h];
  if (log_lambda) *log_lambda = nu;
  return RQ_OK;
}

// ------------------------------------------------------ distortion calibration
// RateQuant §1 / §3.4 (per-quantizer fit of D(b) = alpha * beta^-b), W.10
// (fallback beta = min(beta_fitted, beta_bar) for fits with R^2 < r2_min),
// W.14 (sensitivity cap).  The fit is the least-squares line through
// (b, ln D); points with D <= 0 are left out.

namespace {

// Fit of one head; returns false when fewer than two points are usable.
bool fit_one(const int* bits, const double* d, int n_bits, double& alpha, double& beta, double& r2) {
  double sb = 0.0, sy = 0.0;
  int m = 0;
  for (int i = 0; i < n_bits; ++i)
    if (d[i] > 0.0) {
      sb += bits[i];
      sy += std::log(d[i]);
      ++m;
    }
  if (m < 2) return false;
  const double bm = sb / m, ym = sy / m;
  double sxx = 0.0, sxy = 0.0, syy = 0.0;
  for (int i = 0; i < n_bits; ++i)
    if (d[i] > 0.0) {
      const double db = bits[i] - bm, dy = std::log(d[i]) - ym;
      sxx += db * db;
      sxy += db * dy;
      syy += dy * dy;
    }
  if (!(sxx > 0.0)) return false;
  const double slope = sxy / sxx;
  const double icpt = ym - slope * bm;
  double res = 0.0;
  for (int i = 0; i < n_bits; ++i)
    if (d[i] > 0.0) {
      const double e = std::log(d[i]) - (icpt + slope * bits[i]);
      res += e * e;
    }
  alpha = std::exp(icpt);
  beta = std::exp(-slope);
  r2 = syy > 0.0 ? 1.0 - res / syy : 1.0;
  return true;
}

}  // namespace

extern "C" rq_status rq_fit_distortion(int n_heads, const int* bits, int n_bits, const double* mse, double r2_min,
                                       double* alpha, double* beta, double* r2) {
  if (n_heads < 1 || n_bits < 2 || !bits || !mse || !alpha || !beta || !r2) return RQ_ERR_INVALID_ARG;
  std::vector<double> a(n_heads), b(n_heads), q(n_heads);
  for (int h = 0; h < n_heads; ++h)
    if (!fit_one(bits, mse + (size_t)h * n_bits, n_bits, a[h], b[h], q[h])) return RQ_ERR_INVALID_ARG;
  double sum_good = 0.0, sum_all = 0.0;
  int n_good = 0;
  for (int h = 0; h < n_heads; ++h) {
    sum_all += b[h];
    if (q[h] >= r2_min) {
      sum_good += b[h];
      ++n_good;
    }
  }
  const double beta_bar = n_good > 0 ? sum_good / n_good : sum_all / n_heads;
  for (int h = 0; h < n_heads; ++h) {
    alpha[h] = a[h];
    beta[h] = q[h] >= r2_min ? b[h] : std::min(b[h], beta_bar);
    r2[h] = q[h];
  }
  return RQ_OK;
}

extern "C" rq_status rq_cap_weights(int n, const double* w, double factor, double* w_out) {
  if (n < 1 || !w || !w_out || !(factor > 0.0)) return RQ_ERR_INVALID_ARG;
  double mean = 0.0;
  for (int i = 0; i < n; ++i) mean += w[i];
  mean /= n;
  const double cap = factor * mean;
  for (int i = 0; i < n; ++i) w_out[i] = std::min(w[i], cap);
  return RQ_OK;
}
