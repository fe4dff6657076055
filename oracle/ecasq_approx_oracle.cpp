// ECASQ oracle, part 2: the space-efficient approximation on the surrogate
// entropy H(I,B) and the iterative refinement.
//
// TEST INFRASTRUCTURE ONLY, like ecasq_oracle.cpp (same library, same rules):
// nothing on the product path includes, links or calls it. Plain fp64.
//
// Source: "Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)"
// technical summary (gist.science/pt/paper/2608.18147):
//   §2.3 "Algoritmo de Aproximação Eficiente em Espaço": optimise the joint
//        entropy H(I,B) of the interval index I and the rounding bit B instead of
//        H(X^); H(X^) <= H(I,B) <= H(X^) + 1, so the approximation at budget b
//        has MSE no larger than the optimum at budget b - 1; O(p + d) space.
//   §2.4 "Refinamento Iterativo": from the approximate code, optimise the subsets
//        Q0, Q1, Q2 of the values in turn, each in parallel, by binary search
//        inside its local interval; unbiasedness is kept.
//
// Readings where the page leaves a step open:
//   * (I, B) of an entry in [q_t, q_{t+1}] is (t, 0) with probability
//     1 - u and (t, 1) with probability u, u = (x - q_t)/(q_{t+1} - q_t); an
//     entry on an interior value q_t belongs to the interval that starts there
//     (the bucket rule). So P(I=t, B=0) = L(c_t,c_{t+1})/d, P(I=t, B=1) =
//     R(c_t,c_{t+1})/d and H(I,B) = sum_t h(L_t) + h(R_t).
//   * The approximation minimises MSE + lambda*H(I,B) exactly: the cost is a sum
//     of per-interval terms w(a,c) = V(a,c)/d + lambda*(h(L(a,c)) + h(R(a,c))),
//     minimised by a layered shortest path G_i(c) = min_{a<c} G_{i-1}(a) + w(a,c),
//     G_1(0) = 0; J_IB* = min_{2<=i<=s} G_i(p-1), |Q| = i. Ties: smallest a,
//     then smallest |Q|.
//   * Refinement works on the exact Lagrangian J = MSE + lambda*H(X^) at the
//     same lambda. Q0, Q1, Q2 are the interior values by position mod 3
//     (positions 1 .. m-2; the end values P_0, P_{p-1} stay). Moving the value at
//     position t changes only the intervals (t-1, t), (t, t+1) and the masses
//     mu_{t-1}, mu_t, mu_{t+1}, so values three positions apart move
//     independently. Each one searches its open interval (c_{t-1}, c_{t+1}) for
//     the minimum of its local cost by binary search on the sign of the forward
//     difference (exact for a unimodal local cost), and moves only on a strict
//     decrease. One iteration is the three classes in the order Q0, Q1, Q2; the
//     refinement stops after `iters` iterations or the first iteration that
//     moves nothing.
//   * Budget: the same bisection and two-way time-sharing as the exact solver.
//     The constrained rate is H(I,B) for the approximation alone (the quantity
//     it optimises, and the one the b - 1 guarantee is stated for) and H(X^) once
//     refined (the refinement optimises the exact objective).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

extern "C" {
int eo_bucket(const float* x, int64_t d, const double* P, int p, int64_t* cnt, double* A, double* B);
void eo_tables(const int64_t* cnt, const double* A, const double* B, const double* P, int p, double* V,
               double* R, double* L);
void eo_eval_tables(const double* V, const double* R, const double* L, int p, int64_t d, const int32_t* Q,
                    int m, double* mse, double* H, double* mu);
int eo_threads();
}

namespace {

const double kInfA = std::numeric_limits<double>::infinity();

double hm(double mu, double d) {
  if (!(mu > 0.0)) return 0.0;
  double q = mu / d;
  return -q * std::log2(q);
}

struct Tab {
  const double *V, *R, *L;
  int p;
  double d;
  double v(int a, int c) const { return V[int64_t(a) * p + c]; }
  double r(int a, int c) const { return R[int64_t(a) * p + c]; }
  double l(int a, int c) const { return L[int64_t(a) * p + c]; }
};

// Local exact cost of the value at position t placed at index c, with the other
// values of Q fixed: the two intervals that touch it and the three masses that
// depend on it (everything else in J does not depend on c).
double local_cost(const Tab& T, double lam, const int32_t* Q, int m, int t, int c) {
  const int a = Q[t - 1], e = Q[t + 1];
  double f = (T.v(a, c) + T.v(c, e)) / T.d;
  const double mu_prev = (t - 1 > 0 ? T.r(Q[t - 2], a) : 0.0) + T.l(a, c);
  const double mu_self = T.r(a, c) + T.l(c, e);
  const double mu_next = T.r(c, e) + (t + 1 < m - 1 ? T.l(e, Q[t + 2]) : 0.0);
  f += lam * (hm(mu_prev, T.d) + hm(mu_self, T.d) + hm(mu_next, T.d));
  return f;
}

// Binary search of the local cost over the open interval (c_{t-1}, c_{t+1}):
// step right while the next index is strictly cheaper.
int search_point(const Tab& T, double lam, const int32_t* Q, int m, int t) {
  int lo = Q[t - 1] + 1, hi = Q[t + 1] - 1;
  while (lo < hi) {
    const int mid = lo + (hi - lo) / 2;
    if (local_cost(T, lam, Q, m, t, mid + 1) < local_cost(T, lam, Q, m, t, mid))
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

}  // namespace

extern "C" {

// H(I,B) of a code Q from the tables: sum over intervals of h(L) + h(R).
double eo_hib_tables(const double* V, const double* R, const double* L, int p, int64_t d, const int32_t* Q,
                     int m) {
  (void)V;
  double s = 0.0;
  for (int t = 0; t + 1 < m; ++t) {
    s += hm(L[int64_t(Q[t]) * p + Q[t + 1]], double(d));
    s += hm(R[int64_t(Q[t]) * p + Q[t + 1]], double(d));
  }
  return s;
}

// Independent O(d) H(I,B) from the raw entries and the VALUES of Q: each entry in
// [q_i, q_{i+1}] (i the largest index <= m-2 with q_i <= x) adds 1 - u to the
// cell (i, down) and u to (i, up). Returns -2 if an entry is outside [q_0, q_{m-1}].
int eo_eval_raw_ib(const float* x, int64_t d, const double* q, int m, double* hib) {
  if (m < 2) {
    *hib = 0.0;
    return 0;
  }
  std::vector<double> dn(m - 1, 0.0), up(m - 1, 0.0);
  for (int64_t t = 0; t < d; ++t) {
    const double xv = x[t];
    if (!(xv >= q[0]) || !(xv <= q[m - 1])) return -2;
    const int i = int(std::upper_bound(q, q + (m - 1), xv) - q) - 1;
    const double u = (xv - q[i]) / (q[i + 1] - q[i]);
    dn[i] += 1.0 - u;
    up[i] += u;
  }
  double s = 0.0;
  for (int i = 0; i + 1 < m; ++i) s += hm(dn[i], double(d)) + hm(up[i], double(d));
  *hib = s;
  return 0;
}

// The approximation's DP (§2.3) over the permissible set, fp64.
// Outputs Q (m ascending indices), m and the DP's optimum of MSE + lambda*H(I,B).
int eo_approx_dp(const double* V, const double* R, const double* L, int p, int s, int64_t d, double lam,
                 int32_t* Q, int32_t* m_out, double* Jdp) {
  if (p < 2 || s < 2) return -1;
  if (s > p) s = p;
  const double dd = double(d);
  auto w = [&](int a, int c) {
    const int64_t e = int64_t(a) * p + c;
    return V[e] / dd + lam * (hm(L[e], dd) + hm(R[e], dd));
  };
  std::vector<double> G(size_t(s + 1) * p, kInfA);
  std::vector<int32_t> bp(size_t(s + 1) * p, -1);
  G[size_t(1) * p + 0] = 0.0;
  for (int i = 2; i <= s; ++i) {
    for (int c = i - 1; c <= p - 1; ++c) {
      double best = kInfA;
      int arg = -1;
      for (int a = i - 2; a < c; ++a) {
        const double g = G[size_t(i - 1) * p + a];
        if (!(g < kInfA)) continue;
        const double v = g + w(a, c);
        if (v < best) {
          best = v;
          arg = a;
        }
      }
      G[size_t(i) * p + c] = best;
      bp[size_t(i) * p + c] = arg;
    }
  }
  double bestJ = kInfA;
  int bi = -1;
  for (int i = 2; i <= s; ++i) {
    const double g = G[size_t(i) * p + (p - 1)];
    if (g < bestJ) {
      bestJ = g;
      bi = i;
    }
  }
  if (bi < 0) return -1;
  int c = p - 1;
  for (int i = bi; i >= 1; --i) {
    Q[i - 1] = c;
    c = bp[size_t(i) * p + c];
  }
  *m_out = bi;
  *Jdp = bestJ;
  return 0;
}

// Local exact cost of position t (1 <= t <= m-2) at index c; exposed for tests.
double eo_refine_local(const double* V, const double* R, const double* L, int p, int64_t d, double lam,
                       const int32_t* Q, int m, int t, int c) {
  Tab T{V, R, L, p, double(d)};
  return local_cost(T, lam, Q, m, t, c);
}

// Binary-search result for position t on the current Q; exposed for tests.
int eo_refine_point(const double* V, const double* R, const double* L, int p, int64_t d, double lam,
                    const int32_t* Q, int m, int t) {
  Tab T{V, R, L, p, double(d)};
  return search_point(T, lam, Q, m, t);
}

// Iterative refinement (§2.4) of Q in place. Returns the number of moves made;
// *iters_done is the number of iterations run.
int eo_refine(const double* V, const double* R, const double* L, int p, int64_t d, double lam, int32_t* Q,
              int m, int iters, int32_t* iters_done) {
  Tab T{V, R, L, p, double(d)};
  int moves = 0, it = 0;
  for (; it < iters; ++it) {
    int moved = 0;
    for (int cls = 0; cls < 3; ++cls) {
      // Positions of one class do not interact: taking them one after another
      // gives what a simultaneous update gives.
      for (int t = 1; t <= m - 2; ++t) {
        if ((t - 1) % 3 != cls) continue;
        const int c = search_point(T, lam, Q, m, t);
        if (c != Q[t] && local_cost(T, lam, Q, m, t, c) < local_cost(T, lam, Q, m, t, Q[t])) {
          Q[t] = c;
          ++moved;
        }
      }
    }
    moves += moved;
    if (moved == 0) {
      ++it;
      break;
    }
  }
  if (iters_done) *iters_done = it;
  return moves;
}

// One vector at one lambda: bucket, tables, the approximation's DP, optional
// refinement, and the fp64 evaluation. J is MSE + lambda*H(I,B) without
// refinement and MSE + lambda*H(X^) with it.
int eo_solve_approx(const float* x, int64_t d, const double* P, int p, int s, double lam, int refine,
                    int32_t* Q, int32_t* m, double* J, double* mse, double* H, double* hib) {
  if (P[0] == P[p - 1]) {
    for (int64_t t = 0; t < d; ++t)
      if (double(x[t]) != P[0]) return -2;
    Q[0] = 0;
    *m = 1;
    *J = *mse = *H = *hib = 0.0;
    return 0;
  }
  std::vector<int64_t> cnt(p - 1);
  std::vector<double> A(p - 1), B(p - 1), V(size_t(p) * p), R(size_t(p) * p), L(size_t(p) * p);
  int st = eo_bucket(x, d, P, p, cnt.data(), A.data(), B.data());
  if (st) return st;
  eo_tables(cnt.data(), A.data(), B.data(), P, p, V.data(), R.data(), L.data());
  double Jdp;
  st = eo_approx_dp(V.data(), R.data(), L.data(), p, s, d, lam, Q, m, &Jdp);
  if (st) return st;
  if (refine > 0) eo_refine(V.data(), R.data(), L.data(), p, d, lam, Q, *m, refine, nullptr);
  eo_eval_tables(V.data(), R.data(), L.data(), p, d, Q, *m, mse, H, nullptr);
  *hib = eo_hib_tables(V.data(), R.data(), L.data(), p, d, Q, *m);
  *J = *mse + lam * (refine > 0 ? *H : *hib);
  return 0;
}

// Entropy budget for the approximation: bisection on lambda and two-way
// time-sharing as in the exact solver, on the rate H(I,B) (refine == 0) or H(X^)
// (refine > 0). Reports both entropies of Q1 and Q2.
int eo_solve_approx_budget(const float* x, int64_t d, const double* P, int p, int s, double b, int steps,
                           int refine, int32_t* Q1, int32_t* m1, int32_t* Q2, int32_t* m2, double* theta,
                           double* lam_lo, double* lam_hi, double* H1, double* H2, double* hib1,
                           double* hib2, double* mse1, double* mse2, int32_t* status) {
  *status = 0;
  if (P[0] == P[p - 1]) {
    double J, mse, H, hib;
    int st = eo_solve_approx(x, d, P, p, s, 0.0, refine, Q1, m1, &J, &mse, &H, &hib);
    if (st) return st;
    Q2[0] = Q1[0];
    *m2 = *m1;
    *theta = *lam_lo = *lam_hi = 0.0;
    *H1 = *H2 = *hib1 = *hib2 = *mse1 = *mse2 = 0.0;
    return 0;
  }
  if (s > p) s = p;
  std::vector<int64_t> cnt(p - 1);
  std::vector<double> A(p - 1), B(p - 1), V(size_t(p) * p), R(size_t(p) * p), L(size_t(p) * p);
  int st = eo_bucket(x, d, P, p, cnt.data(), A.data(), B.data());
  if (st) return st;
  eo_tables(cnt.data(), A.data(), B.data(), P, p, V.data(), R.data(), L.data());
  std::vector<int32_t> q(s);
  int32_t mq = 0;
  double Jdp = 0, mse = 0, H = 0, hib = 0;
  auto solve_at = [&](double lam) {
    eo_approx_dp(V.data(), R.data(), L.data(), p, s, d, lam, q.data(), &mq, &Jdp);
    if (refine > 0) eo_refine(V.data(), R.data(), L.data(), p, d, lam, q.data(), mq, refine, nullptr);
    eo_eval_tables(V.data(), R.data(), L.data(), p, d, q.data(), mq, &mse, &H, nullptr);
    hib = eo_hib_tables(V.data(), R.data(), L.data(), p, d, q.data(), mq);
    return refine > 0 ? H : hib;
  };
  auto keep1 = [&]() {
    std::copy(q.begin(), q.begin() + mq, Q1);
    *m1 = mq;
    *H1 = H;
    *hib1 = hib;
    *mse1 = mse;
  };
  auto keep2 = [&]() {
    std::copy(q.begin(), q.begin() + mq, Q2);
    *m2 = mq;
    *H2 = H;
    *hib2 = hib;
    *mse2 = mse;
  };
  double lo = 0.0, hi = (P[p - 1] - P[0]) * (P[p - 1] - P[0]);
  double r1 = solve_at(lo), r2;
  keep1();
  if (r1 <= b) {
    keep2();
    *theta = *lam_lo = *lam_hi = 0.0;
    return 0;
  }
  r2 = solve_at(hi);
  keep2();
  if (r2 > b) {
    *theta = 0.0;
    *lam_lo = lo;
    *lam_hi = hi;
    *status = 1;
    return 0;
  }
  for (int it = 0; it < steps; ++it) {
    const double mid = 0.5 * (lo + hi);
    const double r = solve_at(mid);
    if (r > b) {
      lo = mid;
      r1 = r;
      keep1();
    } else {
      hi = mid;
      r2 = r;
      keep2();
    }
  }
  double th = (b - r2) / (r1 - r2);
  if (th < 0.0) th = 0.0;
  if (th > 1.0) th = 1.0;
  *theta = th;
  *lam_lo = lo;
  *lam_hi = hi;
  return 0;
}

// Batched drivers (OpenMP over vectors), as for the exact solver.
int eo_solve_approx_batch(const float* X, int n, int64_t d, const double* P, int p, int s, const double* lam,
                          int n_lam, int refine, int32_t* Q, int32_t* m, double* J, double* mse, double* H,
                          double* hib, int32_t* status) {
  const int S = std::min(s, p);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t w = 0; w < int64_t(n) * n_lam; ++w) {
    const int r = int(w / n_lam);
    std::vector<int32_t> q(S, -1);
    int32_t mm = 0;
    double jj = 0, ms = 0, hh = 0, hb = 0;
    int st = eo_solve_approx(X + int64_t(r) * d, d, P + int64_t(r) * p, p, s, lam[w], refine, q.data(), &mm,
                             &jj, &ms, &hh, &hb);
    for (int t = 0; t < s; ++t) Q[w * s + t] = (t < mm) ? q[t] : -1;
    m[w] = mm;
    J[w] = jj;
    mse[w] = ms;
    H[w] = hh;
    hib[w] = hb;
    status[w] = st;
  }
  return eo_threads();
}

int eo_solve_approx_budget_batch(const float* X, int n, int64_t d, const double* P, int p, int s, double b,
                                 int steps, int refine, int32_t* Q1, int32_t* m1, int32_t* Q2, int32_t* m2,
                                 double* theta, double* lam_lo, double* lam_hi, double* H1, double* H2,
                                 double* hib1, double* hib2, double* mse1, double* mse2, int32_t* status) {
  const int S = std::min(s, p);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    std::vector<int32_t> q1(S, -1), q2(S, -1);
    int32_t st = 0;
    int rc = eo_solve_approx_budget(X + int64_t(r) * d, d, P + int64_t(r) * p, p, s, b, steps, refine,
                                    q1.data(), &m1[r], q2.data(), &m2[r], &theta[r], &lam_lo[r], &lam_hi[r],
                                    &H1[r], &H2[r], &hib1[r], &hib2[r], &mse1[r], &mse2[r], &st);
    for (int t = 0; t < s; ++t) {
      Q1[int64_t(r) * s + t] = (t < m1[r]) ? q1[t] : -1;
      Q2[int64_t(r) * s + t] = (t < m2[r]) ? q2[t] : -1;
    }
    status[r] = rc ? rc : st;
  }
  return eo_threads();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Hardware-aware permissible set (§5 "Generalidade": any permissible alphabet,
// e.g. the values BF16 can represent). Reading: P is every finite BF16 value
// from the largest one <= min X to the smallest one >= max X (so that
// P_0 <= min X and P_{p-1} >= max X, as unbiasedness needs), ascending, with
// +0 and -0 counted once. Plain enumeration of all 65536 bit patterns.
extern "C" int eo_bf16_alphabet(const float* x, int64_t d, double* P, int p_max) {
  float lo = x[0], hi = x[0];
  for (int64_t t = 0; t < d; ++t) {
    if (!std::isfinite(x[t])) return -2;
    lo = std::min(lo, x[t]);
    hi = std::max(hi, x[t]);
  }
  std::vector<double> all;
  all.reserve(65536);
  for (uint32_t b = 0; b < 65536u; ++b) {
    const uint32_t w = b << 16;
    float f;
    std::memcpy(&f, &w, 4);
    if (std::isfinite(f)) all.push_back(double(f));
  }
  std::sort(all.begin(), all.end());
  all.erase(std::unique(all.begin(), all.end()), all.end());  // -0 == +0
  // largest value <= lo, smallest value >= hi
  auto it_lo = std::upper_bound(all.begin(), all.end(), double(lo));
  auto it_hi = std::lower_bound(all.begin(), all.end(), double(hi));
  if (it_lo == all.begin() || it_hi == all.end()) return -2;
  --it_lo;
  const int count = int(it_hi - it_lo) + 1;
  for (int i = 0; i < count && i < p_max; ++i) P[i] = *(it_lo + i);
  return count;
}
