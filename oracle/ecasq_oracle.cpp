// ECASQ oracle: a plain, slow, fp64 CPU statement of what the solver computes.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or
// call this file: only tests/, __graft_entry__.smoke() and bench.py's
// cpu_baseline / reference leg use it, through oracle/oracle.py. It shares no
// code, header, table or constant generator with the CUDA library.
//
// Source of every definition: "Entropy-Constrained Adaptive Stochastic
// Quantization (ECASQ)" technical summary (gist.science/pt/paper/2608.18147):
//   §1 "O Problema ECASQ"      choose Q subset of P, |Q| <= s, minimise MSE with
//                              E[X^] = X and H(X^) <= b
//   §2.1 "Relaxação Lagrangiana" minimise MSE(Q,X) + lambda*H(X^); varying lambda
//                              traces the Pareto curve; two-way time-sharing of
//                              two quantizers on a random partition hits any b
//   §2.2 "Programação Dinâmica" state dp_OPT(i, l, j): best prefix ending at value
//                              l, plus the MSE of [x_l, x_j] with l, j consecutive
//   §2.2 "Generalização"       arbitrary permissible set P, O(p^2 s + d)
//
// Readings where the page is silent:
//   * MSE is the per-entry mean; H is in bits per entry and is the entropy of the
//     EXPECTED output distribution mu/d of the stochastic quantizer.
//   * Q always holds P_0 and P_{p-1} (unbiasedness needs q_1 <= min X and
//     q_m >= max X; the grids used here span exactly [min X, max X]).
//   * Ties: strict '<' over ascending k keeps the smallest k; over layers the
//     smallest |Q| wins, then the smallest k.
//   * lambda search: bracket [0, (P_{p-1}-P_0)^2], arithmetic bisection,
//     "H(lambda_mid) > b  =>  lambda_lo = lambda_mid".
//   * Time-sharing: a per-entry Bernoulli(theta) selector from Philox stream 1.
//   * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): key = seed (lo, hi),
//     counter = (j >> 2, vector, stream, 0), output word j & 3, u = r * 2^-32;
//     an entry rounds up iff u * (q_hi - q_lo) < x - q_lo.
//
// Compiled with -O2 -fno-fast-math -ffp-contract=off so that the encoder's
// rounding test is exactly two IEEE subtractions and one IEEE product.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const double kInf = std::numeric_limits<double>::infinity();

// Compensated (Kahan) summation, used for the per-bucket moments.
struct Kahan {
  double s = 0.0, c = 0.0;
  void add(double x) {
    double y = x - c;
    double t = s + y;
    c = (t - s) - y;
    s = t;
  }
};

// Per-entry entropy contribution of an output value that receives expected mass
// mu out of d entries: -(mu/d) log2(mu/d), with 0 log 0 = 0 (§1, H(X^)).
double h_mass(double mu, double d) {
  if (!(mu > 0.0)) return 0.0;
  double q = mu / d;
  return -q * std::log2(q);
}

// Bucket of x on the alphabet P: the largest k <= p-2 with P_k <= x, so the last
// bucket [P_{p-2}, P_{p-1}] is closed. Returns -1 when x lies outside [P_0, P_{p-1}].
int bucket_of(double x, const double* P, int p) {
  if (!(x >= P[0]) || !(x <= P[p - 1])) return -1;
  // upper_bound over P[0..p-2]: first element strictly greater than x.
  const double* it = std::upper_bound(P, P + (p - 1), x);
  return int(it - P) - 1;
}

}  // namespace

extern "C" {

int eo_version() { return 1; }

// ---------------------------------------------------------------------------
// Grid: P_k = lo + (hi - lo) * k / (p - 1), P_{p-1} = hi, lo = min X, hi = max X
// (the uniform permissible set of the workloads). Returns 0, or -2 if X holds a
// NaN or an infinity.
int eo_uniform_grid(const float* x, int64_t d, int p, double* P) {
  float lo = x[0], hi = x[0];
  for (int64_t t = 0; t < d; ++t) {
    if (!std::isfinite(x[t])) return -2;
    lo = std::min(lo, x[t]);
    hi = std::max(hi, x[t]);
  }
  const double dlo = lo, dhi = hi;
  for (int k = 0; k < p - 1; ++k) P[k] = dlo + (dhi - dlo) * double(k) / double(p - 1);
  P[p - 1] = dhi;
  return 0;
}

// Per-bucket statistics: cnt_k, A_k = sum (x - P_k), B_k = sum (x - P_k)^2 over
// the entries of bucket k (k = 0 .. p-2). This is the "+d" pass of §2.2.
int eo_bucket(const float* x, int64_t d, const double* P, int p, int64_t* cnt, double* A,
              double* B) {
  std::vector<Kahan> ka(p - 1), kb(p - 1);
  for (int k = 0; k < p - 1; ++k) cnt[k] = 0;
  for (int64_t t = 0; t < d; ++t) {
    double xv = x[t];
    int k = bucket_of(xv, P, p);
    if (k < 0) return -2;
    double y = xv - P[k];
    cnt[k] += 1;
    ka[k].add(y);
    kb[k].add(y * y);
  }
  for (int k = 0; k < p - 1; ++k) {
    A[k] = ka[k].s;
    B[k] = kb[k].s;
  }
  return 0;
}

// Interval tables for every pair a < c (row-major [p][p], entries with a >= c are 0):
//   N  = number of entries in [P_a, P_c)   (buckets a .. c-1)
//   T1 = sum (x - P_a),  T2 = sum (x - P_a)^2,  W = P_c - P_a
//   V  = sum (P_c - x)(x - P_a) = W*T1 - T2     (variance of stochastic rounding)
//   R  = T1 / W  expected number of entries rounded UP to P_c
//   L  = N - R   expected number rounded DOWN to P_a
// Each pair is summed directly over its buckets (O(p^3)): no prefix sums.
void eo_tables(const int64_t* cnt, const double* A, const double* B, const double* P, int p,
               double* V, double* R, double* L) {
  for (int64_t i = 0; i < int64_t(p) * p; ++i) V[i] = R[i] = L[i] = 0.0;
  for (int a = 0; a < p; ++a) {
    for (int c = a + 1; c < p; ++c) {
      double N = 0.0, T1 = 0.0, T2 = 0.0;
      for (int k = a; k < c; ++k) {
        double dk = P[k] - P[a];
        double n = double(cnt[k]);
        N += n;
        T1 += A[k] + n * dk;
        T2 += B[k] + 2.0 * dk * A[k] + n * dk * dk;
      }
      double W = P[c] - P[a];
      double v = W * T1 - T2;
      if (v < 0.0) v = 0.0;
      double r = (W > 0.0) ? T1 / W : 0.0;
      V[a * p + c] = v;
      R[a * p + c] = r;
      L[a * p + c] = N - r;
    }
  }
}

// Objective of a code Q (indices c_0 < ... < c_{m-1} into P) from the tables:
// MSE = sum V / d, masses mu_0 = L(c_0,c_1), mu_t = R(c_{t-1},c_t) + L(c_t,c_{t+1}),
// mu_{m-1} = R(c_{m-2},c_{m-1}); H = sum h(mu_t). Writes mu[m] when mu != null.
void eo_eval_tables(const double* V, const double* R, const double* L, int p, int64_t d,
                    const int32_t* Q, int m, double* mse, double* H, double* mu) {
  double sv = 0.0, sh = 0.0;
  if (m <= 1) {
    if (mu && m == 1) mu[0] = double(d);
    *mse = 0.0;
    *H = 0.0;
    return;
  }
  for (int t = 0; t + 1 < m; ++t) sv += V[Q[t] * p + Q[t + 1]];
  for (int t = 0; t < m; ++t) {
    double u = 0.0;
    if (t > 0) u += R[Q[t - 1] * p + Q[t]];
    if (t + 1 < m) u += L[Q[t] * p + Q[t + 1]];
    if (mu) mu[t] = u;
    sh += h_mass(u, double(d));
  }
  *mse = sv / double(d);
  *H = sh;
}

// Independent O(d) evaluation straight from the raw entries and the VALUES of Q
// (no buckets, no tables): each x in [q_t, q_{t+1}] goes up with probability
// (x - q_t)/(q_{t+1} - q_t); its variance is (q_{t+1} - x)(x - q_t).
// Returns -2 if an entry lies outside [q_0, q_{m-1}].
int eo_eval_raw(const float* x, int64_t d, const double* q, int m, double* mse, double* H,
                double* mu) {
  std::vector<double> acc(std::max(m, 1), 0.0);
  double sv = 0.0;
  if (m == 1) {
    for (int64_t t = 0; t < d; ++t)
      if (double(x[t]) != q[0]) return -2;
    acc[0] = double(d);
  } else {
    for (int64_t t = 0; t < d; ++t) {
      double xv = x[t];
      if (!(xv >= q[0]) || !(xv <= q[m - 1])) return -2;
      int i = int(std::upper_bound(q, q + (m - 1), xv) - q) - 1;  // q_i <= x, i <= m-2
      double w = q[i + 1] - q[i];
      double up = (xv - q[i]) / w;
      sv += (q[i + 1] - xv) * (xv - q[i]);
      acc[i] += 1.0 - up;
      acc[i + 1] += up;
    }
  }
  double sh = 0.0;
  for (int t = 0; t < m; ++t) {
    if (mu) mu[t] = acc[t];
    sh += h_mass(acc[t], double(d));
  }
  *mse = sv / double(d);
  *H = sh;
  return 0;
}

// The exact Lagrangian DP of §2.2 over the permissible set.
// F_i(l, j): least cost of codes whose i-th value (counted from c_1 = 0) is P_l
// and whose next value is P_j; it holds V/d of every interval up to [l, j] and
// lambda*h of the masses of the first i values (the mass of P_l needs both of its
// neighbours, which is why the state is the pair (l, j)).
//   F_1(0, j) = V(0,j)/d + lambda*h(L(0,j))
//   F_i(l, j) = V(l,j)/d + min_k [ F_{i-1}(k,l) + lambda*h(R(k,l) + L(l,j)) ]
//   J*        = min_{i,k} F_i(k, p-1) + lambda*h(R(k, p-1)),  |Q| = i + 1 <= s.
// Outputs Q (m indices, ascending), m, and the DP's own optimum Jdp.
// Returns 0; -1 on bad arguments.
int eo_dp(const double* V, const double* R, const double* L, int p, int s, int64_t d,
          double lam, int32_t* Q, int32_t* m_out, double* Jdp) {
  if (p < 2 || s < 2) return -1;
  if (s > p) s = p;
  const double dd = double(d);
  auto at = [p](int a, int c) { return int64_t(a) * p + c; };
  // Layers 1 .. s-1; every layer holds a full [p][p] plane, +inf where undefined.
  std::vector<double> F(size_t(s) * p * p, kInf);
  std::vector<int32_t> bp(size_t(s) * p * p, -1);
  auto Fi = [&](int i, int l, int j) -> double& { return F[(size_t(i) * p + l) * p + j]; };
  auto Bi = [&](int i, int l, int j) -> int32_t& { return bp[(size_t(i) * p + l) * p + j]; };

  for (int j = 1; j < p; ++j) Fi(1, 0, j) = V[at(0, j)] / dd + lam * h_mass(L[at(0, j)], dd);

  for (int i = 2; i <= s - 1; ++i) {
    const bool last = (i == s - 1);
    for (int l = i - 1; l <= p - 2; ++l) {
      const int j0 = last ? p - 1 : l + 1;
      for (int j = j0; j <= p - 1; ++j) {
        double best = kInf;
        int arg = -1;
        for (int k = 0; k < l; ++k) {
          double g = Fi(i - 1, k, l);
          if (!(g < kInf)) continue;  // state not reachable with i-1 values
          double c = g + lam * h_mass(R[at(k, l)] + L[at(l, j)], dd);
          if (c < best) {
            best = c;
            arg = k;
          }
        }
        if (arg >= 0) {
          Fi(i, l, j) = V[at(l, j)] / dd + best;
          Bi(i, l, j) = arg;
        }
      }
    }
  }

  double bestE = kInf;
  int bi = -1, bk = -1;
  for (int i = 1; i <= s - 1; ++i) {
    for (int k = 0; k <= p - 2; ++k) {
      double f = Fi(i, k, p - 1);
      if (!(f < kInf)) continue;
      double e = f + lam * h_mass(R[at(k, p - 1)], dd);
      if (e < bestE) {
        bestE = e;
        bi = i;
        bk = k;
      }
    }
  }
  if (bi < 0) return -1;
  // Backtrack: values c_1 .. c_{bi+1}.
  std::vector<int32_t> path(bi + 1);
  path[bi] = p - 1;
  path[bi - 1] = bk;
  int l = bk, j = p - 1;
  for (int i = bi; i >= 2; --i) {
    int k = Bi(i, l, j);
    path[i - 2] = k;
    j = l;
    l = k;
  }
  for (int t = 0; t <= bi; ++t) Q[t] = path[t];
  *m_out = bi + 1;
  *Jdp = bestE;
  return 0;
}

// Whole single-vector solve at one lambda: bucket, tables, DP, backtrack and an
// fp64 evaluation of the chosen Q from the tables.
// Degenerate P_0 == P_{p-1} (constant vector): Q = {0}, J = 0.
int eo_solve(const float* x, int64_t d, const double* P, int p, int s, double lam, int32_t* Q,
             int32_t* m, double* J, double* mse, double* H) {
  if (P[0] == P[p - 1]) {
    for (int64_t t = 0; t < d; ++t)
      if (double(x[t]) != P[0]) return -2;
    Q[0] = 0;
    *m = 1;
    *J = *mse = *H = 0.0;
    return 0;
  }
  std::vector<int64_t> cnt(p - 1);
  std::vector<double> A(p - 1), B(p - 1), V(size_t(p) * p), R(size_t(p) * p), L(size_t(p) * p);
  int st = eo_bucket(x, d, P, p, cnt.data(), A.data(), B.data());
  if (st) return st;
  eo_tables(cnt.data(), A.data(), B.data(), P, p, V.data(), R.data(), L.data());
  double Jdp;
  st = eo_dp(V.data(), R.data(), L.data(), p, s, d, lam, Q, m, &Jdp);
  if (st) return st;
  eo_eval_tables(V.data(), R.data(), L.data(), p, d, Q, *m, mse, H, nullptr);
  *J = *mse + lam * (*H);
  return 0;
}

// Entropy budget b (§1, §2.1): lambda bisection plus two-way time-sharing.
// Q1 is the solution at the final lambda_lo (H1 > b), Q2 the one at lambda_hi
// (H2 <= b); theta = (b - H2)/(H1 - H2) is the share of entries coded with Q1.
// Status: 0, or +1 when even lambda_hi leaves H > b (then Q2 = Q(lambda_hi), theta = 0).
// When H(lambda = 0) <= b the budget is slack: Q1 = Q2 = Q(0), theta = 0.
int eo_solve_budget(const float* x, int64_t d, const double* P, int p, int s, double b, int steps,
                    int32_t* Q1, int32_t* m1, int32_t* Q2, int32_t* m2, double* theta,
                    double* lam_lo, double* lam_hi, double* H1, double* H2, double* mse1,
                    double* mse2, int32_t* status) {
  *status = 0;
  if (P[0] == P[p - 1]) {
    double J, mse, H;
    int st = eo_solve(x, d, P, p, s, 0.0, Q1, m1, &J, &mse, &H);
    if (st) return st;
    Q2[0] = Q1[0];
    *m2 = *m1;
    *theta = 0.0;
    *lam_lo = *lam_hi = 0.0;
    *H1 = *H2 = 0.0;
    *mse1 = *mse2 = 0.0;
    return 0;
  }
  if (s > p) s = p;
  std::vector<int64_t> cnt(p - 1);
  std::vector<double> A(p - 1), B(p - 1), V(size_t(p) * p), R(size_t(p) * p), L(size_t(p) * p);
  int st = eo_bucket(x, d, P, p, cnt.data(), A.data(), B.data());
  if (st) return st;
  eo_tables(cnt.data(), A.data(), B.data(), P, p, V.data(), R.data(), L.data());
  std::vector<int32_t> q(s);
  int32_t mq;
  double Jdp, mse, H;
  auto solve_at = [&](double lam) {
    eo_dp(V.data(), R.data(), L.data(), p, s, d, lam, q.data(), &mq, &Jdp);
    eo_eval_tables(V.data(), R.data(), L.data(), p, d, q.data(), mq, &mse, &H, nullptr);
  };
  double lo = 0.0, hi = (P[p - 1] - P[0]) * (P[p - 1] - P[0]);
  solve_at(lo);
  std::copy(q.begin(), q.begin() + mq, Q1);
  *m1 = mq;
  *H1 = H;
  *mse1 = mse;
  if (H <= b) {  // the budget does not bind
    std::copy(q.begin(), q.begin() + mq, Q2);
    *m2 = mq;
    *H2 = H;
    *mse2 = mse;
    *theta = 0.0;
    *lam_lo = *lam_hi = 0.0;
    return 0;
  }
  solve_at(hi);
  std::copy(q.begin(), q.begin() + mq, Q2);
  *m2 = mq;
  *H2 = H;
  *mse2 = mse;
  if (H > b) {  // not reachable inside the bracket
    *theta = 0.0;
    *lam_lo = lo;
    *lam_hi = hi;
    *status = 1;
    return 0;
  }
  for (int it = 0; it < steps; ++it) {
    double mid = 0.5 * (lo + hi);
    solve_at(mid);
    if (H > b) {
      lo = mid;
      std::copy(q.begin(), q.begin() + mq, Q1);
      *m1 = mq;
      *H1 = H;
      *mse1 = mse;
    } else {
      hi = mid;
      std::copy(q.begin(), q.begin() + mq, Q2);
      *m2 = mq;
      *H2 = H;
      *mse2 = mse;
    }
  }
  double th = (b - *H2) / (*H1 - *H2);
  if (th < 0.0) th = 0.0;
  if (th > 1.0) th = 1.0;
  *theta = th;
  *lam_lo = lo;
  *lam_hi = hi;
  return 0;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 counter-based generator (Salmon et al., SC'11): ten rounds of
//   (c0,c1,c2,c3) -> (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0))
// with the key bumped by the Weyl constants between rounds. The 64-bit-word
// variant with the same structure is exposed for a structural check against a
// library implementation.
void eo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3], k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    uint64_t p0 = uint64_t(M0) * c0, p1 = uint64_t(M1) * c2;
    uint32_t n0 = uint32_t(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = uint32_t(p1);
    uint32_t n2 = uint32_t(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = uint32_t(p0);
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

void eo_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
  const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3], k0 = key[0], k1 = key[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    unsigned __int128 p0 = (unsigned __int128)M0 * c0, p1 = (unsigned __int128)M1 * c2;
    uint64_t n0 = uint64_t(p1 >> 64) ^ c1 ^ k0;
    uint64_t n1 = uint64_t(p1);
    uint64_t n2 = uint64_t(p0 >> 64) ^ c3 ^ k1;
    uint64_t n3 = uint64_t(p0);
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// Uniform word for entry j of vector v on a stream: counter (j>>2, v, stream, 0),
// key (seed lo, seed hi), output word j & 3.
static uint32_t philox_word(uint64_t seed, int64_t j, uint32_t v, uint32_t stream) {
  uint32_t ctr[4] = {uint32_t(uint64_t(j) >> 2), v, stream, 0u};
  uint32_t key[2] = {uint32_t(seed), uint32_t(seed >> 32)};
  uint32_t out[4];
  eo_philox4x32_10(ctr, key, out);
  return out[j & 3];
}

// Unbiased stochastic rounding of one vector (§1: E[X^] = X) with optional
// two-way time-sharing (§2.1). Q1/Q2 are P indices. Which code an entry uses:
//   * Q2 == null: Q1 for every entry (part 0).
//   * Q2 != null and 0 < theta < 1: Q1 when u_sel(j) < theta (Philox stream 1),
//     else Q2 (part 1).
//   * Q2 != null otherwise: theta >= 1 gives Q1 only, theta <= 0 Q2 only.
// An entry in [q_i, q_{i+1}] rounds up when u(j) * (q_{i+1} - q_i) < x - q_i
// (Philox stream 0): the test u < (x - q_i)/(q_{i+1} - q_i) with the division
// moved to the other side, each side a single IEEE operation. x = q_i never
// rounds up; x = q_{i+1} always does (u <= 1 - 2^-32). idx[j] is the position in the chosen code and
// hist[part*s + idx] counts entries per part.
int eo_encode(const float* x, int64_t d, const double* P, int p, const int32_t* Q1, int m1,
              const int32_t* Q2, int m2, double theta, int s, uint64_t seed, uint32_t v,
              uint8_t* idx, int64_t* hist) {
  (void)p;
  for (int t = 0; t < 2 * s; ++t) hist[t] = 0;
  std::vector<double> q1(m1), q2(Q2 ? m2 : 0);
  for (int t = 0; t < m1; ++t) q1[t] = P[Q1[t]];
  for (int t = 0; Q2 && t < m2; ++t) q2[t] = P[Q2[t]];
  const bool mix = Q2 && theta > 0.0 && theta < 1.0;
  for (int64_t j = 0; j < d; ++j) {
    int part;
    if (!Q2) {
      part = 0;
    } else if (mix) {
      double us = double(philox_word(seed, j, v, 1u)) * 0x1p-32;
      part = (us < theta) ? 0 : 1;
    } else {
      part = (theta >= 1.0) ? 0 : 1;
    }
    const std::vector<double>& q = part == 0 ? q1 : q2;
    const int m = part == 0 ? m1 : m2;
    const double xv = x[j];
    int out;
    if (m == 1) {
      if (xv != q[0]) return -2;
      out = 0;
    } else {
      if (!(xv >= q[0]) || !(xv <= q[m - 1])) return -2;
      int i = int(std::upper_bound(q.data(), q.data() + (m - 1), xv) - q.data()) - 1;
      // Up with probability (x - q_i)/(q_{i+1} - q_i): u < (x - q_i)/(q_{i+1} - q_i)
      // tested as u * (q_{i+1} - q_i) < x - q_i, each side one IEEE operation.
      double y = xv - q[i];
      double w = q[i + 1] - q[i];
      double u = double(philox_word(seed, j, v, 0u)) * 0x1p-32;
      out = (u * w < y) ? i + 1 : i;
    }
    idx[j] = uint8_t(out);
    hist[part * s + out] += 1;
  }
  return 0;
}

// Reconstruction X^ of one encoded vector: entry j takes the value of its
// index in the code its part used (the part drawn exactly as eo_encode draws
// it), rounded to float32. E[X^] = X is the unbiasedness of §1 "O Problema
// ECASQ". Returns -1 when an index lies outside its code.
int eo_dequantize(const uint8_t* idx, int64_t d, const double* P, const int32_t* Q1, int m1,
                  const int32_t* Q2, int m2, double theta, uint64_t seed, uint32_t v, float* out) {
  const bool mix = Q2 && theta > 0.0 && theta < 1.0;
  for (int64_t j = 0; j < d; ++j) {
    int part;
    if (!Q2) {
      part = 0;
    } else if (mix) {
      double us = double(philox_word(seed, j, v, 1u)) * 0x1p-32;
      part = (us < theta) ? 0 : 1;
    } else {
      part = (theta >= 1.0) ? 0 : 1;
    }
    const int32_t* q = part == 0 ? Q1 : Q2;
    const int m = part == 0 ? m1 : m2;
    if (idx[j] >= m) return -1;
    out[j] = float(P[q[idx[j]]]);
  }
  return 0;
}

// Empirical entropy of the emitted indices: per part H_part = -sum c/d_part log2(c/d_part),
// combined as (d_0 H_0 + d_1 H_1)/d.
double eo_entropy(const int64_t* hist, int s) {
  double tot = 0.0, acc = 0.0;
  for (int part = 0; part < 2; ++part) {
    double dp = 0.0;
    for (int t = 0; t < s; ++t) dp += double(hist[part * s + t]);
    if (dp <= 0.0) continue;
    double hp = 0.0;
    for (int t = 0; t < s; ++t) {
      double c = double(hist[part * s + t]);
      if (c > 0.0) hp -= (c / dp) * std::log2(c / dp);
    }
    acc += dp * hp;
    tot += dp;
  }
  return tot > 0.0 ? acc / tot : 0.0;
}

// ---------------------------------------------------------------------------
// Batched drivers (OpenMP over vectors). Row r of X is x + r*d; P is [n][p].
// Return the number of threads used.

int eo_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int eo_solve_batch(const float* X, int n, int64_t d, const double* P, int p, int s,
                   const double* lam, int n_lam, int32_t* Q, int32_t* m, double* J, double* mse,
                   double* H, int32_t* status) {
  const int S = std::min(s, p);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t w = 0; w < int64_t(n) * n_lam; ++w) {
    const int r = int(w / n_lam);
    std::vector<int32_t> q(S, -1);
    int32_t mm = 0;
    double jj = 0, ms = 0, hh = 0;
    int st = eo_solve(X + int64_t(r) * d, d, P + int64_t(r) * p, p, s, lam[w], q.data(), &mm, &jj,
                      &ms, &hh);
    for (int t = 0; t < s; ++t) Q[w * s + t] = (t < mm) ? q[t] : -1;
    m[w] = mm;
    J[w] = jj;
    mse[w] = ms;
    H[w] = hh;
    status[w] = st;
  }
  return eo_threads();
}

int eo_solve_budget_batch(const float* X, int n, int64_t d, const double* P, int p, int s,
                          double b, int steps, int32_t* Q1, int32_t* m1, int32_t* Q2, int32_t* m2,
                          double* theta, double* lam_lo, double* lam_hi, double* H1, double* H2,
                          double* mse1, double* mse2, int32_t* status) {
  const int S = std::min(s, p);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    std::vector<int32_t> q1(S, -1), q2(S, -1);
    int32_t st = 0;
    int rc = eo_solve_budget(X + int64_t(r) * d, d, P + int64_t(r) * p, p, s, b, steps, q1.data(),
                             &m1[r], q2.data(), &m2[r], &theta[r], &lam_lo[r], &lam_hi[r], &H1[r],
                             &H2[r], &mse1[r], &mse2[r], &st);
    for (int t = 0; t < s; ++t) {
      Q1[int64_t(r) * s + t] = (t < m1[r]) ? q1[t] : -1;
      Q2[int64_t(r) * s + t] = (t < m2[r]) ? q2[t] : -1;
    }
    status[r] = rc ? rc : st;
  }
  return eo_threads();
}

int eo_encode_batch(const float* X, int n, int64_t d, const double* P, int p, const int32_t* Q1,
                    const int32_t* m1, const int32_t* Q2, const int32_t* m2, const double* theta,
                    int s, uint64_t seed, uint8_t* idx, int64_t* hist, int32_t* status) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    status[r] = eo_encode(X + int64_t(r) * d, d, P + int64_t(r) * p, p, Q1 + int64_t(r) * s, m1[r],
                          Q2 ? Q2 + int64_t(r) * s : nullptr, Q2 ? m2[r] : 0,
                          theta ? theta[r] : 0.0, s, seed, uint32_t(r), idx + int64_t(r) * d,
                          hist + int64_t(r) * 2 * s);
  }
  return eo_threads();
}

int eo_dequantize_batch(const uint8_t* idx, int n, int64_t d, const double* P, int p, const int32_t* Q1,
                        const int32_t* m1, const int32_t* Q2, const int32_t* m2, const double* theta, int s,
                        uint64_t seed, float* out, int32_t* status) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    status[r] = eo_dequantize(idx + int64_t(r) * d, d, P + int64_t(r) * p, Q1 + int64_t(r) * s, m1[r],
                              Q2 ? Q2 + int64_t(r) * s : nullptr, Q2 ? m2[r] : 0, theta ? theta[r] : 0.0, seed,
                              uint32_t(r), out + int64_t(r) * d);
  }
  return eo_threads();
}

int eo_grid_batch(const float* X, int n, int64_t d, int p, double* P, int32_t* status) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < n; ++r) status[r] = eo_uniform_grid(X + int64_t(r) * d, d, p, P + int64_t(r) * p);
  return eo_threads();
}

}  // extern "C"
