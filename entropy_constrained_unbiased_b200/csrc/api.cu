// C ABI of libecasq.so (declared in include/ecasq.h): argument checks,
// workspace carving and launch order. All work is enqueued on the caller's
// stream; nothing here allocates device memory or synchronises.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/ecasq.h"
#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {

namespace {
thread_local uint64_t g_launches = 0;

size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct Carver {
  unsigned char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* r = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += al256(sizeof(T) * count);
    return r;
  }
};

// pmax: kMaxP for the exact solver, kMaxPWide for the alphabet-sized passes
// (grid, bucketing, encoding) and the approximation.
bool valid_sizes(int n, int64_t d, int p, int s, int pmax = kMaxP) {
  return n >= 1 && d >= 1 && d <= INT32_MAX && p >= 2 && p <= pmax && s >= 2 && s <= kMaxS;
}

// Workspace layout of the solver calls (ws == null measures it).
struct SolveWs {
  unsigned long long* acc;
  int32_t* flag;
  int64_t* cnt;
  double* A;
  double* B;
  int32_t* bstatus;
  unsigned char* scratch;
  size_t bytes;
};

bool solve_ws(void* ws, int n, int p, const DpPlan& plan, SolveWs* w) {
  Carver c{static_cast<unsigned char*>(ws)};
  const size_t nb = static_cast<size_t>(n) * (p - 1);
  w->acc = c.take<unsigned long long>(3 * nb);
  w->flag = c.take<int32_t>(n);
  w->cnt = c.take<int64_t>(nb);
  w->A = c.take<double>(nb);
  w->B = c.take<double>(nb);
  w->bstatus = c.take<int32_t>(n);
  w->scratch = c.take<unsigned char>(plan.scratch_per_cta * plan.ctas);
  w->bytes = c.off;
  return true;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? ECASQ_OK : ECASQ_ERR_CUDA; }

// Workspace of the approximation: the same bucketing buffers, then its slabs.
size_t approx_ws(void* ws, int n, int p, const ApproxPlan& plan, SolveWs* w) {
  Carver c{static_cast<unsigned char*>(ws)};
  const size_t nb = static_cast<size_t>(n) * (p - 1);
  w->acc = c.take<unsigned long long>(3 * nb);
  w->flag = c.take<int32_t>(n);
  w->cnt = c.take<int64_t>(nb);
  w->A = c.take<double>(nb);
  w->B = c.take<double>(nb);
  w->bstatus = c.take<int32_t>(n);
  w->scratch = c.take<unsigned char>(plan.scratch_per_cta * plan.ctas);
  w->bytes = c.off;
  return c.off;
}

}  // namespace

void note_launch() { ++g_launches; }

}  // namespace ecasq

using namespace ecasq;

extern "C" {

const char* ecasq_status_string(int code) {
  switch (code) {
    case ECASQ_OK: return "ok";
    case ECASQ_ERR_ARG: return "bad argument";
    case ECASQ_ERR_RANGE: return "entry outside [P_0, P_{p-1}] or not finite";
    case ECASQ_ERR_WORKSPACE: return "workspace missing or too small";
    case ECASQ_ERR_CUDA: return "CUDA error";
    case ECASQ_WARN_BUDGET: return "entropy budget not reachable";
    default: return "unknown status";
  }
}

uint64_t ecasq_launch_count(int reset) {
  const uint64_t v = g_launches;
  if (reset) g_launches = 0;
  return v;
}

size_t ecasq_aux_workspace_size(int n, int64_t d, int p) {
  if (!valid_sizes(n, d, p, 2, kMaxPWide)) return 0;
  const int64_t nc = (d + minmax_chunk(d) - 1) / minmax_chunk(d);
  const size_t grid = al256(sizeof(float) * 3 * static_cast<size_t>(n) * nc);
  const size_t bucket = al256(sizeof(unsigned long long) * 3 * static_cast<size_t>(n) * (p - 1)) +
                        al256(sizeof(int32_t) * n);
  return grid > bucket ? grid : bucket;
}

size_t ecasq_workspace_size(int n, int64_t d, int p, int s, int n_lambda, const ecasq_opts* opts) {
  if (!valid_sizes(n, d, p, s) || n_lambda < 1) return 0;
  DpPlan plan;
  if (!dp_plan(n, p, s, opts && opts->dp_fp64, opts && opts->hirschberg, &plan)) return 0;
  SolveWs w;
  solve_ws(nullptr, n, p, plan, &w);
  return w.bytes;
}

int ecasq_uniform_grid(const float* X, int n, int64_t d, int p, double* P, int32_t* status, void* ws,
                       size_t ws_bytes, void* stream) {
  if (!X || !P || !status || !valid_sizes(n, d, p, 2, kMaxPWide)) return ECASQ_ERR_ARG;
  if (!ws || ws_bytes < ecasq_aux_workspace_size(n, d, p)) return ECASQ_ERR_WORKSPACE;
  return cuda_status(launch_uniform_grid(X, n, d, p, P, status, static_cast<float*>(ws),
                                         static_cast<cudaStream_t>(stream)));
}

int ecasq_bf16_alphabet(const float* X, int n, int64_t d, int p_max, double* P, int32_t* p_len, int32_t* status,
                        void* ws, size_t ws_bytes, void* stream) {
  if (!X || !P || !p_len || !status || !valid_sizes(n, d, 2, 2) || p_max < 2 || p_max > 65536) return ECASQ_ERR_ARG;
  if (!ws || ws_bytes < ecasq_aux_workspace_size(n, d, 2)) return ECASQ_ERR_WORKSPACE;
  return cuda_status(launch_bf16_alphabet(X, n, d, p_max, P, p_len, status, static_cast<float*>(ws),
                                          static_cast<cudaStream_t>(stream)));
}

int ecasq_bucket(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt, double* A, double* B,
                 int32_t* status, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !P || !cnt || !A || !B || !status || !valid_sizes(n, d, p, 2, kMaxPWide)) return ECASQ_ERR_ARG;
  if (!ws || ws_bytes < ecasq_aux_workspace_size(n, d, p)) return ECASQ_ERR_WORKSPACE;
  Carver c{static_cast<unsigned char*>(ws)};
  auto* acc = c.take<unsigned long long>(3 * static_cast<size_t>(n) * (p - 1));
  auto* flag = c.take<int32_t>(n);
  return cuda_status(launch_bucket(X, P, n, d, p, cnt, A, B, status, acc, flag, static_cast<cudaStream_t>(stream)));
}

int ecasq_grid_bucket(const float* X, int n, int64_t d, int p, double* P, int64_t* cnt, double* A, double* B,
                      int32_t* status, void* ws, size_t ws_bytes, void* stream) {
  if (!X || !P || !cnt || !A || !B || !status || !valid_sizes(n, d, p, 2, kMaxPWide)) return ECASQ_ERR_ARG;
  if (!ws || ws_bytes < ecasq_aux_workspace_size(n, d, p)) return ECASQ_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (grid_bucket_fused_ok(d, p)) return cuda_status(launch_grid_bucket_fused(X, n, d, p, P, cnt, A, B, status, st));
  // two passes: the grid (its partials), then bucketing (its accumulators), in
  // the same workspace one after the other on the stream
  cudaError_t e = launch_uniform_grid(X, n, d, p, P, status, static_cast<float*>(ws), st);
  if (e != cudaSuccess) return ECASQ_ERR_CUDA;
  Carver c{static_cast<unsigned char*>(ws)};
  auto* acc = c.take<unsigned long long>(3 * static_cast<size_t>(n) * (p - 1));
  auto* flag = c.take<int32_t>(n);
  return cuda_status(launch_bucket(X, P, n, d, p, cnt, A, B, status, acc, flag, st));
}

int ecasq_bucket_noalloc(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt, double* A,
                         double* B, int32_t* status, void* stream) {
  if (!X || !P || !cnt || !A || !B || !status || !valid_sizes(n, d, p, 2)) return ECASQ_ERR_ARG;
  if (bucket_noalloc_bytes(n, p) > bucket_noalloc_capacity()) return ECASQ_ERR_WORKSPACE;
  return cuda_status(launch_bucket_noalloc(X, P, n, d, p, cnt, A, B, status, static_cast<cudaStream_t>(stream)));
}

static int solve_common(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                        int64_t d, int p, int s, int n_lambda, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                        cudaStream_t st, DpArgs* args, DpPlan* plan, SolveWs* w) {
  if (!P || !valid_sizes(n, d, p, s) || n_lambda < 1) return ECASQ_ERR_ARG;
  if (opts && (opts->reserved != 0 || opts->bisect_steps < 0)) return ECASQ_ERR_ARG;
  if (!dp_plan(n, p, s, opts && opts->dp_fp64, opts && opts->hirschberg, plan)) return ECASQ_ERR_ARG;
  solve_ws(ws, n, p, *plan, w);
  if (!ws || ws_bytes < w->bytes) return ECASQ_ERR_WORKSPACE;
  DpArgs& a = *args;
  a = DpArgs{};
  if (X) {
    cudaError_t e = launch_bucket(X, P, n, d, p, w->cnt, w->A, w->B, w->bstatus, w->acc, w->flag, st);
    if (e != cudaSuccess) return ECASQ_ERR_CUDA;
    a.cnt = w->cnt;
    a.A = w->A;
    a.B = w->B;
    a.in_status = w->bstatus;
  } else {
    if (!cnt || !A || !B) return ECASQ_ERR_ARG;
    a.cnt = cnt;
    a.A = A;
    a.B = B;
    a.in_status = nullptr;
  }
  a.P = P;
  a.n = n;
  a.p = p;
  a.s = s < p ? s : p;
  a.s_out = s;
  a.d = d;
  a.scratch = w->scratch;
  a.scratch_per_cta = plan->scratch_per_cta;
  return ECASQ_OK;
}

static int solve_lambdas(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                         int64_t d, int p, int s, const double* lambda, int n_lambda, int32_t* Q, int32_t* Q_len,
                         double* objective, double* mse, double* H, int32_t* status, const ecasq_opts* opts, void* ws,
                         size_t ws_bytes, void* stream) {
  if (!lambda || !Q || !Q_len || !objective || !mse || !H || !status) return ECASQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DpArgs a;
  DpPlan plan;
  SolveWs w;
  int rc = solve_common(X, cnt, A, B, P, n, d, p, s, n_lambda, opts, ws, ws_bytes, st, &a, &plan, &w);
  if (rc != ECASQ_OK) return rc;
  a.mode = 0;
  a.lambda = lambda;
  a.n_lambda = n_lambda;
  a.Q = Q;
  a.Q_len = Q_len;
  a.obj = objective;
  a.mse = mse;
  a.H = H;
  a.status = status;
  return cuda_status(launch_dp(plan, a, st));
}

static int solve_budget(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                        int64_t d, int p, int s, double b, int32_t* Q1, int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len,
                        double* theta, double* lambda_lo, double* lambda_hi, double* H1, double* H2, double* mse1,
                        double* mse2, int32_t* status, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                        void* stream) {
  if (!Q1 || !Q1_len || !Q2 || !Q2_len || !theta || !lambda_lo || !lambda_hi || !H1 || !H2 || !mse1 || !mse2 ||
      !status || !(b >= 0.0))
    return ECASQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DpArgs a;
  DpPlan plan;
  SolveWs w;
  int rc = solve_common(X, cnt, A, B, P, n, d, p, s, 1, opts, ws, ws_bytes, st, &a, &plan, &w);
  if (rc != ECASQ_OK) return rc;
  a.mode = 1;
  a.budget = b;
  a.steps = (opts && opts->bisect_steps > 0) ? opts->bisect_steps : 30;
  a.Q1 = Q1;
  a.Q1_len = Q1_len;
  a.Q2 = Q2;
  a.Q2_len = Q2_len;
  a.theta = theta;
  a.lam_lo = lambda_lo;
  a.lam_hi = lambda_hi;
  a.H1 = H1;
  a.H2 = H2;
  a.mse1 = mse1;
  a.mse2 = mse2;
  a.status = status;
  return cuda_status(launch_dp(plan, a, st));
}

int ecasq_solve(const float* X, const double* P, int n, int64_t d, int p, int s, const double* lambda, int n_lambda,
                int32_t* Q, int32_t* Q_len, double* objective, double* mse, double* H, int32_t* status,
                const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!X) return ECASQ_ERR_ARG;
  return solve_lambdas(X, nullptr, nullptr, nullptr, P, n, d, p, s, lambda, n_lambda, Q, Q_len, objective, mse, H,
                       status, opts, ws, ws_bytes, stream);
}

int ecasq_solve_stats(const int64_t* cnt, const double* A, const double* B, const double* P, int n, int64_t d, int p,
                      int s, const double* lambda, int n_lambda, int32_t* Q, int32_t* Q_len, double* objective,
                      double* mse, double* H, int32_t* status, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                      void* stream) {
  return solve_lambdas(nullptr, cnt, A, B, P, n, d, p, s, lambda, n_lambda, Q, Q_len, objective, mse, H, status, opts,
                       ws, ws_bytes, stream);
}

int ecasq_solve_budget(const float* X, const double* P, int n, int64_t d, int p, int s, double b, int32_t* Q1,
                       int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len, double* theta, double* lambda_lo,
                       double* lambda_hi, double* H1, double* H2, double* mse1, double* mse2, int32_t* status,
                       const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!X) return ECASQ_ERR_ARG;
  return solve_budget(X, nullptr, nullptr, nullptr, P, n, d, p, s, b, Q1, Q1_len, Q2, Q2_len, theta, lambda_lo,
                      lambda_hi, H1, H2, mse1, mse2, status, opts, ws, ws_bytes, stream);
}

int ecasq_solve_budget_stats(const int64_t* cnt, const double* A, const double* B, const double* P, int n, int64_t d,
                             int p, int s, double b, int32_t* Q1, int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len,
                             double* theta, double* lambda_lo, double* lambda_hi, double* H1, double* H2,
                             double* mse1, double* mse2, int32_t* status, const ecasq_opts* opts, void* ws,
                             size_t ws_bytes, void* stream) {
  return solve_budget(nullptr, cnt, A, B, P, n, d, p, s, b, Q1, Q1_len, Q2, Q2_len, theta, lambda_lo, lambda_hi, H1,
                      H2, mse1, mse2, status, opts, ws, ws_bytes, stream);
}

size_t ecasq_approx_workspace_size(int n, int64_t d, int p, int s, const ecasq_opts* opts) {
  if (!valid_sizes(n, d, p, s, kMaxPWide)) return 0;
  ApproxPlan plan;
  if (!approx_plan(n, p, s, opts && opts->dp_fp64, &plan)) return 0;
  SolveWs w;
  return approx_ws(nullptr, n, p, plan, &w);
}

static int approx_common(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                         int64_t d, int p, int s, int refine, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                         cudaStream_t st, ApproxArgs* args, ApproxPlan* plan) {
  if (!P || !valid_sizes(n, d, p, s, kMaxPWide) || refine < 0) return ECASQ_ERR_ARG;
  if (opts && (opts->reserved != 0 || opts->bisect_steps < 0)) return ECASQ_ERR_ARG;
  if (!approx_plan(n, p, s, opts && opts->dp_fp64, plan)) return ECASQ_ERR_ARG;
  SolveWs w;
  approx_ws(ws, n, p, *plan, &w);
  if (!ws || ws_bytes < w.bytes) return ECASQ_ERR_WORKSPACE;
  ApproxArgs& a = *args;
  a = ApproxArgs{};
  if (X) {
    if (launch_bucket(X, P, n, d, p, w.cnt, w.A, w.B, w.bstatus, w.acc, w.flag, st) != cudaSuccess)
      return ECASQ_ERR_CUDA;
    a.cnt = w.cnt;
    a.A = w.A;
    a.B = w.B;
    a.in_status = w.bstatus;
  } else {
    if (!cnt || !A || !B) return ECASQ_ERR_ARG;
    a.cnt = cnt;
    a.A = A;
    a.B = B;
  }
  a.P = P;
  a.n = n;
  a.p = p;
  a.s = s < p ? s : p;
  a.s_out = s;
  a.d = d;
  a.refine = refine;
  a.steps = (opts && opts->bisect_steps > 0) ? opts->bisect_steps : 30;
  a.scratch = w.scratch;
  a.scratch_per_cta = plan->scratch_per_cta;
  return ECASQ_OK;
}

static int approx_lambdas(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P,
                          int n, int64_t d, int p, int s, const double* lambda, int n_lambda, int refine, int32_t* Q,
                          int32_t* Q_len, double* objective, double* mse, double* H, double* H_IB, int32_t* status,
                          const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!lambda || n_lambda < 1 || !Q || !Q_len || !objective || !mse || !H || !H_IB || !status) return ECASQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ApproxArgs a;
  ApproxPlan plan;
  int rc = approx_common(X, cnt, A, B, P, n, d, p, s, refine, opts, ws, ws_bytes, st, &a, &plan);
  if (rc != ECASQ_OK) return rc;
  a.mode = 0;
  a.lambda = lambda;
  a.n_lambda = n_lambda;
  a.Q = Q;
  a.Q_len = Q_len;
  a.obj = objective;
  a.mse = mse;
  a.H = H;
  a.HIB = H_IB;
  a.status = status;
  return cuda_status(launch_approx(plan, a, st));
}

static int approx_budget(const float* X, const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                         int64_t d, int p, int s, double b, int refine, int32_t* Q1, int32_t* Q1_len, int32_t* Q2,
                         int32_t* Q2_len, double* theta, double* lambda_lo, double* lambda_hi, double* H1, double* H2,
                         double* H_IB1, double* H_IB2, double* mse1, double* mse2, int32_t* status,
                         const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!Q1 || !Q1_len || !Q2 || !Q2_len || !theta || !lambda_lo || !lambda_hi || !H1 || !H2 || !H_IB1 || !H_IB2 ||
      !mse1 || !mse2 || !status || !(b >= 0.0))
    return ECASQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ApproxArgs a;
  ApproxPlan plan;
  int rc = approx_common(X, cnt, A, B, P, n, d, p, s, refine, opts, ws, ws_bytes, st, &a, &plan);
  if (rc != ECASQ_OK) return rc;
  a.mode = 1;
  a.budget = b;
  a.Q1 = Q1;
  a.Q1_len = Q1_len;
  a.Q2 = Q2;
  a.Q2_len = Q2_len;
  a.theta = theta;
  a.lam_lo = lambda_lo;
  a.lam_hi = lambda_hi;
  a.H1 = H1;
  a.H2 = H2;
  a.HIB1 = H_IB1;
  a.HIB2 = H_IB2;
  a.mse1 = mse1;
  a.mse2 = mse2;
  a.status = status;
  return cuda_status(launch_approx(plan, a, st));
}

int ecasq_solve_approx(const float* X, const double* P, int n, int64_t d, int p, int s, const double* lambda,
                       int n_lambda, int refine_iters, int32_t* Q, int32_t* Q_len, double* objective, double* mse,
                       double* H, double* H_IB, int32_t* status, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                       void* stream) {
  if (!X) return ECASQ_ERR_ARG;
  return approx_lambdas(X, nullptr, nullptr, nullptr, P, n, d, p, s, lambda, n_lambda, refine_iters, Q, Q_len,
                        objective, mse, H, H_IB, status, opts, ws, ws_bytes, stream);
}

int ecasq_solve_approx_stats(const int64_t* cnt, const double* A, const double* B, const double* P, int n, int64_t d,
                             int p, int s, const double* lambda, int n_lambda, int refine_iters, int32_t* Q,
                             int32_t* Q_len, double* objective, double* mse, double* H, double* H_IB, int32_t* status,
                             const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  return approx_lambdas(nullptr, cnt, A, B, P, n, d, p, s, lambda, n_lambda, refine_iters, Q, Q_len, objective, mse,
                        H, H_IB, status, opts, ws, ws_bytes, stream);
}

int ecasq_solve_approx_budget(const float* X, const double* P, int n, int64_t d, int p, int s, double b,
                              int refine_iters, int32_t* Q1, int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len,
                              double* theta, double* lambda_lo, double* lambda_hi, double* H1, double* H2,
                              double* H_IB1, double* H_IB2, double* mse1, double* mse2, int32_t* status,
                              const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream) {
  if (!X) return ECASQ_ERR_ARG;
  return approx_budget(X, nullptr, nullptr, nullptr, P, n, d, p, s, b, refine_iters, Q1, Q1_len, Q2, Q2_len, theta,
                       lambda_lo, lambda_hi, H1, H2, H_IB1, H_IB2, mse1, mse2, status, opts, ws, ws_bytes, stream);
}

int ecasq_solve_approx_budget_stats(const int64_t* cnt, const double* A, const double* B, const double* P, int n,
                                    int64_t d, int p, int s, double b, int refine_iters, int32_t* Q1, int32_t* Q1_len,
                                    int32_t* Q2, int32_t* Q2_len, double* theta, double* lambda_lo,
                                    double* lambda_hi, double* H1, double* H2, double* H_IB1, double* H_IB2,
                                    double* mse1, double* mse2, int32_t* status, const ecasq_opts* opts, void* ws,
                                    size_t ws_bytes, void* stream) {
  return approx_budget(nullptr, cnt, A, B, P, n, d, p, s, b, refine_iters, Q1, Q1_len, Q2, Q2_len, theta, lambda_lo,
                       lambda_hi, H1, H2, H_IB1, H_IB2, mse1, mse2, status, opts, ws, ws_bytes, stream);
}

int ecasq_encode(const float* X, const double* P, int n, int64_t d, int p, int s, const int32_t* Q1,
                 const int32_t* Q1_len, const int32_t* Q2, const int32_t* Q2_len, const double* theta, uint64_t seed,
                 uint8_t* idx, int64_t* hist, int32_t* status, void* stream) {
  // s is the row stride of the codes and the histogram (a code of up to 256
  // values: indices fit in uint8), not bound by the solvers' code size.
  if (!X || !P || !Q1 || !Q1_len || !idx || !hist || !status || !valid_sizes(n, d, p, 2, kMaxPWide) || s < 1 ||
      s > 256)
    return ECASQ_ERR_ARG;
  if (Q2 && !Q2_len) return ECASQ_ERR_ARG;
  return cuda_status(launch_encode(X, P, n, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, seed, idx, hist, status,
                                   static_cast<cudaStream_t>(stream)));
}

int ecasq_dequantize(const uint8_t* idx, const double* P, int n, int64_t d, int p, int s, const int32_t* Q1,
                     const int32_t* Q1_len, const int32_t* Q2, const int32_t* Q2_len, const double* theta,
                     uint64_t seed, float* Xhat, int32_t* status, void* stream) {
  if (!idx || !P || !Q1 || !Q1_len || !Xhat || !status || !valid_sizes(n, d, p, 2, kMaxPWide) || s < 1 || s > 256)
    return ECASQ_ERR_ARG;
  if (Q2 && !Q2_len) return ECASQ_ERR_ARG;
  return cuda_status(launch_dequantize(idx, P, n, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, seed, Xhat, status,
                                       static_cast<cudaStream_t>(stream)));
}

int64_t ecasq_rans_segments(int64_t d) { return d >= 1 ? rans_segments(d) : 0; }
int64_t ecasq_rans_segment_words(void) { return rans_segment_words(); }

int ecasq_rans_encode(const uint8_t* idx, const int64_t* hist, const double* theta, int two_codes, int n, int64_t d,
                      int s, uint64_t seed, uint16_t* words, int32_t* seg_len, int32_t* status, void* stream) {
  if (!idx || !hist || !words || !seg_len || !status || !valid_sizes(n, d, 2, 2) || s < 1 || s > 256)
    return ECASQ_ERR_ARG;
  return cuda_status(launch_rans_encode(idx, hist, theta, two_codes, n, d, s, seed, words, seg_len, status,
                                        static_cast<cudaStream_t>(stream)));
}

int ecasq_rans_decode(const uint16_t* words, const int32_t* seg_len, const int64_t* hist, const double* theta,
                      int two_codes, int n, int64_t d, int s, uint64_t seed, uint8_t* idx, int32_t* status,
                      void* stream) {
  if (!idx || !hist || !words || !seg_len || !status || !valid_sizes(n, d, 2, 2) || s < 1 || s > 256)
    return ECASQ_ERR_ARG;
  return cuda_status(launch_rans_decode(words, seg_len, hist, theta, two_codes, n, d, s, seed, idx, status,
                                        static_cast<cudaStream_t>(stream)));
}

int ecasq_entropy(const int64_t* hist, int n, int s, double* H, void* stream) {
  if (!hist || !H || n < 1 || s < 1 || s > 256) return ECASQ_ERR_ARG;
  return cuda_status(launch_entropy(hist, n, s, H, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
