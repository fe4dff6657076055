/*
 * ecasq.h — C ABI of libecasq.so, the B200 (sm_100a) ECASQ solver.
 *
 * ECASQ = entropy-constrained adaptive stochastic quantization, as defined in the
 * technical summary "Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)"
 * (gist.science/pt/paper/2608.18147):
 *   §1   "O Problema ECASQ": for a vector X in R^d, a permissible alphabet P
 *        (p sorted values), a code size s and an entropy budget b, choose
 *        Q subset of P with |Q| <= s that minimises the MSE of unbiased stochastic
 *        rounding onto Q (E[X^] = X) subject to H(X^) <= b bits per entry.
 *   §2.1 "Relaxação Lagrangiana": minimise MSE(Q,X) + lambda * H(X^); varying
 *        lambda traces the Pareto curve; two-way time-sharing of two quantizers
 *        on a random partition of the input reaches any budget b.
 *   §2.2 "Programação Dinâmica Ótima": the exact DP over the pair state
 *        dp_OPT(i, l, j) (the entropy of a value depends on both neighbours);
 *        "Generalização": arbitrary P in O(p^2 s + d) after bucketing X onto P.
 *
 * Conventions shared by every entry point
 *   - Every array argument is DEVICE memory owned by the caller (for example a
 *     torch tensor), row-major and contiguous, unless marked "host". The
 *     library allocates nothing: scratch comes from the caller's workspace
 *     (ecasq_workspace_size), which must stay alive until the stream work ends.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream). The return value is a HOST status for
 *     argument and launch errors only. Errors found by the device (an entry
 *     outside [P_0, P_{p-1}], a NaN/Inf, a budget that cannot be met) are
 *     written per vector to the `status` array, which the caller reads after
 *     the stream work is done.
 *   - X is float32 [n][d]; P is float64 [n][p], strictly increasing per row,
 *     with P_0 <= min X and max X <= P_{p-1}. The solver keeps P_0 and P_{p-1}
 *     in every code (the uniform grid of ecasq_uniform_grid spans exactly
 *     [min X, max X], so both ends are forced by unbiasedness there).
 *   - A code Q is returned as ascending indices into the vector's row of P,
 *     padded with -1 up to s; Q_len holds |Q|.
 *   - Limits: 2 <= s <= 255 (s > p is treated as s = p), 1 <= d <= 2^31 - 1,
 *     n >= 1; 2 <= p <= 512 for the exact solver (ecasq_solve*,
 *     ecasq_workspace_size), 2 <= p <= 65536 for the grid, bucketing,
 *     encoding, the reconstruction and the approximation (large alphabets, e.g.
 *     every BF16 value of a range; above 512 values the approximation runs fp32
 *     layers only).
 *   - Entropies are in bits per entry; the MSE is the per-entry mean
 *     (1/d) * sum (q_hi - x)(x - q_lo); the objective is MSE + lambda * H.
 */
#ifndef ECASQ_H_
#define ECASQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host return codes and per-vector device status codes. */
#define ECASQ_OK 0
#define ECASQ_ERR_ARG (-1)       /* bad argument (host), or P not increasing (device) */
#define ECASQ_ERR_RANGE (-2)     /* device: an entry is NaN/Inf or outside [P_0, P_{p-1}] */
#define ECASQ_ERR_WORKSPACE (-3) /* host: workspace missing or smaller than required */
#define ECASQ_ERR_CUDA (-4)      /* host: a CUDA launch or runtime call failed */
#define ECASQ_WARN_BUDGET 1      /* device: H(lambda_hi) > b; result is the code at lambda_hi */

/* Solver options (host struct, may be NULL for the defaults). */
typedef struct ecasq_opts {
  int dp_fp64;      /* 0 (default): DP layer values in fp32 with the MUFU log2;
                       1: fp64 DP (parity mode). The chosen code is always
                       re-evaluated in fp64. */
  int hirschberg;   /* 0 (default): store back-pointers; 1: recompute them
                       (O(p^2) DP memory per vector, §2.2 "Algoritmo de Hirschberg"). */
  int bisect_steps; /* lambda bisection steps of ecasq_solve_budget (default 30). */
  int reserved;     /* must be 0 */
} ecasq_opts;

/* Bytes of workspace that ecasq_solve / ecasq_solve_budget / ecasq_solve_stats /
 * ecasq_solve_budget_stats need for these sizes on the CURRENT device
 * (n_lambda = lambdas per vector; 1 for the budget solver). Returns 0 on bad
 * arguments. ecasq_bucket and ecasq_uniform_grid need ecasq_aux_workspace_size. */
size_t ecasq_workspace_size(int n, int64_t d, int p, int s, int n_lambda, const ecasq_opts* opts);

/* Workspace of ecasq_uniform_grid and ecasq_bucket for these sizes. */
size_t ecasq_aux_workspace_size(int n, int64_t d, int p);

/* Uniform permissible set on each row's range (the alphabet of the workloads
 * above; §2.2 "Generalização" allows any P): P[r][k] = lo + (hi-lo)*k/(p-1)
 * in fp64 with lo = min X[r], hi = max X[r], and P[r][p-1] = hi exactly.
 * status[r] = ECASQ_ERR_RANGE when row r holds a NaN or an infinity. */
int ecasq_uniform_grid(const float* X, int n, int64_t d, int p, double* P, int32_t* status,
                       void* ws, size_t ws_bytes, void* stream);

/* Hardware-aware permissible set (§5 "Generalidade": any alphabet, e.g. the
 * values BF16 can represent): per row, every finite BF16 value from the largest
 * one <= min X to the smallest one >= max X, ascending, with +0 and -0 counted
 * once; P_0 <= min X and P_{p-1} >= max X as the solver requires.
 * P [n][p_max] float64 (entries past the row's count are NaN), p_len [n] = the
 * row's count even when it exceeds p_max. status[r] = ECASQ_ERR_RANGE for a
 * NaN/Inf entry or a range beyond the finite BF16 values, ECASQ_ERR_ARG when
 * the count exceeds p_max (P then holds the first p_max values).
 * 2 <= p_max <= 65536. Rows with different counts need separate solver calls
 * (the solver takes one p per call). Workspace: ecasq_aux_workspace_size(n, d, 2). */
int ecasq_bf16_alphabet(const float* X, int n, int64_t d, int p_max, double* P, int32_t* p_len,
                        int32_t* status, void* ws, size_t ws_bytes, void* stream);

/* Bucketing of each row onto its alphabet (the "+d" term of §2.2
 * "Generalização"): bucket k = max{k <= p-2 : P_k <= x}, so the last bucket is
 * closed; per bucket the count cnt (int64 [n][p-1]) and the shifted moments
 * A = sum (x - P_k), B = sum (x - P_k)^2 (float64 [n][p-1]).
 * status[r] = ECASQ_ERR_RANGE when an entry of row r lies outside [P_0, P_{p-1}]
 * or is NaN. */
int ecasq_bucket(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                 double* A, double* B, int32_t* status, void* ws, size_t ws_bytes, void* stream);

/* ecasq_uniform_grid followed by ecasq_bucket, in one call: P, cnt, A, B and
 * status as those two calls give them (the grid bit for bit). Rows of at most
 * 16384 entries with p <= 129 are read from HBM once (each row is staged in
 * shared memory, its grid and its statistics computed from there); other sizes
 * run the two passes. A row holding a NaN or an infinity gets a NaN grid,
 * status ECASQ_ERR_RANGE and (on the one-read path) zero statistics. On the
 * one-read path, status ECASQ_ERR_CUDA marks a row whose staging copy the
 * device stopped waiting for. Workspace: ecasq_aux_workspace_size(n, d, p). */
int ecasq_grid_bucket(const float* X, int n, int64_t d, int p, double* P, int64_t* cnt, double* A,
                      double* B, int32_t* status, void* ws, size_t ws_bytes, void* stream);

/* ecasq_bucket without a workspace, for callers that cannot allocate device
 * memory where they bucket: plugins inside a framework whose own caching
 * allocator owns all device memory, and fixed-budget real-time or embedded
 * pipelines that forbid cudaMalloc after start-up (it can synchronise the
 * device and can fail under fragmentation). The ECASQ page has no counterpart;
 * this is an interface convenience around the same bucketing kernels.
 * Outputs, layout and status are those of ecasq_bucket.
 * Scratch: a fixed 8 MiB array in the library's device memory, held by every
 * GPU that loads the library until the process exits. It must hold
 * 24*n*(p-1) + 4*n bytes (each term rounded up to 256), e.g. n <= 2748 rows at
 * p = 128 or n <= 1369 at p = 256; larger sizes return ECASQ_ERR_WORKSPACE
 * and launch nothing. The call allocates nothing: the first call on a device
 * resolves the array's device address (with that device current), so make
 * that first call before any stream capture. The address is kept for the
 * life of the process: a cudaDeviceReset (or any other teardown of the
 * device's primary context) invalidates it, so do not call this entry point on
 * a device after resetting it. Every call on a device shares the array (the
 * call clears it on the stream before use): calls that overlap on the same
 * GPU race, so serialise them (one stream, or events). */
int ecasq_bucket_noalloc(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                         double* A, double* B, int32_t* status, void* stream);

/* Exact Lagrangian solve (§2.1 + §2.2) of every row at n_lambda multipliers:
 * lambda is [n][n_lambda] (>= 0). For row r and multiplier t the code
 * Q[(r*n_lambda + t)*s ...] minimises MSE + lambda*H over |Q| <= s with
 * P_0, P_{p-1} in Q; objective/mse/H [n][n_lambda] are its fp64 values.
 * Ties: smallest |Q|, then smallest indices. Buckets X internally. */
int ecasq_solve(const float* X, const double* P, int n, int64_t d, int p, int s,
                const double* lambda, int n_lambda, int32_t* Q, int32_t* Q_len,
                double* objective, double* mse, double* H, int32_t* status,
                const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream);

/* Same, from bucket statistics produced by ecasq_bucket (cnt, A, B as above). */
int ecasq_solve_stats(const int64_t* cnt, const double* A, const double* B, const double* P,
                      int n, int64_t d, int p, int s, const double* lambda, int n_lambda,
                      int32_t* Q, int32_t* Q_len, double* objective, double* mse, double* H,
                      int32_t* status, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                      void* stream);

/* Entropy budget b (§1 constraint, §2.1 time-sharing), per row:
 * bracket [0, (P_{p-1} - P_0)^2], arithmetic bisection (opts->bisect_steps,
 * default 30) with "H(mid) > b => lambda_lo = mid". Q1 [n][s] is the code at
 * the final lambda_lo (H1 > b), Q2 the code at lambda_hi (H2 <= b), and
 * theta [n] = (b - H2)/(H1 - H2) the share of entries coded with Q1, so that
 * theta*H1 + (1-theta)*H2 = b. If H at lambda = 0 is already <= b: Q1 = Q2 =
 * that code, theta = 0. If H(lambda_hi) > b: status = ECASQ_WARN_BUDGET,
 * Q2 = code at lambda_hi, theta = 0. */
int ecasq_solve_budget(const float* X, const double* P, int n, int64_t d, int p, int s, double b,
                       int32_t* Q1, int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len, double* theta,
                       double* lambda_lo, double* lambda_hi, double* H1, double* H2, double* mse1,
                       double* mse2, int32_t* status, const ecasq_opts* opts, void* ws,
                       size_t ws_bytes, void* stream);

/* Same, from bucket statistics. */
int ecasq_solve_budget_stats(const int64_t* cnt, const double* A, const double* B, const double* P,
                             int n, int64_t d, int p, int s, double b, int32_t* Q1,
                             int32_t* Q1_len, int32_t* Q2, int32_t* Q2_len, double* theta,
                             double* lambda_lo, double* lambda_hi, double* H1, double* H2,
                             double* mse1, double* mse2, int32_t* status,
                             const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream);

/* ---- Space-efficient approximation (§2.3) and iterative refinement (§2.4) ----
 *
 * The approximation replaces H(X^) by H(I,B), the entropy of the pair (index I
 * of the code interval [q_t, q_{t+1}] holding the entry, rounding bit B). An
 * entry on an interior code value belongs to the interval that starts there.
 * With L, R the expected down/up counts of an interval,
 *   H(I,B) = sum over intervals of h(L) + h(R),  h(mu) = -(mu/d) log2(mu/d),
 * and H(X^) <= H(I,B) <= H(X^) + 1. MSE + lambda*H(I,B) is a sum of
 * per-interval costs, so its exact minimiser (P_0, P_{p-1} in Q, |Q| <= s) is a
 * layered shortest path in O(p^2 s) time with O(p s) state; at budget b its MSE
 * is no larger than the exact optimum's at b - 1.
 *
 * refine_iters > 0 then refines the code on the exact objective MSE +
 * lambda*H(X^) at the same lambda: the interior values, in three classes by
 * position mod 3 (a class moves at once, since a value's move changes only its
 * two intervals and three masses), each search the open interval between their
 * neighbours by binary search on the sign of the forward difference of their
 * local cost and move only on a strict decrease; up to refine_iters iterations
 * (classes 0, 1, 2), stopping early after an iteration with no move. The
 * refinement never changes |Q|.
 *
 * Layers run in fp32 (default) or fp64 (opts->dp_fp64); refinement and the
 * reported figures are fp64. opts->hirschberg is ignored (no back-pointers are
 * kept). Workspace: ecasq_approx_workspace_size. Returns as the exact solver.
 *
 * Alphabets of more than 512 values (up to 65536): the pair terms are computed
 * for every relaxation from six O(p) prefix sums over the buckets instead of
 * O(p^2) tables (memory O(p s) per vector), the layers run in fp32 (dp_fp64 = 1
 * returns ECASQ_ERR_ARG), the refinement compares local costs from the same
 * prefix sums in fp64, and the reported figures are direct fp64 sums over each
 * interval's buckets. Time O(p^2 s) per solve. */
size_t ecasq_approx_workspace_size(int n, int64_t d, int p, int s, const ecasq_opts* opts);

/* Per row and multiplier (lambda [n][n_lambda] >= 0): the code Q [n][n_lambda][s]
 * and its fp64 mse, H = H(X^), H_IB = H(I,B) [n][n_lambda]; objective = mse +
 * lambda*H_IB without refinement, mse + lambda*H with it. Buckets X internally. */
int ecasq_solve_approx(const float* X, const double* P, int n, int64_t d, int p, int s,
                       const double* lambda, int n_lambda, int refine_iters, int32_t* Q,
                       int32_t* Q_len, double* objective, double* mse, double* H, double* H_IB,
                       int32_t* status, const ecasq_opts* opts, void* ws, size_t ws_bytes,
                       void* stream);

/* Same, from bucket statistics (ecasq_bucket). */
int ecasq_solve_approx_stats(const int64_t* cnt, const double* A, const double* B, const double* P,
                             int n, int64_t d, int p, int s, const double* lambda, int n_lambda,
                             int refine_iters, int32_t* Q, int32_t* Q_len, double* objective,
                             double* mse, double* H, double* H_IB, int32_t* status,
                             const ecasq_opts* opts, void* ws, size_t ws_bytes, void* stream);

/* Entropy budget b with the bisection and two-way time-sharing of
 * ecasq_solve_budget. The constrained rate is H(I,B) when refine_iters == 0 and
 * H(X^) otherwise; theta = (b - rate2)/(rate1 - rate2). H1/H2 are H(X^) and
 * H_IB1/H_IB2 are H(I,B) of Q1/Q2, whichever rate is constrained. */
int ecasq_solve_approx_budget(const float* X, const double* P, int n, int64_t d, int p, int s,
                              double b, int refine_iters, int32_t* Q1, int32_t* Q1_len, int32_t* Q2,
                              int32_t* Q2_len, double* theta, double* lambda_lo, double* lambda_hi,
                              double* H1, double* H2, double* H_IB1, double* H_IB2, double* mse1,
                              double* mse2, int32_t* status, const ecasq_opts* opts, void* ws,
                              size_t ws_bytes, void* stream);

/* Same, from bucket statistics. */
int ecasq_solve_approx_budget_stats(const int64_t* cnt, const double* A, const double* B,
                                    const double* P, int n, int64_t d, int p, int s, double b,
                                    int refine_iters, int32_t* Q1, int32_t* Q1_len, int32_t* Q2,
                                    int32_t* Q2_len, double* theta, double* lambda_lo,
                                    double* lambda_hi, double* H1, double* H2, double* H_IB1,
                                    double* H_IB2, double* mse1, double* mse2, int32_t* status,
                                    const ecasq_opts* opts, void* ws, size_t ws_bytes,
                                    void* stream);

/* Unbiased stochastic rounding (§1, E[X^] = X) with optional two-way
 * time-sharing (§2.1), counter-based randomness Philox4x32-10 (Salmon et al.,
 * SC'11) keyed by seed (low word, high word), counter (j >> 2, r, stream, 0),
 * output word j & 3, u = word * 2^-32, for entry j of row r:
 *   - Q2 == NULL: every entry uses Q1 (part 0).
 *   - Q2 != NULL, 0 < theta[r] < 1: entry uses Q1 iff u(stream 1) < theta[r],
 *     else Q2 (part 1); theta >= 1: Q1 only; theta <= 0 (or theta NULL): Q2 only.
 *   - x in [q_i, q_{i+1}] of its code rounds up with probability
 *     (x - q_i)/(q_{i+1} - q_i); the test, with the division moved across, is
 *     u(stream 0) * (q_{i+1} - q_i) < x - q_i, each side one IEEE fp64
 *     operation with round-to-nearest (the width q_{i+1} - q_i is one
 *     subtraction, the product one multiplication, x - q_i one subtraction;
 *     no fused multiply-add), so x = q_i never rounds up and x = q_{i+1}
 *     always does. The time-sharing test u(stream 1) < theta[r] is the exact
 *     integer test word < ceil(theta[r] * 2^32).
 * idx [n][d] uint8 = position of the emitted value in the code used (so s <= 256);
 * hist [n][2][s] int64 counts per part and position (overwritten).
 * status[r] = ECASQ_ERR_RANGE for an entry outside its code's range. */
int ecasq_encode(const float* X, const double* P, int n, int64_t d, int p, int s,
                 const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2,
                 const int32_t* Q2_len, const double* theta, uint64_t seed, uint8_t* idx,
                 int64_t* hist, int32_t* status, void* stream);

/* Reconstruction X^ from the emitted indices (§1 "O Problema ECASQ": the
 * quantized value of each entry, with E[X^] = X; §2.1: the time-sharing part
 * drawn again from seed and theta exactly as ecasq_encode drew it):
 * Xhat[r][j] = P[r][Q_part[r][idx[r][j]]] rounded to float32, with Q1, Q1_len,
 * Q2, Q2_len, theta, s and seed as given to ecasq_encode. Xhat [n][d] float32
 * (device, caller-owned). status[r] = ECASQ_ERR_RANGE when an index is not
 * below its code's length (or a code holds an index outside P); that row's
 * values are then unspecified. Asynchronous; allocates nothing. */
int ecasq_dequantize(const uint8_t* idx, const double* P, int n, int64_t d, int p, int s,
                     const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2,
                     const int32_t* Q2_len, const double* theta, uint64_t seed, float* Xhat,
                     int32_t* status, void* stream);

/* Empirical entropy of the emitted indices from hist [n][2][s] (§1, H(X^)):
 * per part H_part = -sum c/d_part log2(c/d_part), combined as
 * (d_0 H_0 + d_1 H_1)/(d_0 + d_1). H [n] float64. */
int ecasq_entropy(const int64_t* hist, int n, int s, double* H, void* stream);

/* Lossless entropy coding of the emitted indices (§1 "Contexto": the
 * quantizer's output goes through an entropy coder that gives frequent values
 * shorter bit strings; H(X^) is what it approaches). Static-model rANS (Duda,
 * arXiv:1311.2540), one model per row and part from hist [n][2][s] (the
 * histogram ecasq_encode wrote): probabilities quantised to M = 2^15, f_i =
 * max(1, floor(c_i M / n_part)) for the symbols that occur, the shortfall to M
 * added to the most frequent symbol (lowest index on ties), an excess taken from
 * the largest frequencies first (none below 1). The part of each entry is not
 * coded: it is recomputed from seed and theta exactly as ecasq_encode drew it
 * (two_codes = 0: every entry in part 0, as with Q2 == NULL; otherwise the
 * theta rule of ecasq_encode, theta NULL meaning part 1).
 * 32-bit states in [2^16, 2^32), 16-bit words; a row is cut into segments of
 * 16384 entries (ecasq_rans_segments(d) of them), each coded by 32 interleaved
 * states: the 32 entries of a step go one per state, the renormalisation words
 * of a step are stacked in state order, the final states follow as (low, high)
 * pairs. words [n][segments][ecasq_rans_segment_words()] uint16; seg_len
 * [n][segments] int32 = words used (the coded size of a row is 16 * sum bits).
 * status[r] = ECASQ_ERR_ARG when an index has no frequency in its part's model
 * (encode) or the stream is malformed (decode). Asynchronous; device memory. */
int64_t ecasq_rans_segments(int64_t d);
int64_t ecasq_rans_segment_words(void);
int ecasq_rans_encode(const uint8_t* idx, const int64_t* hist, const double* theta, int two_codes, int n,
                      int64_t d, int s, uint64_t seed, uint16_t* words, int32_t* seg_len, int32_t* status,
                      void* stream);
/* Inverse of ecasq_rans_encode: idx [n][d] uint8 from the words, the same hist,
 * theta, two_codes and seed. */
int ecasq_rans_decode(const uint16_t* words, const int32_t* seg_len, const int64_t* hist, const double* theta,
                      int two_codes, int n, int64_t d, int s, uint64_t seed, uint8_t* idx, int32_t* status,
                      void* stream);

/* Static text for a status code. */
const char* ecasq_status_string(int code);

/* Number of kernel launches issued by the calling host thread through this
 * library since the last reset (instrumentation for benchmarks). */
uint64_t ecasq_launch_count(int reset);

#ifdef __cplusplus
}
#endif

#endif /* ECASQ_H_ */
