// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace ecasq {

// Counts kernel launches issued through the library (per host thread).
void note_launch();

// ---- grid + bucketing (grid_bucket.cu) ----
int bucket_fraction_bits(int64_t d);
int64_t minmax_chunk(int64_t d);
int64_t bucket_chunk(int64_t d);
size_t bucket_smem_bytes(int p);
cudaError_t launch_uniform_grid(const float* X, int n, int64_t d, int p, double* P, int32_t* status,
                                float* part, cudaStream_t st);
cudaError_t launch_bucket(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                          double* A, double* B, int32_t* status, unsigned long long* acc,
                          int32_t* flag, cudaStream_t st);

// Uniform grid + bucketing in one read of X (rows that fit in shared memory).
bool grid_bucket_fused_ok(int64_t d, int p);
cudaError_t launch_grid_bucket_fused(const float* X, int n, int64_t d, int p, double* P, int64_t* cnt, double* A,
                                     double* B, int32_t* status, cudaStream_t st);

cudaError_t launch_bf16_alphabet(const float* X, int n, int64_t d, int p_max, double* P, int32_t* p_len,
                                 int32_t* status, float* part, cudaStream_t st);

size_t bucket_noalloc_bytes(int n, int p);
size_t bucket_noalloc_capacity();
cudaError_t launch_bucket_noalloc(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                                  double* A, double* B, int32_t* status, cudaStream_t st);

// ---- DP solver (dp.cu) ----
struct DpArgs {
  // bucket statistics [n][p-1] and alphabet [n][p]
  const int64_t* cnt;
  const double* A;
  const double* B;
  const double* P;
  const int32_t* in_status;  // [n] status of the bucketing pass, or null
  int n, p, s;               // s already clamped to p
  int64_t d;
  // mode 0: list of lambdas per vector; mode 1: entropy budget
  int mode;
  const double* lambda;  // [n][n_lambda]
  int n_lambda;
  double budget;
  int steps;
  // mode 0 outputs ([n][n_lambda] and [n][n_lambda][s_out])
  int32_t* Q;
  int32_t* Q_len;
  double* obj;
  double* mse;
  double* H;
  // mode 1 outputs ([n] and [n][s_out])
  int32_t* Q1;
  int32_t* Q1_len;
  int32_t* Q2;
  int32_t* Q2_len;
  double* theta;
  double* lam_lo;
  double* lam_hi;
  double* H1;
  double* H2;
  double* mse1;
  double* mse2;
  int32_t* status;  // [n]
  int s_out;        // row stride of the Q outputs (the caller's s)
  int hirschberg;   // 1: no back-pointers, divide-and-conquer recovery of the code
  // per-CTA global scratch
  unsigned char* scratch;
  size_t scratch_per_cta;
};

struct DpPlan {
  bool fp64;
  bool hirschberg;
  bool smem_tables;  // pair tables resident in shared memory
  int cluster;       // CTAs per vector (a thread-block cluster when > 1)
  int threads;
  int ctas;
  size_t smem_bytes;
  size_t scratch_per_cta;
};

// Plan for the current device; ok = false when the sizes are out of range.
bool dp_plan(int n, int p, int s, bool fp64, bool hirschberg, DpPlan* plan);
cudaError_t launch_dp(const DpPlan& plan, DpArgs args, cudaStream_t st);

// Exact count of (k, l, j) triples one solve evaluates (host).
int64_t dp_triples(int p, int s);

// ---- approximation on H(I,B) + refinement (approx.cu) ----
struct ApproxArgs {
  const int64_t* cnt;
  const double* A;
  const double* B;
  const double* P;
  const int32_t* in_status;
  int n, p, s;  // s already clamped to p
  int64_t d;
  int refine;  // refinement iterations (0: none)
  int mode;    // 0: lambda list, 1: entropy budget
  const double* lambda;
  int n_lambda;
  double budget;
  int steps;
  int32_t* Q;
  int32_t* Q_len;
  double* obj;
  double* mse;
  double* H;
  double* HIB;
  int32_t* Q1;
  int32_t* Q1_len;
  int32_t* Q2;
  int32_t* Q2_len;
  double* theta;
  double* lam_lo;
  double* lam_hi;
  double* H1;
  double* H2;
  double* HIB1;
  double* HIB2;
  double* mse1;
  double* mse2;
  int32_t* status;
  int s_out;
  unsigned char* scratch;
  size_t scratch_per_cta;
};

struct ApproxPlan {
  bool wide;  // alphabet beyond 512 values: pair terms from prefix sums (fp32 layers only)
  bool fp64;
  bool smem;  // cost table and layers in shared memory
  bool split;  // each column's a range shared by two threads (few vectors)
  int threads;
  int ctas;
  size_t smem_bytes;
  size_t scratch_per_cta;
};

bool approx_plan(int n, int p, int s, bool fp64, ApproxPlan* plan);
cudaError_t launch_approx(const ApproxPlan& plan, ApproxArgs args, cudaStream_t st);
// (i, a, c) relaxations of one solve of the layered shortest path (host).
int64_t approx_pair_layers(int p, int s);

// ---- entropy coder for the indices (rans.cu) ----
int64_t rans_segments(int64_t d);
int64_t rans_segment_words();
cudaError_t launch_rans_encode(const uint8_t* idx, const int64_t* hist, const double* theta, int two_codes, int n,
                               int64_t d, int s, uint64_t seed, uint16_t* words, int32_t* seg_len, int32_t* status,
                               cudaStream_t st);
cudaError_t launch_rans_decode(const uint16_t* words, const int32_t* seg_len, const int64_t* hist, const double* theta,
                               int two_codes, int n, int64_t d, int s, uint64_t seed, uint8_t* idx, int32_t* status,
                               cudaStream_t st);

// Entries per CTA for kernels that take rows in chunks: `full`, unless the
// n * ceil(d / full) CTAs would leave some of the `resident` CTA slots empty
// (few or short rows); then ceil(resident / n) chunks per row, each a multiple
// of `align` (a power of two) and at least `min_chunk`. Smaller chunks on
// grids that already fill the GPU only add per-CTA setups.
inline int64_t fill_chunk(int n, int64_t d, int64_t resident, int64_t full, int64_t align, int64_t min_chunk) {
  if (d <= 0) return full;
  if (static_cast<int64_t>(n) * ((d + full - 1) / full) >= resident) return full;
  const int64_t k = (resident + n - 1) / n;
  const int64_t chunk = (((d + k - 1) / k) + align - 1) & ~(align - 1);
  return chunk < min_chunk ? min_chunk : (chunk > full ? full : chunk);
}

// ---- encoder (encode.cu) ----
cudaError_t launch_encode(const float* X, const double* P, int n, int64_t d, int p, int s,
                          const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2,
                          const int32_t* Q2_len, const double* theta, uint64_t seed, uint8_t* idx,
                          int64_t* hist, int32_t* status, cudaStream_t st);
cudaError_t launch_entropy(const int64_t* hist, int n, int s, double* H, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* idx, const double* P, int n, int64_t d, int p, int s,
                              const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2, const int32_t* Q2_len,
                              const double* theta, uint64_t seed, float* Xhat, int32_t* status, cudaStream_t st);

}  // namespace ecasq
