// Unbiased stochastic rounding onto a code Q, two-way time-sharing and the
// empirical entropy of the emitted indices.
//
// ECASQ summary (gist.science/pt/paper/2608.18147):
//   §1   unbiasedness E[X^] = X: an entry x in [q_i, q_{i+1}] is emitted as
//        q_{i+1} with probability (x - q_i)/(q_{i+1} - q_i), else q_i; the
//        quantity constrained is the entropy H(X^) of the emitted values;
//   §2.1 two-way time-sharing: two quantizers run on a random partition of the
//        input, a share theta of the entries on Q1 and the rest on Q2.
// Randomness: Philox4x32-10 keyed by the seed, counter (j >> 2, row, stream, 0);
// word j & 3 serves entry j. Stream 0 draws the rounding, stream 1 the
// partition. Each thread owns four consecutive entries, so one Philox block per
// stream serves one float4 of X.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {
namespace {

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / kWarp;
constexpr int64_t kEncChunk = 16384;  // entries per CTA (multiple of 4)

// Rounding test: x in [q_t, q_{t+1}] goes up iff u * (q_{t+1} - q_t) < x - q_t,
// i.e. u < (x - q_t)/(q_{t+1} - q_t) with the division moved across; each side
// is one IEEE fp64 operation, so the decision is reproducible on any IEEE
// machine. x = q_t never goes up, x = q_{t+1} always does.
__global__ void __launch_bounds__(kEncThreads)
k_encode(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d, int p, int s,
         const int32_t* __restrict__ Q1, const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
         const int32_t* __restrict__ Q2_len, const double* __restrict__ theta, uint32_t key0, uint32_t key1,
         uint8_t* __restrict__ idx, unsigned long long* __restrict__ hist, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = blockIdx.y;
  double* sP = reinterpret_cast<double*>(smem);   // [p]
  double* sq = sP + p;                             // [2][s] code values
  double* sw = sq + 2 * s;                         // [2][s] interval widths q_{t+1} - q_t
  unsigned int* sh = reinterpret_cast<unsigned int*>(sw + 2 * s);      // [warps][2s] counts
  float* sT = reinterpret_cast<float*>(sh + kEncWarps * 2 * s);                     // [p] exact fp32 thresholds
  unsigned char* imap = reinterpret_cast<unsigned char*>(sT + p);                      // [2][p]
  __shared__ int s_m[2];
  __shared__ int s_bad;

  const double* P = Pall + static_cast<int64_t>(r) * p;
  const bool has2 = (Q2 != nullptr);
  const double th = (has2 && theta) ? theta[r] : 0.0;
  const bool mix = has2 && th > 0.0 && th < 1.0;
  const int fixed_part = (!has2 || th >= 1.0) ? 0 : 1;
  const int nbins = 2 * s;

  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    sP[k] = P[k];
    sT[k] = __double2float_ru(P[k]);
  }
  if (threadIdx.x == 0) {
    s_bad = 0;
    s_m[0] = Q1_len[r];
    s_m[1] = has2 ? Q2_len[r] : 0;
  }
  for (int k = threadIdx.x; k < 2 * p; k += blockDim.x) imap[k] = 255;
  for (int k = threadIdx.x; k < kEncWarps * nbins; k += blockDim.x) sh[k] = 0u;
  __syncthreads();
  // A code must hold 1..s increasing indices into P; anything else marks the
  // row invalid and leaves its outputs untouched.
  {
    int bad_code = 0;
    for (int part = 0; part < 2; ++part) {
      const int m = s_m[part];
      const int32_t* Q = (part == 0 ? Q1 : Q2);
      const bool used = (part == 0) ? (fixed_part == 0 || mix) : (fixed_part == 1 || mix);
      if (!used) continue;
      if (Q == nullptr || m < 1 || m > s) {
        bad_code = 1;
        continue;
      }
      const int32_t* q = Q + static_cast<int64_t>(r) * s;
      for (int t = threadIdx.x; t < m; t += blockDim.x)
        if (q[t] < 0 || q[t] >= p || (t > 0 && q[t] <= q[t - 1])) bad_code = 1;
    }
    if (__syncthreads_or(bad_code)) {
      if (threadIdx.x == 0) status[r] = kStatusArg;
      return;
    }
  }
  // Code values, interval widths and the bucket -> interval map of each part.
  for (int part = 0; part < 2; ++part) {
    const int m = s_m[part];
    const int32_t* Q = (part == 0 ? Q1 : Q2);
    const bool used = (part == 0) ? (fixed_part == 0 || mix) : (fixed_part == 1 || mix);
    if (!used) continue;
    const int32_t* q = Q + static_cast<int64_t>(r) * s;
    for (int t = threadIdx.x; t < m; t += blockDim.x) {
      sq[part * s + t] = sP[q[t]];
      if (t + 1 < m) sw[part * s + t] = __dsub_rn(sP[q[t + 1]], sP[q[t]]);
    }
    for (int t = threadIdx.x; t < m - 1; t += blockDim.x)
      for (int k = q[t]; k < q[t + 1]; ++k) imap[part * p + k] = static_cast<unsigned char>(t);
  }
  __syncthreads();

  // Part test u < theta with u = sel * 2^-32: theta * 2^32 is exact in fp64 and
  // sel is an integer, so it is sel < ceil(theta * 2^32) (at most 2^32).
  const uint64_t th_cut = mix ? static_cast<uint64_t>(ceil(th * 0x1p32)) : 0;
  const float scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
  const float top = __double2float_rd(sP[p - 1]);
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * kEncChunk;
  const int64_t end = beg + kEncChunk < d ? beg + kEncChunk : d;
  const float* x = X + static_cast<int64_t>(r) * d;
  uint8_t* o = idx + static_cast<int64_t>(r) * d;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) && ((d & 3) == 0);
  unsigned int* wh = sh + warp_id() * nbins;
  int bad = 0;

  for (int64_t g = beg + 4 * static_cast<int64_t>(threadIdx.x); g < end; g += 4 * kEncThreads) {
    float xv[4];
    const int cnt = (end - g) >= 4 ? 4 : static_cast<int>(end - g);
    if (vec && cnt == 4) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(x + g));
      xv[0] = v.x;
      xv[1] = v.y;
      xv[2] = v.z;
      xv[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) xv[e] = (e < cnt) ? __ldcs(x + g + e) : 0.0f;
    }
    const uint32_t blk = static_cast<uint32_t>(static_cast<uint64_t>(g) >> 2);
    const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), key0, key1);
    uint4 su = make_uint4(0u, 0u, 0u, 0u);
    if (mix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), key0, key1);
    const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
    const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e >= cnt) break;
      const double xd = static_cast<double>(xv[e]);
      int part = fixed_part;
      if (mix) part = (static_cast<uint64_t>(sel[e]) < th_cut) ? 0 : 1;
      const int m = s_m[part];
      int out = 0;
      if (m == 1) {
        if (xd != sq[part * s]) bad = 1;
      } else {
        const int k = bucket_f32(xv[e], sT, top, p, scale);
        int t = (k >= 0) ? imap[part * p + k] : 255;
        if (t == 255) {
          if (xd == sq[part * s + m - 1])
            t = m - 2;
          else
            bad = 1;
        }
        if (t != 255) {
          const double y = __dsub_rn(xd, sq[part * s + t]);
          const double u = static_cast<double>(rw[e]) * 0x1p-32;
          out = t + ((__dmul_rn(u, sw[part * s + t]) < y) ? 1 : 0);
        }
      }
      packed |= static_cast<uint32_t>(out) << (8 * e);
      atomicAdd(wh + part * s + out, 1u);
    }
    if (cnt == 4 && ((reinterpret_cast<uintptr_t>(o + g) & 3u) == 0)) {
      *reinterpret_cast<uint32_t*>(o + g) = packed;
    } else {
      for (int e = 0; e < cnt; ++e) o[g + e] = static_cast<uint8_t>(packed >> (8 * e));
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();
  unsigned long long* gh = hist + static_cast<int64_t>(r) * nbins;
  for (int b = threadIdx.x; b < nbins; b += blockDim.x) {
    unsigned long long tot = 0;
#pragma unroll
    for (int w = 0; w < kEncWarps; ++w) tot += sh[w * nbins + b];
    if (tot) atomicAdd(gh + b, tot);
  }
  if (threadIdx.x == 0 && s_bad) status[r] = kStatusRange;
}

// H = (d0 H0 + d1 H1)/(d0 + d1), H_part = -sum c/d_part log2(c/d_part). One warp per row.
__global__ void k_entropy(const int64_t* __restrict__ hist, int n, int s, double* __restrict__ H) {
  const int r = blockIdx.x * (blockDim.x / kWarp) + warp_id();
  if (r >= n) return;
  const int64_t* h = hist + static_cast<int64_t>(r) * 2 * s;
  double acc = 0.0, tot = 0.0;
  for (int part = 0; part < 2; ++part) {
    double dp = 0.0;
    for (int t = lane_id(); t < s; t += kWarp) dp += static_cast<double>(h[part * s + t]);
    dp = warp_sum(dp);
    if (dp <= 0.0) continue;
    double hp = 0.0;
    for (int t = lane_id(); t < s; t += kWarp) {
      const double c = static_cast<double>(h[part * s + t]);
      if (c > 0.0) hp -= (c / dp) * log2(c / dp);
    }
    hp = warp_sum(hp);
    acc += dp * hp;
    tot += dp;
  }
  if (lane_id() == 0) H[r] = tot > 0.0 ? acc / tot : 0.0;
}

size_t encode_smem(int p, int s) {
  return sizeof(double) * (p + 4 * s) + sizeof(unsigned int) * kEncWarps * 2 * s + sizeof(float) * p + 2 * p;
}

}  // namespace

cudaError_t launch_encode(const float* X, const double* P, int n, int64_t d, int p, int s,
                          const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2,
                          const int32_t* Q2_len, const double* theta, uint64_t seed, uint8_t* idx,
                          int64_t* hist, int32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(int64_t) * 2 * s * static_cast<size_t>(n), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(status, 0, sizeof(int32_t) * n, st);
  if (e != cudaSuccess) return e;
  const int nc = static_cast<int>((d + kEncChunk - 1) / kEncChunk);
  const size_t smem = encode_smem(p, s);
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  k_encode<<<dim3(nc, n), kEncThreads, smem, st>>>(X, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, k0, k1, idx,
                                                    reinterpret_cast<unsigned long long*>(hist), status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_entropy(const int64_t* hist, int n, int s, double* H, cudaStream_t st) {
  const int wpb = 8;
  k_entropy<<<(n + wpb - 1) / wpb, wpb * kWarp, 0, st>>>(hist, n, s, H);
  note_launch();
  return cudaGetLastError();
}

}  // namespace ecasq
