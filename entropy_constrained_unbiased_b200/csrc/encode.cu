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

// Per-CTA state of the encoder in shared memory: the row's alphabet, both
// codes, and the per-bucket records of the fast path.
struct EncRow {
  const double* P;       // [p]
  const float* T;        // [p] smallest float >= P_k
  const double* q;       // [2][s] code values
  const double* w;       // [2][s] widths q_{t+1} - q_t
  const unsigned char* tmap;  // [2][p] bucket -> interval (255: none)
  unsigned int* hist;    // [warps][2s + 1] (bin 2s: entries the fast path left to the exact one)
  int p, s, m[2];
  float top, scale;
  int bad;
};

// Rounding test: x in [q_t, q_{t+1}] goes up iff u * (q_{t+1} - q_t) < x - q_t,
// i.e. u < (x - q_t)/(q_{t+1} - q_t) with the division moved across; each side
// is one IEEE fp64 operation, so the decision is reproducible on any IEEE
// machine. x = q_t never goes up, x = q_{t+1} always does.
//
// Exact coding of one entry of part `part` (any code, any row): the threshold
// search for the bucket, the top code value beyond the alphabet's last bucket,
// one-value codes, entries outside the code's range (flagged).
__device__ __forceinline__ int enc_exact(EncRow& S, float xf, int part, uint32_t word) {
  const int m = S.m[part], s = S.s;
  const double xd = static_cast<double>(xf);
  if (m == 1) {
    if (xd != S.q[part * s]) S.bad = 1;
    return 0;
  }
  const int k = bucket_f32(xf, S.T, S.top, S.p, S.scale);
  const int t = (k >= 0) ? S.tmap[part * S.p + k] : 255;
  if (t == 255) {
    if (xd == S.q[part * s + m - 1]) return m - 1;
    S.bad = 1;
    return 0;
  }
  const double y = __dsub_rn(xd, S.q[part * s + t]);
  const double prod = __dmul_rn(__dmul_rn(static_cast<double>(word), 0x1p-32), S.w[part * s + t]);
  return t + ((prod < y) ? 1 : 0);
}

// The entries of a group of up to four that the fast path did not decide (bit
// e of okm clear): exact code, histogram, byte in `packed`. Kept out of line so
// that the fast loop carries none of it.
__device__ __noinline__ uint32_t enc_fix(EncRow* S, const float* xv, const uint32_t* rw, const int* part, int cnt,
                                         unsigned okm, uint32_t packed) {
  unsigned int* wh = S->hist + warp_id() * (2 * S->s + 1);
  for (int e = 0; e < cnt; ++e) {
    if (okm & (1u << e)) continue;
    const int out = enc_exact(*S, xv[e], part[e], rw[e]);
    atomicAdd(wh + part[e] * S->s + out, 1u);
    packed = (packed & ~(0xFFu << (8 * e))) | (static_cast<uint32_t>(out) << (8 * e));
  }
  return packed;
}

// Bucket of an entry on the fast path: on rows whose alphabet is a uniform
// grid (every P_k within 2^-36 bucket widths of P_0 + k D), g = x s + c in fp32
// with s = 1/D, c = -P_0/D; when g - floor(g) is farther from 0 and 1 than the
// error bound of that evaluation (plus 2^-36), floor(g) is the bucket for
// certain. Per bucket k and part a record holds the code value q_t of its
// interval and w' = (q_{t+1} - q_t) 2^-32; with u = word 2^-32 (both scalings
// exact) u (q_{t+1} - q_t) = word w' as real numbers, so the product is
// taken as word * w' in one rounding.
template <bool kMix>
__device__ __forceinline__ void encode_row(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d,
                                           int p, int s, const int32_t* __restrict__ Q1,
                                           const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
                                           const int32_t* __restrict__ Q2_len, const double* __restrict__ theta,
                                           const Philox4x32::RoundKeys& K, uint8_t* __restrict__ idx,
                                           unsigned long long* __restrict__ hist, int32_t* __restrict__ status,
                                           unsigned char* smem, EncRow& S, int& s_wexact) {
  const int r = blockIdx.y;
  const int nbins = 2 * s + 1;
  double2* sR = reinterpret_cast<double2*>(smem);                          // [2][p] (q_t, w') per bucket
  double* sP = reinterpret_cast<double*>(sR + 2 * p);                       // [p]
  double* sq = sP + p;                                                      // [2][s] code values
  double* sw = sq + 2 * s;                                                  // [2][s] widths
  unsigned int* sh = reinterpret_cast<unsigned int*>(sw + 2 * s);           // [warps][2s + 1] counts
  float* sT = reinterpret_cast<float*>(sh + kEncWarps * nbins);             // [p] exact fp32 thresholds
  unsigned char* tmap = reinterpret_cast<unsigned char*>(sT + p);           // [2][p] bucket -> interval

  const double* P = Pall + static_cast<int64_t>(r) * p;
  const bool has2 = (Q2 != nullptr);
  const double th = (has2 && theta) ? theta[r] : 0.0;
  const bool mix = has2 && th > 0.0 && th < 1.0;
  const int fixed_part = (!has2 || th >= 1.0) ? 0 : 1;

  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    sP[k] = P[k];
    sT[k] = __double2float_ru(P[k]);
  }
  if (threadIdx.x == 0) {
    S.P = sP;
    S.T = sT;
    S.q = sq;
    S.w = sw;
    S.tmap = tmap;
    S.hist = sh;
    S.p = p;
    S.s = s;
    S.m[0] = Q1_len[r];
    S.m[1] = has2 ? Q2_len[r] : 0;
    S.bad = 0;
    s_wexact = 1;
  }
  for (int k = threadIdx.x; k < 2 * p; k += blockDim.x) {
    tmap[k] = 255;
    sR[k] = make_double2(0.0, 0.0);
  }
  for (int k = threadIdx.x; k < kEncWarps * nbins; k += blockDim.x) sh[k] = 0u;
  __syncthreads();
  // A code must hold 1..s increasing indices into P; anything else marks the
  // row invalid and leaves its outputs untouched.
  {
    int bad_code = 0;
    for (int part = 0; part < 2; ++part) {
      const int m = S.m[part];
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
  // Code values, widths, the bucket -> interval map and the per-bucket records.
  bool single = false;  // a used code with one value
  for (int part = 0; part < 2; ++part) {
    const int m = S.m[part];
    const int32_t* Q = (part == 0 ? Q1 : Q2);
    const bool used = (part == 0) ? (fixed_part == 0 || mix) : (fixed_part == 1 || mix);
    if (!used) continue;
    if (m == 1) single = true;
    const int32_t* q = Q + static_cast<int64_t>(r) * s;
    for (int t = threadIdx.x; t < m; t += blockDim.x) {
      sq[part * s + t] = sP[q[t]];
      if (t + 1 < m) {
        const double w = __dsub_rn(sP[q[t + 1]], sP[q[t]]);
        const double ws = __dmul_rn(w, 0x1p-32);
        sw[part * s + t] = w;
        if (!(__dmul_rn(ws, 0x1p32) == w) || !(ws >= 0x1p-1022)) s_wexact = 0;  // scaling not exact
        for (int k = q[t]; k < q[t + 1]; ++k) {
          tmap[part * p + k] = static_cast<unsigned char>(t);
          sR[part * p + k] = make_double2(sP[q[t]], ws);
        }
      }
    }
  }
  const RowGrid g = row_grid(sP, p);
  const bool uni = row_is_uniform(sP, p, g, nullptr);  // includes a barrier
  const float s_f = static_cast<float>(g.invD);
  const float c_f = static_cast<float>(-(g.P0 * g.invD));
  float eps_f = 1.0f;
  if (uni) {
    const double M = fmax(fabs(g.P0), fabs(sP[p - 1]));
    const double bound = 0x1p-23 * (static_cast<double>(p) + 1.0 + 3.0 * M * g.invD) + 0x1p-30;
    if (bound < 0x1p-6) eps_f = static_cast<float>(bound);
  }
  if (threadIdx.x == 0) {
    S.scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
    S.top = __double2float_rd(sP[p - 1]);
  }
  __syncthreads();
  const bool fast = uni && !single && s_wexact != 0 && eps_f < 1.0f;

  // Part test u < theta with u = sel * 2^-32: theta * 2^32 is exact in fp64 and
  // sel is an integer, so it is sel < ceil(theta * 2^32), i.e. sel <= cut - 1
  // (cut >= 1 whenever theta > 0).
  const uint32_t th_last = mix ? static_cast<uint32_t>(static_cast<uint64_t>(ceil(th * 0x1p32)) - 1u) : 0u;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * kEncChunk;
  const int len = static_cast<int>((beg + kEncChunk < d ? beg + kEncChunk : d) - beg);
  const float* x = X + static_cast<int64_t>(r) * d + beg;
  uint8_t* o = idx + static_cast<int64_t>(r) * d + beg;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) && ((reinterpret_cast<uintptr_t>(o) & 3u) == 0);
  const int nf = vec ? (len >> 2) : 0;  // full float4 groups on the vector path
  unsigned int* wh = sh + warp_id() * nbins;
  const int trash = 2 * s;
  const uint32_t blk0 = static_cast<uint32_t>(static_cast<uint64_t>(beg) >> 2);
  Philox4x32::RoundKeys rk;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    rk.k0[i] = K.k0[i];
    rk.k1[i] = K.k1[i];
  }

  if (fast) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    uint32_t* o4 = reinterpret_cast<uint32_t*>(o);
    const unsigned pm2 = static_cast<unsigned>(p - 2);
    const float lim = 0.5f - eps_f;
    for (int f = threadIdx.x; f < nf; f += kEncThreads) {
      const float4 v = __ldcs(x4 + f);
      const float xv[4] = {v.x, v.y, v.z, v.w};
      const uint32_t blk = blk0 + static_cast<uint32_t>(f);
      const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), rk);
      uint4 su = make_uint4(0u, 0u, 0u, 0u);
      if (kMix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), rk);
      const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
      const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
      int part[4];
      uint32_t packed = 0;
      unsigned okm = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        part[e] = kMix ? (sel[e] <= th_last ? 0 : 1) : fixed_part;
        const float gf = fmaf(xv[e], s_f, c_f);
        const float kf = floorf(gf);
        const int k = static_cast<int>(kf);
        const bool kin = static_cast<unsigned>(k) <= pm2;
        const int pk = part[e] * p + (kin ? k : 0);
        const double2 rec = sR[pk];
        const int t = tmap[pk];
        const bool ok = kin && fabsf((gf - kf) - 0.5f) < lim && t != 255;
        const double y = __dsub_rn(static_cast<double>(xv[e]), rec.x);
        const double prod = __dmul_rn(static_cast<double>(rw[e]), rec.y);
        const int out = t + ((prod < y) ? 1 : 0);
        atomicAdd(wh + (ok ? part[e] * s + out : trash), 1u);
        packed |= static_cast<uint32_t>(out & 0xFF) << (8 * e);
        okm |= ok ? (1u << e) : 0u;
      }
      if (okm != 0xFu) packed = enc_fix(&S, xv, rw, part, 4, okm, packed);
      o4[f] = packed;
    }
  }
  // every other entry (rows off the fast path, unaligned rows, the last < 4
  // entries) through the exact coding
  for (int j = 4 * nf + 4 * threadIdx.x; j < len; j += 4 * kEncThreads) {
    const int cnt = len - j < 4 ? len - j : 4;
    float xv[4] = {0.f, 0.f, 0.f, 0.f};
    for (int e = 0; e < cnt; ++e) xv[e] = __ldcs(x + j + e);
    // the Philox counter block of entry j is its index in the row >> 2
    const uint32_t blk = blk0 + static_cast<uint32_t>(j >> 2);
    const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), rk);
    uint4 su = make_uint4(0u, 0u, 0u, 0u);
    if (mix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), rk);
    const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
    const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
    int part[4];
    for (int e = 0; e < 4; ++e) part[e] = mix ? (sel[e] <= th_last ? 0 : 1) : fixed_part;
    const uint32_t packed = enc_fix(&S, xv, rw, part, cnt, 0u, 0u);
    for (int e = 0; e < cnt; ++e) o[j + e] = static_cast<uint8_t>(packed >> (8 * e));
  }
  __syncthreads();
  unsigned long long* gh = hist + static_cast<int64_t>(r) * 2 * s;
  for (int b = threadIdx.x; b < 2 * s; b += blockDim.x) {
    unsigned long long tot = 0;
#pragma unroll
    for (int w = 0; w < kEncWarps; ++w) tot += sh[w * nbins + b];
    if (tot) atomicAdd(gh + b, tot);
  }
  if (threadIdx.x == 0 && S.bad) status[r] = kStatusRange;
}

// One CTA per (row, chunk of kEncChunk entries); rows coded with two codes
// (0 < theta < 1) and rows coded with one take separate specialisations.
__global__ void __launch_bounds__(kEncThreads)
k_encode(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d, int p, int s,
         const int32_t* __restrict__ Q1, const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
         const int32_t* __restrict__ Q2_len, const double* __restrict__ theta, const Philox4x32::RoundKeys K,
         uint8_t* __restrict__ idx, unsigned long long* __restrict__ hist, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ EncRow S;
  __shared__ int s_wexact;
  const double th = (Q2 != nullptr && theta) ? theta[blockIdx.y] : 0.0;
  if (Q2 != nullptr && th > 0.0 && th < 1.0)
    encode_row<true>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, smem, S, s_wexact);
  else
    encode_row<false>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, smem, S, s_wexact);
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
  return sizeof(double2) * 2 * p + sizeof(double) * (p + 4 * s) + sizeof(unsigned int) * kEncWarps * (2 * s + 1) +
         sizeof(float) * p + 2 * p;
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
  const Philox4x32::RoundKeys K =
      Philox4x32::round_keys(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  k_encode<<<dim3(nc, n), kEncThreads, smem, st>>>(X, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx,
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
