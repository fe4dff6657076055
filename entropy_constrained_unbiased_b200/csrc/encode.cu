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
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {
namespace {

constexpr int kEncThreads = 256;
constexpr int kEncWarps = kEncThreads / kWarp;
constexpr int64_t kEncChunk = 65536;    // entries per encoder CTA on grids that fill the GPU
constexpr int64_t kEncMinChunk = 4096;  // fewest entries per encoder CTA
constexpr int kEncCtasPerSm = 5;         // resident encoder CTAs per SM (48 registers a thread)
constexpr int64_t kDeqChunk = 32768;  // entries per reconstruction CTA on grids that fill the GPU
constexpr int kDeqCtasPerSm = 8;      // resident reconstruction CTAs per SM

// Per-CTA state of the encoder in shared memory: the row's alphabet, both
// codes, and the per-bucket records of the fast path.
struct EncRow {
  const double* P;       // [p]
  const float* T;        // [p] smallest float >= P_k
  const double* q;       // [2][s] code values
  const int32_t* qi;     // [2][s] code indices into P
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
  const double w = __dsub_rn(S.P[S.qi[part * s + t + 1]], S.P[S.qi[part * s + t]]);
  const double prod = __dmul_rn(__dmul_rn(static_cast<double>(word), 0x1p-32), w);
  return t + ((prod < y) ? 1 : 0);
}

// Exact code of one entry that the fast path did not decide, with its
// histogram count; kept out of line (scalar arguments, so that the fast loop
// keeps its values in registers) so that the fast loop carries none of it.
// One instance per kernel (kTag): a callee shared by two kernels gets a
// calling convention fitted to neither, and the fast loop spills more.
template <int kTag>
__device__ __noinline__ int enc_fix1(EncRow* S, float x, uint32_t word, int part) {
  const int out = enc_exact(*S, x, part, word);
  red_shared_inc(smem_addr(S->hist + warp_id() * (2 * S->s + 1) + part * S->s + out));
  return out;
}

// Bucket of an entry on the fast path: on rows whose alphabet is a uniform
// grid (every P_k within 2^-36 bucket widths of P_0 + k D), g = x s + c in fp32
// with s = 1/D, c = -P_0/D; when g - floor(g) is farther from 0 and 1 than the
// error bound of that evaluation (plus 2^-36), floor(g) is the bucket for
// certain. Per bucket k and part a record holds the code value q_t of its
// interval and w' = (q_{t+1} - q_t) 2^-32; with u = word 2^-32 (both scalings
// exact) u (q_{t+1} - q_t) = word w' as real numbers, so the product is
// taken as word * w' in one rounding.
template <bool kMix, int kTag>
__device__ __forceinline__ void encode_row(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d,
                                           int p, int s, const int32_t* __restrict__ Q1,
                                           const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
                                           const int32_t* __restrict__ Q2_len, const double* __restrict__ theta,
                                           const Philox4x32::RoundKeys& K, uint8_t* __restrict__ idx,
                                           unsigned long long* __restrict__ hist, int32_t* __restrict__ status,
                                           int64_t chunk, unsigned char* smem, EncRow& S, int& s_wexact) {
  const int r = blockIdx.y;
  const int nbins = 2 * s + 1;
  double2* sR = reinterpret_cast<double2*>(smem);                          // [2][p] (q_t, w') per bucket
  double* sP = reinterpret_cast<double*>(sR + 2 * p);                       // [p]
  double* sq = sP + p;                                                      // [2][s] code values
  unsigned int* sh = reinterpret_cast<unsigned int*>(sq + 2 * s);           // [warps][2s + 1] counts
  float* sT = reinterpret_cast<float*>(sh + kEncWarps * nbins);             // [p] exact fp32 thresholds
  int32_t* sqi = reinterpret_cast<int32_t*>(sT + p);                      // [2][s] code indices
  unsigned char* tmap = reinterpret_cast<unsigned char*>(sqi + 2 * s);      // [2][p] bucket -> interval

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
    S.qi = sqi;
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
        if (!(__dmul_rn(ws, 0x1p32) == w) || !(ws >= 0x1p-1022)) s_wexact = 0;  // scaling not exact
      }
    }
    for (int t = threadIdx.x; t < m; t += blockDim.x) sqi[part * s + t] = q[t];
  }
  __syncthreads();
  // bucket k lies in interval t = max{t <= m-2 : q_t <= k} when q_0 <= k < q_{m-1}
  for (int part = 0; part < 2; ++part) {
    const int m = S.m[part];
    const bool used = (part == 0) ? (fixed_part == 0 || mix) : (fixed_part == 1 || mix);
    if (!used || m < 2) continue;
    const int32_t* qi = sqi + part * s;
    for (int k = threadIdx.x; k < p; k += blockDim.x) {
      if (k < qi[0] || k >= qi[m - 1]) continue;
      int lo = 0, hi = m - 2;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (qi[mid] <= k)
          lo = mid;
        else
          hi = mid - 1;
      }
      tmap[part * p + k] = static_cast<unsigned char>(lo);
      const double w = __dsub_rn(sP[qi[lo + 1]], sP[qi[lo]]);
      sR[part * p + k] = make_double2(sq[part * s + lo], __dmul_rn(w, 0x1p-32));
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
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int len = static_cast<int>((beg + chunk < d ? beg + chunk : d) - beg);
  const float* x = X + static_cast<int64_t>(r) * d + beg;
  uint8_t* o = idx + static_cast<int64_t>(r) * d + beg;
  const bool vec = ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) && ((reinterpret_cast<uintptr_t>(o) & 3u) == 0);
  const int nf = vec ? (len >> 2) : 0;  // full float4 groups on the vector path
  const uint32_t wh_base = smem_addr(sh + warp_id() * nbins);
  const int trash = 2 * s;
  // histogram word addresses: part 1's bins, the fixed part's, the trash bin
  const uint32_t wh_p1 = wh_base + 4u * static_cast<uint32_t>(s);
  const uint32_t wh_fixed = wh_base + 4u * static_cast<uint32_t>(fixed_part * s);
  const uint32_t wh_trash = wh_base + 4u * static_cast<uint32_t>(trash);
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
    float4 nxt = (threadIdx.x < nf) ? __ldcs(x4 + threadIdx.x) : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int f = threadIdx.x; f < nf; f += kEncThreads) {
      const float4 v = nxt;
      if (f + kEncThreads < nf) nxt = __ldcs(x4 + f + kEncThreads);
      const float xv[4] = {v.x, v.y, v.z, v.w};
      const uint32_t blk = blk0 + static_cast<uint32_t>(f);
      const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), rk);
      uint4 su = make_uint4(0u, 0u, 0u, 0u);
      if (kMix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), rk);
      const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
      const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
      int part[4];
      uint32_t ob[4];
      bool allok = true;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        part[e] = kMix ? (sel[e] <= th_last ? 0 : 1) : fixed_part;
        // floor(g) by rounding (g - 0.5) to an integer with 1.5 * 2^23 (exact for
        // 0 <= g < 2^22; at integer g the fractional test below fails)
        const float gf = fmaf(xv[e], s_f, c_f);
        const float tf = __fadd_rn(__fadd_rn(gf, -0.5f), 12582912.0f);
        const float kf = __fsub_rn(tf, 12582912.0f);
        const int k = __float_as_int(tf) - 0x4B400000;
        const bool kin = static_cast<unsigned>(k) <= pm2;
        const int pk = part[e] * p + (kin ? k : 0);
        const double2 rec = sR[pk];
        const int t = tmap[pk];
        const bool ok = kin && fabsf((gf - kf) - 0.5f) < lim && t != 255;
        const double y = __dsub_rn(static_cast<double>(xv[e]), rec.x);
        const double prod = __dmul_rn(static_cast<double>(rw[e]), rec.y);
        const int out = t + ((prod < y) ? 1 : 0);
        const uint32_t hb = kMix ? (part[e] ? wh_p1 : wh_base) : wh_fixed;
        red_shared_inc(ok ? hb + 4u * static_cast<uint32_t>(out) : wh_trash);
        ob[e] = static_cast<uint32_t>(out);
        allok = allok && ok;
      }
      // bytes 0 of ob[0..3] into one word (out <= 255 on the fast path)
      uint32_t packed = __byte_perm(__byte_perm(ob[0], ob[1], 0x0040), __byte_perm(ob[2], ob[3], 0x0040), 0x5410);
      if (!allok) {
        // the rare entries off the fast path: redo the test and code them exactly
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float gf = fmaf(xv[e], s_f, c_f);
          const float tf = __fadd_rn(__fadd_rn(gf, -0.5f), 12582912.0f);
          const float kf = __fsub_rn(tf, 12582912.0f);
          const int k = __float_as_int(tf) - 0x4B400000;
          const bool kin = static_cast<unsigned>(k) <= pm2;
          const int t = tmap[part[e] * p + (kin ? k : 0)];
          const bool ok = kin && fabsf((gf - kf) - 0.5f) < lim && t != 255;
          if (!ok) {
            const int out = enc_fix1<kTag>(&S, xv[e], rw[e], part[e]);
            packed = (packed & ~(0xFFu << (8 * e))) | (static_cast<uint32_t>(out) << (8 * e));
          }
        }
      }
      o4[f] = packed;
    }
  }
  // every other entry (rows off the fast path, unaligned rows, the last < 4
  // entries) through the exact coding
  for (int j = 4 * nf + 4 * threadIdx.x; j < len; j += 4 * kEncThreads) {
    const int cnt = len - j < 4 ? len - j : 4;
    float xv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < cnt) xv[e] = __ldcs(x + j + e);
    // the Philox counter block of entry j is its index in the row >> 2
    const uint32_t blk = blk0 + static_cast<uint32_t>(j >> 2);
    const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), rk);
    uint4 su = make_uint4(0u, 0u, 0u, 0u);
    if (mix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), rk);
    const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
    const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e < cnt) {
        const int part = mix ? (sel[e] <= th_last ? 0 : 1) : fixed_part;
        o[j + e] = static_cast<uint8_t>(enc_fix1<kTag>(&S, xv[e], rw[e], part));
      }
    }
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
__global__ void __launch_bounds__(kEncThreads, kEncCtasPerSm)
k_encode(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d, int p, int s,
         const int32_t* __restrict__ Q1, const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
         const int32_t* __restrict__ Q2_len, const double* __restrict__ theta, const Philox4x32::RoundKeys K,
         uint8_t* __restrict__ idx, unsigned long long* __restrict__ hist, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ EncRow S;
  __shared__ int s_wexact;
  const double th = (Q2 != nullptr && theta) ? theta[blockIdx.y] : 0.0;
  if (Q2 != nullptr && th > 0.0 && th < 1.0)
    encode_row<true, 0>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, kEncChunk, smem, S,
                     s_wexact);
  else
    encode_row<false, 0>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, kEncChunk, smem, S,
                      s_wexact);
}

// k_encode with chunks of `chunk` entries (a multiple of 4, below kEncChunk),
// for grids of few or short rows that kEncChunk would leave part-empty.
__global__ void __launch_bounds__(kEncThreads, kEncCtasPerSm)
k_encode_chunked(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d, int p, int s,
                 const int32_t* __restrict__ Q1, const int32_t* __restrict__ Q1_len,
                 const int32_t* __restrict__ Q2, const int32_t* __restrict__ Q2_len,
                 const double* __restrict__ theta, const Philox4x32::RoundKeys K, uint8_t* __restrict__ idx,
                 unsigned long long* __restrict__ hist, int32_t* __restrict__ status, int64_t chunk) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ EncRow S;
  __shared__ int s_wexact;
  const double th = (Q2 != nullptr && theta) ? theta[blockIdx.y] : 0.0;
  if (Q2 != nullptr && th > 0.0 && th < 1.0)
    encode_row<true, 1>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, chunk, smem, S,
                     s_wexact);
  else
    encode_row<false, 1>(X, Pall, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx, hist, status, chunk, smem, S,
                      s_wexact);
}

// Encoder for large alphabets (p > 512): no per-bucket tables; the interval of
// an entry is found by bisection over the code's values (at most 256), the
// largest t <= m-2 with q_t <= x, exactly as the rounding rule reads. Same
// randomness, tests and outputs as k_encode.
__global__ void __launch_bounds__(kEncThreads)
k_encode_code(const float* __restrict__ X, const double* __restrict__ Pall, int64_t d, int p, int s,
              const int32_t* __restrict__ Q1, const int32_t* __restrict__ Q1_len, const int32_t* __restrict__ Q2,
              const int32_t* __restrict__ Q2_len, const double* __restrict__ theta, const Philox4x32::RoundKeys K,
              uint8_t* __restrict__ idx, unsigned long long* __restrict__ hist, int32_t* __restrict__ status,
              int64_t chunk) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int s_m[2];
  __shared__ int s_bad;
  const int r = blockIdx.y;
  double* sq = reinterpret_cast<double*>(smem);                      // [2][s] code values
  unsigned int* sh = reinterpret_cast<unsigned int*>(sq + 2 * s);   // [warps][2s] counts
  const int nbins = 2 * s;
  const double* P = Pall + static_cast<int64_t>(r) * p;
  const bool has2 = (Q2 != nullptr);
  const double th = (has2 && theta) ? theta[r] : 0.0;
  const bool mix = has2 && th > 0.0 && th < 1.0;
  const int fixed_part = (!has2 || th >= 1.0) ? 0 : 1;
  if (threadIdx.x == 0) {
    s_bad = 0;
    s_m[0] = Q1_len[r];
    s_m[1] = has2 ? Q2_len[r] : 0;
  }
  for (int k = threadIdx.x; k < kEncWarps * nbins; k += blockDim.x) sh[k] = 0u;
  __syncthreads();
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
    for (int t = threadIdx.x; t < m; t += blockDim.x) {
      if (q[t] < 0 || q[t] >= p || (t > 0 && q[t] <= q[t - 1]))
        bad_code = 1;
      else
        sq[part * s + t] = P[q[t]];
    }
  }
  if (__syncthreads_or(bad_code)) {
    if (threadIdx.x == 0) status[r] = kStatusArg;
    return;
  }
  const uint32_t th_last = mix ? static_cast<uint32_t>(static_cast<uint64_t>(ceil(th * 0x1p32)) - 1u) : 0u;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int len = static_cast<int>((beg + chunk < d ? beg + chunk : d) - beg);
  const float* x = X + static_cast<int64_t>(r) * d + beg;
  uint8_t* o = idx + static_cast<int64_t>(r) * d + beg;
  const uint32_t blk0 = static_cast<uint32_t>(static_cast<uint64_t>(beg) >> 2);
  const uint32_t wh_base = smem_addr(sh + warp_id() * nbins);
  int bad = 0;
  for (int j = 4 * threadIdx.x; j < len; j += 4 * kEncThreads) {
    const int cnt = len - j < 4 ? len - j : 4;
    const uint32_t blk = blk0 + static_cast<uint32_t>(j >> 2);
    const uint4 ru = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 0u, 0u), K);
    uint4 su = make_uint4(0u, 0u, 0u, 0u);
    if (mix) su = Philox4x32::block(make_uint4(blk, static_cast<uint32_t>(r), 1u, 0u), K);
    const uint32_t rw[4] = {ru.x, ru.y, ru.z, ru.w};
    const uint32_t sel[4] = {su.x, su.y, su.z, su.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e >= cnt) continue;
      const int part = mix ? (sel[e] <= th_last ? 0 : 1) : fixed_part;
      const int m = s_m[part];
      const double* qv = sq + part * s;
      const double xd = static_cast<double>(__ldcs(x + j + e));
      int out = 0;
      if (m == 1) {
        if (xd != qv[0]) bad = 1;
      } else if (!(xd >= qv[0]) || !(xd <= qv[m - 1])) {
        bad = 1;
      } else {
        int lo = 0, hi = m - 2;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (qv[mid] <= xd)
            lo = mid;
          else
            hi = mid - 1;
        }
        const double y = __dsub_rn(xd, qv[lo]);
        const double w = __dsub_rn(qv[lo + 1], qv[lo]);
        const double u = __dmul_rn(static_cast<double>(rw[e]), 0x1p-32);
        out = lo + ((__dmul_rn(u, w) < y) ? 1 : 0);
      }
      o[j + e] = static_cast<uint8_t>(out);
      red_shared_inc(wh_base + 4u * static_cast<uint32_t>(part * s + out));
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

// SM count of the current device, read once per device.
cudaError_t device_sms(int* sms) {
  static std::once_flag once[64];
  static int count[64];
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev]() {
    if (cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) count[dev] = 0;
  });
  *sms = count[dev] > 0 ? count[dev] : 1;
  return cudaSuccess;
}

size_t encode_smem(int p, int s) {
  return sizeof(double2) * 2 * p + sizeof(double) * (p + 2 * s) + sizeof(unsigned int) * kEncWarps * (2 * s + 1) +
         sizeof(float) * p + sizeof(int32_t) * 2 * s + 2 * p;
}

}  // namespace

// ---- reconstruction X^ from the indices ---------------------------------------
// X^[r][j] = P[r][Q_part[idx[r][j]]] rounded to float32, the part of entry j
// drawn as k_encode draws it (§1 "O Problema ECASQ": the emitted value whose
// expectation is the entry; §2.1: time-sharing). One CTA per (row, chunk of
// kDeqChunk entries); the codes' values sit in shared memory as float32; a
// thread handles 16 entries at a time on 16-byte aligned rows, else four (one
// Philox block of the part stream per four entries when the row mixes codes).
namespace {
template <bool kFixed>
__global__ void __launch_bounds__(kEncThreads) k_dequantize(const uint8_t* __restrict__ idx,
                                                           const double* __restrict__ Pall, int64_t d, int p, int s,
                                                           const int32_t* __restrict__ Q1,
                                                           const int32_t* __restrict__ Q1_len,
                                                           const int32_t* __restrict__ Q2,
                                                           const int32_t* __restrict__ Q2_len,
                                                           const double* __restrict__ theta,
                                                           const Philox4x32::RoundKeys K, float* __restrict__ out,
                                                           int32_t* __restrict__ status, int64_t chunk_arg) {
  const int64_t chunk = kFixed ? kDeqChunk : chunk_arg;  // entries of this CTA's chunk
  __shared__ float qv[2][256];
  __shared__ int s_m[2];
  __shared__ int s_bad;
  const int r = blockIdx.y;
  const bool has2 = (Q2 != nullptr);
  const double th = (has2 && theta) ? theta[r] : 0.0;
  const bool mix = has2 && th > 0.0 && th < 1.0;
  const int fixed_part = (!has2 || th >= 1.0) ? 0 : 1;
  if (threadIdx.x == 0) {
    s_m[0] = Q1_len[r];
    s_m[1] = has2 ? Q2_len[r] : 0;
    s_bad = 0;
  }
  __syncthreads();
  int bad = 0;
  for (int k = threadIdx.x; k < 2 * 256; k += blockDim.x) {
    const int part = k >> 8, t = k & 255;
    const int32_t* Q = part == 0 ? Q1 : Q2;
    float v = __int_as_float(0x7fc00000);  // no value: an index here is an error
    if (Q && t < s && t < s_m[part]) {
      const int32_t q = Q[static_cast<int64_t>(r) * s + t];
      if (q >= 0 && q < p)
        v = static_cast<float>(Pall[static_cast<int64_t>(r) * p + q]);
      else
        bad = 1;
    }
    qv[part][t] = v;
  }
  if (bad) s_bad = 1;
  __syncthreads();
  const int m0 = s_m[0], m1 = s_m[1];
  // u < theta with u = word * 2^-32 is word <= ceil(theta * 2^32) - 1
  const uint32_t th_last = mix ? static_cast<uint32_t>(static_cast<uint64_t>(ceil(th * 0x1p32)) - 1u) : 0u;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int len = static_cast<int>((beg + chunk < d ? beg + chunk : d) - beg);
  const uint8_t* ix = idx + static_cast<int64_t>(r) * d + beg;
  float* o = out + static_cast<int64_t>(r) * d + beg;
  const uint32_t blk0 = static_cast<uint32_t>(static_cast<uint64_t>(beg) >> 2);
  Philox4x32::RoundKeys rk;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    rk.k0[i] = K.k0[i];
    rk.k1[i] = K.k1[i];
  }
  auto value = [&](uint32_t sel, uint32_t i) {
    const int part = mix ? (sel <= th_last ? 0 : 1) : fixed_part;
    bad |= static_cast<int>(i) >= (part == 0 ? m0 : m1);
    return qv[part][i];
  };
  const bool vec16 = ((reinterpret_cast<uintptr_t>(ix) & 15u) == 0) && ((reinterpret_cast<uintptr_t>(o) & 15u) == 0);
  int j16 = 0;
  if (vec16) {
    // 16 entries per thread and step: one 16-byte index load, four Philox
    // blocks of the part stream (mixed rows), four 16-byte stores
    const int n16 = len >> 4;
    for (int g = threadIdx.x; g < n16; g += blockDim.x) {
      const uint4 b16 = *reinterpret_cast<const uint4*>(ix + 16 * g);
      const uint32_t w32[4] = {b16.x, b16.y, b16.z, b16.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 sel = make_uint4(0u, 0u, 0u, 0u);
        if (mix)
          sel = Philox4x32::block(
              make_uint4(blk0 + static_cast<uint32_t>(4 * g + q), static_cast<uint32_t>(r), 1u, 0u), rk);
        const float4 v = make_float4(value(sel.x, w32[q] & 0xFFu), value(sel.y, (w32[q] >> 8) & 0xFFu),
                                     value(sel.z, (w32[q] >> 16) & 0xFFu), value(sel.w, w32[q] >> 24));
        __stcs(reinterpret_cast<float4*>(o + 16 * g + 4 * q), v);
      }
    }
    j16 = n16 << 4;
  }
  // the rest (rows off 16-byte alignment, the last < 16 entries) four at a
  // time; beg and j16 are multiples of 4, so group g holds the entries of
  // Philox block blk0 + g
  for (int g = (j16 >> 2) + threadIdx.x; 4 * g < len; g += blockDim.x) {
    const int j = 4 * g;
    const int cnt = len - j < 4 ? len - j : 4;
    uint4 sel = make_uint4(0u, 0u, 0u, 0u);
    if (mix) sel = Philox4x32::block(make_uint4(blk0 + static_cast<uint32_t>(g), static_cast<uint32_t>(r), 1u, 0u), rk);
    const uint32_t sv[4] = {sel.x, sel.y, sel.z, sel.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e < cnt) o[j + e] = value(sv[e], ix[j + e]);
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) atomicExch(status + r, kStatusRange);
}
}  // namespace

cudaError_t launch_dequantize(const uint8_t* idx, const double* P, int n, int64_t d, int p, int s,
                              const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2, const int32_t* Q2_len,
                              const double* theta, uint64_t seed, float* Xhat, int32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t) * n, st);
  if (e != cudaSuccess) return e;
  // resident CTAs: the SM count x 8 (256 threads of 32 registers)
  int sms = 1;
  e = device_sms(&sms);
  if (e != cudaSuccess) return e;
  const int64_t chunk = fill_chunk(n, d, static_cast<int64_t>(sms) * kDeqCtasPerSm, kDeqChunk, 16, kEncMinChunk);
  const int nc = static_cast<int>((d + chunk - 1) / chunk);
  const Philox4x32::RoundKeys K =
      Philox4x32::round_keys(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  if (chunk == kDeqChunk)
    k_dequantize<true><<<dim3(nc, n), kEncThreads, 0, st>>>(idx, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, Xhat,
                                                             status, chunk);
  else
    k_dequantize<false><<<dim3(nc, n), kEncThreads, 0, st>>>(idx, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K,
                                                              Xhat, status, chunk);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* X, const double* P, int n, int64_t d, int p, int s,
                          const int32_t* Q1, const int32_t* Q1_len, const int32_t* Q2,
                          const int32_t* Q2_len, const double* theta, uint64_t seed, uint8_t* idx,
                          int64_t* hist, int32_t* status, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(int64_t) * 2 * s * static_cast<size_t>(n), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(status, 0, sizeof(int32_t) * n, st);
  if (e != cudaSuccess) return e;
  const size_t smem = encode_smem(p, s);
  const size_t sm2 = sizeof(double) * 2 * s + sizeof(unsigned int) * kEncWarps * 2 * s;
  const Philox4x32::RoundKeys K =
      Philox4x32::round_keys(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  // resident CTAs: the SM count x the 5 CTAs per SM that k_encode's launch
  // bounds ask for
  int sms = 1;
  e = device_sms(&sms);
  if (e != cudaSuccess) return e;
  const int64_t chunk = fill_chunk(n, d, static_cast<int64_t>(sms) * kEncCtasPerSm, kEncChunk, 4, kEncMinChunk);
  const int nc = static_cast<int>((d + chunk - 1) / chunk);
  if (p > kMaxP) {
    k_encode_code<<<dim3(nc, n), kEncThreads, sm2, st>>>(X, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx,
                                                         reinterpret_cast<unsigned long long*>(hist), status, chunk);
  } else if (chunk == kEncChunk) {
    k_encode<<<dim3(nc, n), kEncThreads, smem, st>>>(X, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K, idx,
                                                      reinterpret_cast<unsigned long long*>(hist), status);
  } else {
    k_encode_chunked<<<dim3(nc, n), kEncThreads, smem, st>>>(X, P, d, p, s, Q1, Q1_len, Q2, Q2_len, theta, K,
                                                              idx, reinterpret_cast<unsigned long long*>(hist),
                                                              status, chunk);
  }
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
