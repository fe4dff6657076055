// Row statistics, uniform grid and bucketing of X onto the permissible set P.
//
// ECASQ summary (gist.science/pt/paper/2608.18147) §2.2 "Generalização": for an
// arbitrary permissible set P the solver costs O(p^2 s + d); the O(d) part is
// one pass that buckets every entry onto P and accumulates per-bucket
// statistics, from which every interval table is built without touching X
// again. Both kernels here are HBM-bound streams over X (4 bytes per entry).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {

// ---------------------------------------------------------------------------
// Row min / max / finiteness, one chunk of one row per CTA.
// partial layout per (row, chunk): float lo, float hi, int bad (3 x 32-bit).

namespace {

constexpr int kGridThreads = 256;

__device__ __forceinline__ void mm_update(float v, float& lo, float& hi, int& bad) {
  if (!isfinite(v)) bad = 1;
  lo = fminf(lo, v);
  hi = fmaxf(hi, v);
}

__global__ void __launch_bounds__(kGridThreads)
k_minmax_partial(const float* __restrict__ X, int64_t d, int64_t chunk, int n_chunks,
                 float* __restrict__ part) {
  const int r = blockIdx.y;
  const int c = blockIdx.x;
  const float* x = X + static_cast<int64_t>(r) * d;
  const int64_t beg = static_cast<int64_t>(c) * chunk;
  const int64_t end = beg + chunk < d ? beg + chunk : d;
  float lo = INFINITY, hi = -INFINITY;
  int bad = 0;
  // Vector loads when the chunk start is 16-byte aligned.
  const bool vec = ((reinterpret_cast<uintptr_t>(x + beg) & 15u) == 0);
  int64_t t = beg;
  if (vec) {
    const int64_t nv = (end - beg) >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(x + beg);
    for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
      const float4 v = __ldcs(x4 + i);
      mm_update(v.x, lo, hi, bad);
      mm_update(v.y, lo, hi, bad);
      mm_update(v.z, lo, hi, bad);
      mm_update(v.w, lo, hi, bad);
    }
    t = beg + (nv << 2);
  }
  for (int64_t i = t + threadIdx.x; i < end; i += blockDim.x) mm_update(__ldcs(x + i), lo, hi, bad);

  __shared__ float s_lo[kGridThreads / kWarp], s_hi[kGridThreads / kWarp];
  __shared__ int s_bad[kGridThreads / kWarp];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (lane_id() == 0) {
    s_lo[warp_id()] = lo;
    s_hi[warp_id()] = hi;
    s_bad[warp_id()] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kGridThreads / kWarp; ++w) {
      lo = fminf(lo, s_lo[w]);
      hi = fmaxf(hi, s_hi[w]);
      bad |= s_bad[w];
    }
    float* o = part + (static_cast<int64_t>(r) * n_chunks + c) * 3;
    o[0] = lo;
    o[1] = hi;
    o[2] = __int_as_float(bad);
  }
}

// P_k = lo + (hi - lo) * k / (p - 1) in IEEE fp64 with round-to-nearest and no
// contraction; P_{p-1} = hi.
__global__ void k_grid_finish(const float* __restrict__ part, int n_chunks, int p,
                              double* __restrict__ P, int32_t* __restrict__ status) {
  const int r = blockIdx.x;
  __shared__ float s_lo, s_hi;
  __shared__ int s_bad;
  if (threadIdx.x == 0) {
    float lo = INFINITY, hi = -INFINITY;
    int bad = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const float* o = part + (static_cast<int64_t>(r) * n_chunks + c) * 3;
      lo = fminf(lo, o[0]);
      hi = fmaxf(hi, o[1]);
      bad |= __float_as_int(o[2]);
    }
    s_lo = lo;
    s_hi = hi;
    s_bad = bad;
    if (status) status[r] = bad ? kStatusRange : kStatusOk;
  }
  __syncthreads();
  const double lo = s_lo, hi = s_hi;
  const double span = __dsub_rn(hi, lo);
  const double den = static_cast<double>(p - 1);
  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    double v;
    if (k == p - 1)
      v = hi;
    else
      v = __dadd_rn(lo, __ddiv_rn(__dmul_rn(span, static_cast<double>(k)), den));
    P[static_cast<int64_t>(r) * p + k] = s_bad ? __longlong_as_double(0x7ff8000000000000ll) : v;
  }
}

// Hardware-aware permissible set ("Entropy-Constrained Adaptive Stochastic
// Quantization (ECASQ)", §5 "Generalidade": any permissible alphabet, e.g. the
// values BF16 can represent): every finite BF16 value from the largest one
// <= min X to the smallest one >= max X, ascending, +0 and -0 once.
// A BF16 pattern b is the top half of an fp32. Ordered by value, the finite
// patterns map to 16-bit keys: b | 0x8000 for a clear sign bit, ~b for a set
// one (-0 -> 0x7FFF, +0 -> 0x8000), so the set is a key range less -0 when +0
// is in it.
__device__ __forceinline__ unsigned bf16_key(unsigned b) { return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u); }
__device__ __forceinline__ unsigned bf16_of_key(unsigned k) { return (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu); }
// Largest BF16 pattern with value <= x, and smallest with value >= x.
__device__ __forceinline__ unsigned bf16_down(float x) {
  const unsigned u = __float_as_uint(x), b = u >> 16;
  return ((u & 0xFFFFu) == 0u || !(u & 0x80000000u)) ? b : b + 1u;
}
__device__ __forceinline__ unsigned bf16_up(float x) {
  const unsigned u = __float_as_uint(x), b = u >> 16;
  return ((u & 0xFFFFu) == 0u || (u & 0x80000000u)) ? b : b + 1u;
}
__device__ __forceinline__ bool bf16_finite(unsigned b) { return (b & 0x7F80u) != 0x7F80u; }

__global__ void k_bf16_finish(const float* __restrict__ part, int n_chunks, int p_max, double* __restrict__ P,
                              int32_t* __restrict__ p_len, int32_t* __restrict__ status) {
  const int r = blockIdx.x;
  __shared__ unsigned s_klo, s_khi;
  __shared__ int s_cnt;
  if (threadIdx.x == 0) {
    float lo = INFINITY, hi = -INFINITY;
    int bad = 0;
    for (int c = 0; c < n_chunks; ++c) {
      const float* o = part + (static_cast<int64_t>(r) * n_chunks + c) * 3;
      lo = fminf(lo, o[0]);
      hi = fmaxf(hi, o[1]);
      bad |= __float_as_int(o[2]);
    }
    int st = kStatusOk, cnt = 0;
    unsigned klo = 0, khi = 0;
    const unsigned blo = bf16_down(lo), bhi = bf16_up(hi);
    if (bad || !bf16_finite(blo) || !bf16_finite(bhi)) {
      st = kStatusRange;
    } else {
      klo = bf16_key(blo);
      khi = bf16_key(bhi);
      cnt = static_cast<int>(khi - klo) + 1 - ((klo <= 0x7FFFu && khi >= 0x8000u) ? 1 : 0);
      if (cnt > p_max) st = kStatusArg;
    }
    s_klo = klo;
    s_khi = khi;
    s_cnt = st == kStatusRange ? 0 : cnt;
    p_len[r] = s_cnt;
    if (status) status[r] = st;
  }
  __syncthreads();
  const unsigned klo = s_klo, khi = s_khi;
  const bool skip_neg0 = klo <= 0x7FFFu && khi >= 0x8000u;
  const int cnt = s_cnt;
  for (int t = threadIdx.x; t < p_max; t += blockDim.x) {
    double v = __longlong_as_double(0x7ff8000000000000ll);
    if (t < cnt) {
      unsigned k = klo + static_cast<unsigned>(t);
      if (skip_neg0 && k >= 0x7FFFu) k += 1u;
      v = static_cast<double>(__uint_as_float(bf16_of_key(k) << 16));
    }
    P[static_cast<int64_t>(r) * p_max + t] = v;
  }
}

// ---------------------------------------------------------------------------
// Bucketing: constants and the per-CTA state shared by the kernels below.

constexpr int kBucketThreads = 256;
constexpr int kBucketSub = 8192;          // entries between two folds of the shared counters
constexpr int kBucketSubsPerCta = 8;      // 65536 entries per CTA
constexpr int kBucketOwn = 2;             // buckets owned per thread (p - 1 <= 511)
constexpr int kBucketCtasPerSm = 3;       // resident k_bucket CTAs per SM
constexpr int kHotW = 48;                 // buckets with one counter per lane
constexpr int kLimbBlock = kHotW * kWarp + kMaxP;  // words per limb: [kHotW][32] lane counters, then [kMaxP]
constexpr int kLimbBits = 18;
constexpr double kFastEps = 0x1p-20;      // distance of v from a grid point on the fast path
// The fast path evaluates G = (x - P_0)/D as fma(x, 1/D, -P_0/D); the rounding
// of -P_0/D and of 1/D then move G by at most (2|P_0/D| + p) 2^-53, below 2^-37
// bucket widths for |P_0/D| <= 2^15 (rows straddling zero have |P_0/D| <= p). Rows beyond
// that take the exact search for every entry.
constexpr double kFmaOffsetMax = 0x1p15;

// k = floor(G) and v = G - k for 0 <= G < 2^31 away from the integers, with
// fp64 additions instead of conversions: (G - 0.5) is exact, and adding
// 1.5 * 2^52 rounds it to the nearest integer, which is floor(G) unless G is an
// integer (then v = 0 or 1 and the caller's fast-path test fails); the integer
// sits in the low word. Outside that range k and v are meaningless and the
// test fails as well (k out of [0, p-2], or v not finite).
__device__ __forceinline__ void floor_split(double G, int& k, double& v) {
  const double t = __dadd_rn(__dadd_rn(G, -0.5), 0x1.8p52);
  k = __double2loint(t);
  v = __dsub_rn(G, __dsub_rn(t, 0x1.8p52));
}

// Per-CTA state of the bucketing kernel in shared memory.
struct BucketRow {
  const double* P;   // [p]
  const double* E;   // [p] eta_k (uniform rows) or 1/D_k (other rows)
  const float* T;    // [p] smallest float >= P_k
  unsigned int* cnt;   // [kMaxP] counts
  unsigned int* limb;  // [4][kLimbBlock]
  double invD, twoF, twoH;
  float top, scale;
  int p, hot0, uni, bad;
};

// Fixed point: a = v 2^(F+14) + 2^52 + 2^13 keeps round(v 2^F) in bits 14.. of
// the integer part, so the low limb is the low word >> 14 and the high limb the
// low bits of the high word.
// cnt_base, limb_base: shared-window byte addresses of the counts and limbs.
__device__ __forceinline__ void bucket_add(uint32_t cnt_base, uint32_t limb_base, int k, double v, int hot0,
                                           int lane, double twoF, double twoH) {
  const double magic = 0x1p52 + 0x1p13;
  red_shared_inc(cnt_base + 4u * static_cast<uint32_t>(k));
  const double a = fma(v, twoF, magic);
  const double t = v * twoH;
  const double b = fma(t, t, magic);
  const int hk = k - hot0;
  const int off = (static_cast<unsigned>(hk) < static_cast<unsigned>(kHotW)) ? hk * kWarp + lane : kHotW * kWarp + k;
  const uint32_t c = limb_base + 4u * static_cast<uint32_t>(off);
  constexpr int kL = 4 * kLimbBlock;  // bytes between limbs
  red_shared_add<0>(c, static_cast<unsigned>(__double2loint(a)) >> 14);
  red_shared_add<kL>(c, static_cast<unsigned>(__double2hiint(a)) & 0x7FFFFu);
  red_shared_add<2 * kL>(c, static_cast<unsigned>(__double2loint(b)) >> 14);
  red_shared_add<3 * kL>(c, static_cast<unsigned>(__double2hiint(b)) & 0x7FFFFu);
}

// Exact bucket k = max{k <= p-2 : P_k <= x} (fp32-threshold search) and offset
// v of up to four entries, then their counters; entries outside
// [P_0, P_{p-1}] or NaN set the bad flag. Uniform rows: v = clamp((x - P_k)/D
// + eta_k, 0, 1); other rows: v = min((x - P_k)/D_k, 1). Kept out of line: on
// uniform rows it runs only for groups holding an entry within 2^-20 bucket
// widths of a grid point.
// One instance per kernel (kTag): a callee shared by two kernels gets a calling
// convention fitted to neither.
template <int kTag>
__device__ __noinline__ void bucket_exact(BucketRow* S, const float* xv, int cnt) {
  const int lane = lane_id();
  for (int e = 0; e < cnt; ++e) {
    const float xf = xv[e];
    const int k = bucket_f32(xf, S->T, S->top, S->p, S->scale);
    if (k < 0) {
      S->bad = 1;
      continue;
    }
    const double y = __dsub_rn(static_cast<double>(xf), S->P[k]);
    const double w = S->uni ? __dadd_rn(__dmul_rn(y, S->invD), S->E[k]) : __dmul_rn(y, S->E[k]);
    bucket_add(smem_addr(S->cnt), smem_addr(S->limb), k, fmin(fmax(w, 0.0), 1.0), S->hot0, lane, S->twoF,
               S->twoH);
  }
}

// Bucketing (the "+d" pass of §2.2 "Generalização"). An entry x of bucket k
// (P_k <= x < P_{k+1}; the last bucket closed) contributes a normalised offset
// v in [0, 1], kept as fixed point: round(v 2^F) and round(v^2 2^F) with F = 36
// fraction bits (32 for rows of 2^27 entries or more, so that the 64-bit row
// sums cannot overflow). Integer sums make the result independent of the order
// of addition. The finish kernel turns them back into A_k = sum (x - P_k) and
// B_k = sum (x - P_k)^2.
//
// Two ways to find k and v:
//  * uniform rows: P_k = P_0 + (k + eta_k) D with D = (P_{p-1} - P_0)/(p-1)
//    and |eta_k| <= 2^-36 for every k (an fp64 uniform grid qualifies unless
//    |P_0| is very large against the span). G = (x - P_0)/D, evaluated in fp64
//    as fma(x, 1/D, -P_0/D), is within 2^-37 bucket widths of its exact value
//    (p <= 512, |P_0/D| <= 2^15), so when
//    v = G - floor(G) lies more than 2^-20 from 0 and from 1, k = floor(G) is
//    the entry's bucket for certain and v = (x - P_k)/D + eta_k up to that
//    error: no shared-memory lookup at all. Groups of four entries holding one
//    within 2^-20 of a grid point take the exact search, with
//    v = clamp((x - P_k)/D + eta_k, 0, 1), the clamp moving v by at most |eta_k|.
//    Then A_k = D (S1 - n_k eta_k) and B_k = D^2 (S2 - 2 eta_k S1 + n_k eta_k^2)
//    with S1 = sum v, S2 = sum v^2.
//  * other rows: k by the exact search on P, v = (x - P_k)/D_k, A_k = D_k S1,
//    B_k = D_k^2 S2.
//
// Accumulation: 32-bit shared-memory counters, added by return-less atomics:
// per entry the count (an increment, which the hardware combines across lanes
// that hit the same counter) and two limbs (bits 0..17 and 18..F) of each
// moment. Additions of different values to one address by lanes of a warp are
// serialised, and real data concentrates in a few buckets, so the limbs of the
// kHotW busiest consecutive buckets (chosen from a sample of the CTA's entries)
// get one counter per lane, laid out [bucket][lane] so that the 32 lanes of a
// warp always fall on 32 distinct banks; the other buckets share one counter
// per bucket. Shared counters are folded into 64-bit registers of the bucket's
// owner thread every 8192 entries (8192 limbs of at most 2^18 stay below 2^32);
// a lane counter receives at most 2048 entries per CTA and is summed once at
// the end. Each CTA adds its totals to the row's 64-bit sums in global memory.
// kFixed: chunks of kBucketSub * kBucketSubsPerCta entries; else `chunk_arg`
// entries (a multiple of 4, smaller), for grids of few or short rows.
template <bool kFixed>
__global__ void __launch_bounds__(kBucketThreads, kBucketCtasPerSm)
k_bucket(const float* __restrict__ X, int64_t d, const double* __restrict__ Pall, int p, int fb,
         unsigned long long* __restrict__ acc, int32_t* __restrict__ flag, int64_t chunk_arg) {
  __shared__ unsigned int sc[kMaxP];                 // counts (every bucket)
  __shared__ unsigned int sl[4 * kLimbBlock];       // limbs: [4][kLimbBlock]
  __shared__ unsigned int spre[kMaxP + 1];           // sample counts, then their prefix sums
  __shared__ BucketRow S;
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = blockIdx.y;
  const int nb = p - 1;
  double* sP = reinterpret_cast<double*>(smem);      // [p] P
  double* sE = sP + p;                               // [p] eta_k (uniform rows) or 1/D_k (other rows)
  float* sT = reinterpret_cast<float*>(sE + p);      // [p] smallest float >= P_k

  const double* P = Pall + static_cast<int64_t>(r) * p;
  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    sP[k] = P[k];
    sT[k] = __double2float_ru(P[k]);
  }
  for (int k = threadIdx.x; k < kMaxP; k += blockDim.x) sc[k] = 0u;
  for (int k = threadIdx.x; k <= kMaxP; k += blockDim.x) spre[k] = 0u;
  for (int k = threadIdx.x; k < 4 * kLimbBlock; k += blockDim.x) sl[k] = 0u;
  __syncthreads();
  const RowGrid g = row_grid(sP, p);
  const bool uni = row_is_uniform(sP, p, g, sE);  // includes a barrier
  if (!uni) {
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
      const double w = __dsub_rn(sP[k + 1], sP[k]);
      sE[k] = w > 0.0 ? __ddiv_rn(1.0, w) : 0.0;
    }
  }
  const double twoF = ldexp(1.0, fb + 14), twoH = ldexp(1.0, (fb + 14) / 2);
  if (threadIdx.x == 0) {
    S.P = sP;
    S.E = sE;
    S.T = sT;
    S.cnt = sc;
    S.limb = sl;
    S.invD = g.invD;
    S.twoF = twoF;
    S.twoH = twoH;
    S.top = __double2float_rd(sP[p - 1]);
    S.scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
    S.p = p;
    S.hot0 = 0;
    S.uni = uni;
    S.bad = 0;
  }
  __syncthreads();
  const int lane = lane_id();
  const unsigned pm2 = static_cast<unsigned>(p - 2);
  const double lim = 0.5 - kFastEps;
  const double c0 = -(g.P0 * g.invD);
  const bool fastg = uni && fabs(c0) <= kFmaOffsetMax;

  const float* x = X + static_cast<int64_t>(r) * d;
  const int64_t chunk = kFixed ? static_cast<int64_t>(kBucketSub) * kBucketSubsPerCta : chunk_arg;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int len = static_cast<int>((beg + chunk < d ? beg + chunk : d) - beg);
  const float* xc = x + beg;

  // Hot window: bucket counts of a sample of blockDim entries spread over the
  // chunk, then the kHotW consecutive buckets with the most sampled entries.
  {
    const int i = threadIdx.x * (len > kBucketThreads ? len / kBucketThreads : 1);
    if (i < len) {
      const float xf = __ldg(xc + i);
      int k = -1;
      if (uni) {
        const double G = __dmul_rn(__dsub_rn(static_cast<double>(xf), g.P0), g.invD);
        const double kf = floor(G);
        if (kf >= 0.0 && kf <= static_cast<double>(p - 2)) k = static_cast<int>(kf);
      } else {
        k = bucket_f32(xf, sT, S.top, p, S.scale);
      }
      if (k >= 0) atomicAdd(spre + k, 1u);
    }
    __syncthreads();
    if (warp_id() == 0) {
      unsigned run = 0;
      for (int j = 0; j < 16; ++j) run += spre[lane * 16 + j];
      unsigned excl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, excl, o);
        if (lane >= o) excl += t;
      }
      excl -= run;
      unsigned cnts[16];
      for (int j = 0; j < 16; ++j) cnts[j] = spre[lane * 16 + j];
      __syncwarp();
      for (int j = 0; j < 16; ++j) {
        spre[lane * 16 + j] = excl;  // exclusive prefix; spre[kMaxP] = total
        excl += cnts[j];
      }
      if (lane == 31) spre[kMaxP] = excl;
      __syncwarp();
      const int last = nb > kHotW ? nb - kHotW : 0;
      unsigned best = 0;
      int bs = 0x7fffffff;
      for (int s0 = lane; s0 <= last; s0 += kWarp) {
        const unsigned sum = spre[s0 + kHotW < kMaxP ? s0 + kHotW : kMaxP] - spre[s0];
        if (bs == 0x7fffffff || sum > best) {
          best = sum;
          bs = s0;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int os = __shfl_xor_sync(0xffffffffu, bs, o);
        if (os != 0x7fffffff && (bs == 0x7fffffff || ob > best || (ob == best && os < bs))) {
          best = ob;
          bs = os;
        }
      }
      if (lane == 0) S.hot0 = bs == 0x7fffffff ? 0 : bs;
    }
    __syncthreads();
  }
  const int hot0 = S.hot0;
  const uint32_t sc_base = smem_addr(sc), sl_base = smem_addr(sl);

  // Main pass: the float4 groups from the first 16-byte boundary, kB per
  // thread per step with the next kB loads in flight, the counters folded every
  // kBucketSub entries; then the head and tail entries.
  const int head = (reinterpret_cast<uintptr_t>(x) & 3u) ? len
                   : static_cast<int>(((16u - (reinterpret_cast<uintptr_t>(xc) & 15u)) & 15u) >> 2);
  const int h = head < len ? head : len;
  const int nv = (len - h) >> 2;
  const float4* x4 = reinterpret_cast<const float4*>(xc + h);
  constexpr int kB = 2;
  constexpr int kStepsPerFold = kBucketSub / (4 * kBucketThreads * kB);  // steps between two folds
  const int steps = (nv + kBucketThreads * kB - 1) / (kBucketThreads * kB);
  unsigned long long tc[kBucketOwn] = {}, ta[kBucketOwn] = {}, tb[kBucketOwn] = {};
  auto fold = [&]() {
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kBucketOwn; ++j) {
      const int k = threadIdx.x + j * kBucketThreads;
      if (k < nb) {
        const int o = kHotW * kWarp + k;
        tc[j] += sc[k];
        ta[j] += static_cast<unsigned long long>(sl[o]) +
                 (static_cast<unsigned long long>(sl[kLimbBlock + o]) << kLimbBits);
        tb[j] += static_cast<unsigned long long>(sl[2 * kLimbBlock + o]) +
                 (static_cast<unsigned long long>(sl[3 * kLimbBlock + o]) << kLimbBits);
        sc[k] = sl[o] = sl[kLimbBlock + o] = sl[2 * kLimbBlock + o] = sl[3 * kLimbBlock + o] = 0u;
      }
    }
    __syncthreads();
  };
  float4 nxt[kB];
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int i = threadIdx.x + u * kBucketThreads;
    nxt[u] = (i < nv) ? __ldcs(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int st = 0; st < steps; ++st) {
    float4 cur[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      cur[u] = nxt[u];
      const int i = threadIdx.x + ((st + 1) * kB + u) * kBucketThreads;
      nxt[u] = (i < nv) ? __ldcs(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int i = threadIdx.x + (st * kB + u) * kBucketThreads;
      if (i < nv) {
        const float xv[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
        int k[4];
        double v[4];
        bool all = fastg;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double G = fma(static_cast<double>(xv[e]), g.invD, c0);
          floor_split(G, k[e], v[e]);
          all = all && fabs(v[e] - 0.5) < lim && static_cast<unsigned>(k[e]) <= pm2;
        }
        if (all) {
#pragma unroll
          for (int e = 0; e < 4; ++e) bucket_add(sc_base, sl_base, k[e], v[e], hot0, lane, twoF, twoH);
        } else {
          bucket_exact<kFixed ? 0 : 1>(&S, xv, 4);
        }
      }
    }
    if ((st + 1) % kStepsPerFold == 0) fold();
  }
  // head and tail entries (fewer than 4 + 4), one per thread
  {
    const int tail0 = h + 4 * nv;
    if (threadIdx.x < h || (threadIdx.x >= 4 && threadIdx.x - 4 + tail0 < len)) {
      const int i = threadIdx.x < h ? threadIdx.x : tail0 + threadIdx.x - 4;
      const float xv[1] = {__ldcs(xc + i)};
      bucket_exact<kFixed ? 0 : 1>(&S, xv, 1);
    }
  }
  fold();
  unsigned long long* gacc = acc + static_cast<int64_t>(r) * nb * 3;
#pragma unroll
  for (int j = 0; j < kBucketOwn; ++j) {
    const int k = threadIdx.x + j * kBucketThreads;
    if (k < nb) {
      if (tc[j]) atomicAdd(gacc + 3 * k + 0, tc[j]);
      if (ta[j]) atomicAdd(gacc + 3 * k + 1, ta[j]);
      if (tb[j]) atomicAdd(gacc + 3 * k + 2, tb[j]);
    }
  }
  // lane counters of the hot buckets: one (limb, bucket) sum over the lanes per thread
  for (int q = threadIdx.x; q < 4 * kHotW; q += blockDim.x) {
    const int li = q / kHotW, j = q - li * kHotW, k = hot0 + j;
    if (k >= nb) continue;
    const unsigned int* c = sl + li * kLimbBlock + j * kWarp;
    unsigned long long sum = 0;
#pragma unroll 8
    for (int l = 0; l < kWarp; ++l) sum += c[(l + lane) & (kWarp - 1)];
    if (sum) atomicAdd(gacc + 3 * k + 1 + (li >> 1), sum << ((li & 1) ? kLimbBits : 0));
  }
  if (threadIdx.x == 0 && S.bad) atomicOr(flag + r, 1);
}

// ---------------------------------------------------------------------------
// Bucketing of long rows with small alphabets (p <= 257, d >= 2^16): the same
// fixed point, fast path and exact fallback as k_bucket, with every bucket's
// limbs in per-lane counters (4 limbs x 256 buckets x 32 lanes x 4 bytes = 128
// KB of shared memory, one bank per lane), so a limb atomic never serialises
// and its address is k * 32 + lane. One persistent CTA of 1024 threads per SM
// walks a contiguous range of (row, 64K-entry chunk) pairs. Lane counters
// receive at most 32 * 256 entries per 256K entries of the CTA; every 256K
// entries, and when the row changes, each thread folds one (limb, bucket) row
// of 32 lane counters into a 64-bit register, and at a row change the CTA
// adds its totals to the row's sums in global memory.

constexpr int kWideThreads = 1024;
constexpr int kWideChunk = 65536;           // entries per (row, chunk) work item
constexpr int kWideChunksPerFold = 4;       // 2^18 entries between two folds
constexpr int kWideBuckets = 256;           // p - 1 <= 256
constexpr int kWideLimbBlock = kWideBuckets * kWarp;
constexpr size_t kWideSmem = sizeof(unsigned int) * (4 * kWideLimbBlock + kWideBuckets) +
                             (sizeof(double) * 2 + sizeof(float)) * (kWideBuckets + 1);

struct WideRow {
  const double* P;
  const double* E;
  const float* T;
  unsigned int* cnt;
  unsigned int* limb;
  double invD, twoF, twoH;
  float top, scale;
  int p, uni, bad;
};

// cnt_base, lane_base: shared-window byte addresses of the counts and of this
// lane's column of limb counters ([4][buckets][32], kLB words per limb).
template <int kLB = kWideLimbBlock>
__device__ __forceinline__ void wide_add(uint32_t cnt_base, uint32_t lane_base, int k, double v, double twoF,
                                         double twoH) {
  const double magic = 0x1p52 + 0x1p13;
  red_shared_inc(cnt_base + 4u * static_cast<uint32_t>(k));
  const double a = fma(v, twoF, magic);
  const double t = v * twoH;
  const double b = fma(t, t, magic);
  const uint32_t c = lane_base + static_cast<uint32_t>(k) * (4u * kWarp);
  constexpr int kL = 4 * kLB;  // bytes between limbs
  red_shared_add<0>(c, static_cast<unsigned>(__double2loint(a)) >> 14);
  red_shared_add<kL>(c, static_cast<unsigned>(__double2hiint(a)) & 0x7FFFFu);
  red_shared_add<2 * kL>(c, static_cast<unsigned>(__double2loint(b)) >> 14);
  red_shared_add<3 * kL>(c, static_cast<unsigned>(__double2hiint(b)) & 0x7FFFFu);
}

template <int kLB = kWideLimbBlock>
__device__ __noinline__ void wide_exact(WideRow* S, const float* xv, int cnt) {
  const uint32_t lane_base = smem_addr(S->limb + lane_id()), cnt_base = smem_addr(S->cnt);
  for (int e = 0; e < cnt; ++e) {
    const float xf = xv[e];
    const int k = bucket_f32(xf, S->T, S->top, S->p, S->scale);
    if (k < 0) {
      S->bad = 1;
      continue;
    }
    const double y = __dsub_rn(static_cast<double>(xf), S->P[k]);
    const double w = S->uni ? __dadd_rn(__dmul_rn(y, S->invD), S->E[k]) : __dmul_rn(y, S->E[k]);
    wide_add<kLB>(cnt_base, lane_base, k, fmin(fmax(w, 0.0), 1.0), S->twoF, S->twoH);
  }
}

__global__ void __launch_bounds__(kWideThreads, 1)
k_bucket_wide(const float* __restrict__ X, int n, int64_t d, const double* __restrict__ Pall, int p, int fb,
              unsigned long long* __restrict__ acc, int32_t* __restrict__ flag) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ WideRow S;
  unsigned int* sl = reinterpret_cast<unsigned int*>(smem);          // [4][256][32] lane counters
  unsigned int* sc = sl + 4 * kWideLimbBlock;                        // [256] counts
  double* sP = reinterpret_cast<double*>(sc + kWideBuckets);         // [p]
  double* sE = sP + (kWideBuckets + 1);                              // [p]
  float* sT = reinterpret_cast<float*>(sE + (kWideBuckets + 1));     // [p]
  const int nb = p - 1;
  const int lane = lane_id();
  const int tid = threadIdx.x;
  const double twoF = ldexp(1.0, fb + 14), twoH = ldexp(1.0, (fb + 14) / 2);
  const unsigned pm2 = static_cast<unsigned>(p - 2);
  const double lim = 0.5 - kFastEps;
  // the (limb, bucket) row of 32 lane counters this thread folds
  const int fl = tid / kWideBuckets, fk = tid % kWideBuckets;
  unsigned long long facc = 0, fcnt = 0;

  for (int k = tid; k < 4 * kWideLimbBlock; k += kWideThreads) sl[k] = 0u;
  for (int k = tid; k < kWideBuckets; k += kWideThreads) sc[k] = 0u;

  const int64_t cpr = (d + kWideChunk - 1) / kWideChunk;  // chunks per row
  const int64_t Q = static_cast<int64_t>(n) * cpr;
  const int64_t q0 = Q * blockIdx.x / gridDim.x, q1 = Q * (blockIdx.x + 1) / gridDim.x;
  int row = -1;
  RowGrid g{};
  bool uni = false, fastg = false;
  double c0 = 0.0;
  int since_fold = 0;

  // fold the lane counters and counts into registers (all threads)
  auto fold = [&]() {
    __syncthreads();
    uint4* c4 = reinterpret_cast<uint4*>(sl + fl * kWideLimbBlock + fk * kWarp);
    unsigned long long sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int jj = (j + tid) & 7;  // rotate the 16-byte column: threads of a quarter-warp on distinct banks
      const uint4 v = c4[jj];
      sum += static_cast<unsigned long long>(v.x) + v.y + v.z + v.w;
      c4[jj] = make_uint4(0u, 0u, 0u, 0u);
    }
    facc += sum;
    if (fl == 0) {
      fcnt += sc[fk];
      sc[fk] = 0u;
    }
    __syncthreads();
  };
  // add the folded totals of `row` to its global sums
  auto flush = [&]() {
    if (fk < nb) {
      unsigned long long* gacc = acc + (static_cast<int64_t>(row) * nb + fk) * 3;
      if (facc) atomicAdd(gacc + 1 + (fl >> 1), facc << ((fl & 1) ? kLimbBits : 0));
      if (fl == 0 && fcnt) atomicAdd(gacc, fcnt);
    }
    facc = 0;
    fcnt = 0;
    if (tid == 0 && S.bad) atomicOr(flag + row, 1);
  };

  for (int64_t q = q0; q < q1; ++q) {
    const int r = static_cast<int>(q / cpr);
    const int64_t ci = q - static_cast<int64_t>(r) * cpr;
    if (r != row) {
      if (row >= 0) {
        fold();
        flush();
        since_fold = 0;
      }
      __syncthreads();
      row = r;
      const double* P = Pall + static_cast<int64_t>(r) * p;
      for (int k = tid; k < p; k += kWideThreads) {
        sP[k] = P[k];
        sT[k] = __double2float_ru(P[k]);
      }
      __syncthreads();
      g = row_grid(sP, p);
      uni = row_is_uniform(sP, p, g, sE);  // includes a barrier
      c0 = -(g.P0 * g.invD);
      fastg = uni && fabs(c0) <= kFmaOffsetMax;
      if (!uni) {
        for (int k = tid; k < nb; k += kWideThreads) {
          const double w = __dsub_rn(sP[k + 1], sP[k]);
          sE[k] = w > 0.0 ? __ddiv_rn(1.0, w) : 0.0;
        }
      }
      if (tid == 0) {
        S.P = sP;
        S.E = sE;
        S.T = sT;
        S.cnt = sc;
        S.limb = sl;
        S.invD = g.invD;
        S.twoF = twoF;
        S.twoH = twoH;
        S.top = __double2float_rd(sP[p - 1]);
        S.scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
        S.p = p;
        S.uni = uni;
        S.bad = 0;
      }
      __syncthreads();
    }
    const float* xc = X + static_cast<int64_t>(r) * d + ci * kWideChunk;
    const int len = static_cast<int>((ci + 1) * kWideChunk < d ? kWideChunk : d - ci * kWideChunk);
    const int head = (reinterpret_cast<uintptr_t>(X + static_cast<int64_t>(r) * d) & 3u)
                         ? len
                         : static_cast<int>(((16u - (reinterpret_cast<uintptr_t>(xc) & 15u)) & 15u) >> 2);
    const int h = head < len ? head : len;
    const int nv = (len - h) >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(xc + h);
    const uint32_t lane_base = smem_addr(sl + lane), cnt_base = smem_addr(sc);
    constexpr int kB = 2;
    float4 nxt[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int i = tid + u * kWideThreads;
      nxt[u] = (i < nv) ? __ldcs(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int i0 = 0; i0 < nv; i0 += kB * kWideThreads) {
      float4 cur[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        cur[u] = nxt[u];
        const int i = i0 + tid + (kB + u) * kWideThreads;
        nxt[u] = (i < nv) ? __ldcs(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        if (i0 + tid + u * kWideThreads < nv) {
          const float xv[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
          int k[4];
          double v[4];
          bool all = fastg;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const double G = fma(static_cast<double>(xv[e]), g.invD, c0);
            floor_split(G, k[e], v[e]);
            all = all && fabs(v[e] - 0.5) < lim && static_cast<unsigned>(k[e]) <= pm2;
          }
          if (all) {
#pragma unroll
            for (int e = 0; e < 4; ++e) wide_add(cnt_base, lane_base, k[e], v[e], twoF, twoH);
          } else {
            wide_exact(&S, xv, 4);
          }
        }
      }
    }
    {
      const int tail0 = h + 4 * nv;
      if (tid < h || (tid >= 4 && tid - 4 + tail0 < len)) {
        const int i = tid < h ? tid : tail0 + tid - 4;
        const float xv[1] = {__ldcs(xc + i)};
        wide_exact(&S, xv, 1);
      }
    }
    if (++since_fold == kWideChunksPerFold) {
      fold();
      since_fold = 0;
    }
  }
  if (row >= 0) {
    fold();
    flush();
  }
}

// ---------------------------------------------------------------------------
// Uniform grid and bucketing in one read of X, for rows that fit in shared
// memory (d <= 16384) and alphabets of at most 129 values. One persistent CTA
// walks rows blockIdx.x, blockIdx.x + gridDim.x, ...; each row is staged in
// shared memory by an untiled bulk copy (the next row's copy is issued before
// the current row is processed, into the other of two buffers), then:
//   min / max / finiteness -> the uniform grid, computed exactly as
//   k_grid_finish does (P_k = lo + (hi - lo) k / (p - 1) in IEEE fp64, no
//   contraction, P_{p-1} = hi) and written out; the bucketing of k_bucket_wide
//   from shared memory into per-lane counters (4 limbs x 128 buckets x 32
//   lanes, 64 KB); and the finish of k_bucket_finish for the row's buckets, so
//   that cnt, A, B are written directly (no global atomics, no finish kernel).
// Rows that hold a NaN or an infinity get a NaN grid, zero statistics and
// status ECASQ_ERR_RANGE. A bounded wait for a staging copy that gives up
// marks the row with status kStatusStall and ends the CTA after waiting (also
// bounded) for its other copy in flight.

constexpr int kFuseThreads = 512;
constexpr int kFuseMaxD = 16384;                    // entries of a staged row
constexpr int kFuseBuckets = 128;                   // p - 1 <= 128
constexpr int kFuseLimbBlock = kFuseBuckets * kWarp;
constexpr int kFuseWaitLimit = 1 << 22;

size_t fuse_smem_bytes(int64_t d) {
  const size_t dpad = static_cast<size_t>((d + 3) & ~int64_t(3));
  return 16 + 2 * 4 * dpad + 4 * (4 * kFuseLimbBlock + kFuseBuckets) + 8 * 4 * kFuseBuckets +
         (8 * 2 + 4) * (kFuseBuckets + 1) + 4 * 3 * (kFuseThreads / kWarp);
}

__global__ void __launch_bounds__(kFuseThreads, 2)
k_grid_bucket_rows(const float* __restrict__ X, int n, int64_t d, int p, int fb, double* __restrict__ Pout,
                   int64_t* __restrict__ cnt_out, double* __restrict__ A_out, double* __restrict__ B_out,
                   int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ WideRow S;
  __shared__ float s_lo, s_hi;
  __shared__ int s_bad;
  const int dpad = static_cast<int>((d + 3) & ~int64_t(3));
  unsigned long long* mbar = reinterpret_cast<unsigned long long*>(smem);  // [2]
  float* buf0 = reinterpret_cast<float*>(smem + 16);
  float* buf1 = buf0 + dpad;
  unsigned int* sl = reinterpret_cast<unsigned int*>(buf1 + dpad);         // [4][128][32] lane counters
  unsigned int* sc = sl + 4 * kFuseLimbBlock;                              // [128] counts
  unsigned long long* ssum = reinterpret_cast<unsigned long long*>(sc + kFuseBuckets);  // [4][128] limb sums
  double* sP = reinterpret_cast<double*>(ssum + 4 * kFuseBuckets);         // [129]
  double* sE = sP + (kFuseBuckets + 1);                                     // [129]
  float* sT = reinterpret_cast<float*>(sE + (kFuseBuckets + 1));          // [129]
  float* sred = sT + (kFuseBuckets + 1);                                   // [warps][3]
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int nb = p - 1;
  const double twoF = ldexp(1.0, fb + 14), twoH = ldexp(1.0, (fb + 14) / 2);
  const unsigned pm2 = static_cast<unsigned>(p - 2);
  const double lim = 0.5 - kFastEps;
  // bulk staging needs 16-byte aligned rows of a multiple of 16 bytes
  const bool bulk = ((d & 3) == 0) && ((reinterpret_cast<uintptr_t>(X) & 15u) == 0);
  const uint32_t bytes = static_cast<uint32_t>(d * 4);
  const uint32_t mb0 = smem_addr(mbar), mb1 = smem_addr(mbar + 1);
  const uint32_t bb0 = smem_addr(buf0), bb1 = smem_addr(buf1);

  for (int k = tid; k < 4 * kFuseLimbBlock; k += kFuseThreads) sl[k] = 0u;
  for (int k = tid; k < kFuseBuckets; k += kFuseThreads) sc[k] = 0u;
  if (tid == 0) {
    if (bulk) {
      mbar_init(mb0, 1);
      mbar_init(mb1, 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  if (tid == 0 && bulk && blockIdx.x < n) {
    mbar_expect_tx(mb0, bytes);
    bulk_copy_g2s(bb0, X + static_cast<int64_t>(blockIdx.x) * d, bytes, mb0);
  }

  int it = 0;
  for (int r = blockIdx.x; r < n; r += gridDim.x, ++it) {
    const int b = it & 1;
    const float* xs = b ? buf1 : buf0;
    // the next row's copy into the other buffer (free since the previous
    // iteration's last barrier)
    if (tid == 0 && bulk && r + static_cast<int>(gridDim.x) < n) {
      fence_proxy_async_shared();
      mbar_expect_tx(b ? mb0 : mb1, bytes);
      bulk_copy_g2s(b ? bb0 : bb1, X + static_cast<int64_t>(r + gridDim.x) * d, bytes, b ? mb0 : mb1);
    }
    if (bulk) {
      const bool ok = mbar_wait_bounded(b ? mb1 : mb0, static_cast<uint32_t>((it >> 1) & 1), kFuseWaitLimit);
      if (__syncthreads_or(!ok)) {
        if (tid == 0) {
          status[r] = kStatusStall;
          // the other buffer's copy, if one was issued, before the CTA ends
          if (r + static_cast<int>(gridDim.x) < n)
            mbar_wait_bounded(b ? mb0 : mb1, static_cast<uint32_t>(((it + 1) >> 1) & 1), kFuseWaitLimit);
        }
        return;
      }
    } else {
      float* xw = b ? buf1 : buf0;
      const float* xg = X + static_cast<int64_t>(r) * d;
      for (int i = tid; i < d; i += kFuseThreads) xw[i] = xg[i];
      __syncthreads();
    }

    // min / max / finiteness of the row
    {
      float lo = INFINITY, hi = -INFINITY;
      int bad = 0;
      const int nf = static_cast<int>(d >> 2);
      const float4* x4 = reinterpret_cast<const float4*>(xs);
      for (int i = tid; i < nf; i += kFuseThreads) {
        const float4 v = x4[i];
        mm_update(v.x, lo, hi, bad);
        mm_update(v.y, lo, hi, bad);
        mm_update(v.z, lo, hi, bad);
        mm_update(v.w, lo, hi, bad);
      }
      for (int i = 4 * nf + tid; i < d; i += kFuseThreads) mm_update(xs[i], lo, hi, bad);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        bad |= __shfl_xor_sync(0xffffffffu, bad, o);
      }
      if (lane == 0) {
        sred[3 * warp] = lo;
        sred[3 * warp + 1] = hi;
        sred[3 * warp + 2] = __int_as_float(bad);
      }
      __syncthreads();
      if (tid == 0) {
        for (int w = 1; w < kFuseThreads / kWarp; ++w) {
          lo = fminf(lo, sred[3 * w]);
          hi = fmaxf(hi, sred[3 * w + 1]);
          bad |= __float_as_int(sred[3 * w + 2]);
        }
        s_lo = lo;
        s_hi = hi;
        s_bad = bad;
      }
      __syncthreads();
    }
    const bool row_bad = s_bad != 0;
    {
      // the uniform grid, as k_grid_finish computes it
      const double lo = s_lo, hi = s_hi;
      const double span = __dsub_rn(hi, lo);
      const double den = static_cast<double>(p - 1);
      for (int k = tid; k < p; k += kFuseThreads) {
        const double v = (k == p - 1) ? hi : __dadd_rn(lo, __ddiv_rn(__dmul_rn(span, static_cast<double>(k)), den));
        Pout[static_cast<int64_t>(r) * p + k] = row_bad ? __longlong_as_double(0x7ff8000000000000ll) : v;
        sP[k] = v;
        sT[k] = __double2float_ru(v);
      }
    }
    int64_t* cr = cnt_out + static_cast<int64_t>(r) * nb;
    double* Ar = A_out + static_cast<int64_t>(r) * nb;
    double* Br = B_out + static_cast<int64_t>(r) * nb;
    if (row_bad) {
      for (int k = tid; k < nb; k += kFuseThreads) {
        cr[k] = 0;
        Ar[k] = 0.0;
        Br[k] = 0.0;
      }
      if (tid == 0) status[r] = kStatusRange;
      __syncthreads();
      continue;
    }
    __syncthreads();
    const RowGrid g = row_grid(sP, p);
    const bool uni = row_is_uniform(sP, p, g, sE);  // includes a barrier
    if (!uni) {
      for (int k = tid; k < nb; k += kFuseThreads) {
        const double w = __dsub_rn(sP[k + 1], sP[k]);
        sE[k] = w > 0.0 ? __ddiv_rn(1.0, w) : 0.0;
      }
    }
    const double c0 = -(g.P0 * g.invD);
    const bool fastg = uni && fabs(c0) <= kFmaOffsetMax;
    if (tid == 0) {
      S.P = sP;
      S.E = sE;
      S.T = sT;
      S.cnt = sc;
      S.limb = sl;
      S.invD = g.invD;
      S.twoF = twoF;
      S.twoH = twoH;
      S.top = __double2float_rd(sP[p - 1]);
      S.scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
      S.p = p;
      S.uni = uni;
      S.bad = 0;
    }
    __syncthreads();

    // bucketing from shared memory
    {
      const uint32_t lane_base = smem_addr(sl + lane), cnt_base = smem_addr(sc);
      const int nf = static_cast<int>(d >> 2);
      const float4* x4 = reinterpret_cast<const float4*>(xs);
      for (int i = tid; i < nf; i += kFuseThreads) {
        const float4 c4 = x4[i];
        const float xv[4] = {c4.x, c4.y, c4.z, c4.w};
        int k[4];
        double v[4];
        bool all = fastg;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double G = fma(static_cast<double>(xv[e]), g.invD, c0);
          floor_split(G, k[e], v[e]);
          all = all && fabs(v[e] - 0.5) < lim && static_cast<unsigned>(k[e]) <= pm2;
        }
        if (all) {
#pragma unroll
          for (int e = 0; e < 4; ++e) wide_add<kFuseLimbBlock>(cnt_base, lane_base, k[e], v[e], twoF, twoH);
        } else {
          wide_exact<kFuseLimbBlock>(&S, xv, 4);
        }
      }
      for (int i = 4 * nf + tid; i < d; i += kFuseThreads) {
        const float xv[1] = {xs[i]};
        wide_exact<kFuseLimbBlock>(&S, xv, 1);
      }
    }
    __syncthreads();
    // the row's limb sums (thread: one limb of one bucket), then its statistics
    {
      const int li = tid / kFuseBuckets, k = tid % kFuseBuckets;
      unsigned long long sum = 0;
      if (k < nb && sc[k] != 0u) {
        uint4* c4 = reinterpret_cast<uint4*>(sl + li * kFuseLimbBlock + k * kWarp);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int jj = (j + tid) & 7;
          const uint4 v = c4[jj];
          sum += static_cast<unsigned long long>(v.x) + v.y + v.z + v.w;
          c4[jj] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      ssum[li * kFuseBuckets + k] = sum;
    }
    __syncthreads();
    {
      const double inv_two_fb = ldexp(1.0, -fb);
      for (int k = tid; k < nb; k += kFuseThreads) {
        const unsigned long long cn = sc[k];
        const unsigned long long s1 = ssum[k] + (ssum[kFuseBuckets + k] << kLimbBits);
        const unsigned long long s2 = ssum[2 * kFuseBuckets + k] + (ssum[3 * kFuseBuckets + k] << kLimbBits);
        const double c = static_cast<double>(cn);
        const double S1 = static_cast<double>(s1) * inv_two_fb;
        const double S2 = static_cast<double>(s2) * inv_two_fb;
        cr[k] = static_cast<int64_t>(cn);
        if (uni) {
          const double e = sE[k];
          Ar[k] = g.D * (S1 - c * e);
          Br[k] = g.D * g.D * (S2 - 2.0 * e * S1 + c * e * e);
        } else {
          const double w = sP[k + 1] - sP[k];
          Ar[k] = S1 * w;
          Br[k] = S2 * w * w;
        }
        sc[k] = 0u;
      }
      if (tid == 0) status[r] = S.bad ? kStatusRange : kStatusOk;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Bucketing for alphabets beyond the shared-memory counters (p > 512, up to
// 65536 values, e.g. every BF16 value of a range): the bucket by bisection on
// the row of P, the offset v as in k_bucket (uniform rows: (x - P_k)/D + eta_k;
// other rows: (x - P_k)/D_k), and 64-bit global additions of the count and the
// two fixed-point moments. A large alphabet spreads the entries over many
// buckets, so few additions contend.

constexpr int kGenThreads = 256;
constexpr int64_t kGenChunk = 16384;

__global__ void __launch_bounds__(kGenThreads)
k_bucket_general(const float* __restrict__ X, int64_t d, const double* __restrict__ Pall, int p, int fb,
                 unsigned long long* __restrict__ acc, int32_t* __restrict__ flag) {
  __shared__ int s_bad;
  const int r = blockIdx.y;
  const int nb = p - 1;
  const double* P = Pall + static_cast<int64_t>(r) * p;
  if (threadIdx.x == 0) s_bad = 0;
  const RowGrid g = row_grid(P, p);
  const bool uni = row_is_uniform(P, p, g, nullptr);  // includes a barrier
  const double twoF = ldexp(1.0, fb);
  const double P0 = P[0], Pl = P[p - 1];
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * kGenChunk;
  const int64_t end = beg + kGenChunk < d ? beg + kGenChunk : d;
  const float* x = X + static_cast<int64_t>(r) * d;
  unsigned long long* ga = acc + static_cast<int64_t>(r) * nb * 3;
  int bad = 0;
  for (int64_t i = beg + threadIdx.x; i < end; i += kGenThreads) {
    const double xd = static_cast<double>(__ldcs(x + i));
    if (!(xd >= P0) || !(xd <= Pl)) {
      bad = 1;
      continue;
    }
    int lo = 0, hi = p - 2;  // the largest k <= p-2 with P_k <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P[mid] <= xd)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int k = lo;
    const double y = __dsub_rn(xd, P[k]);
    double v;
    if (uni) {
      v = __dadd_rn(__dmul_rn(y, g.invD), grid_eta(P[k], g.P0, g.invD, k));
    } else {
      const double w = __dsub_rn(P[k + 1], P[k]);
      v = w > 0.0 ? __ddiv_rn(y, w) : 0.0;
    }
    v = fmin(fmax(v, 0.0), 1.0);
    unsigned long long* c = ga + 3 * static_cast<int64_t>(k);
    atomicAdd(c, 1ull);
    atomicAdd(c + 1, __double2ull_rn(v * twoF));
    atomicAdd(c + 2, __double2ull_rn(__dmul_rn(v, v) * twoF));
  }
  if (bad) s_bad = 1;
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) atomicOr(flag + r, 1);
}

// Fixed-point row sums -> cnt (int64), A = sum (x - P_k), B = sum (x - P_k)^2 (fp64).
__global__ void k_bucket_finish(const unsigned long long* __restrict__ acc, const double* __restrict__ Pall,
                                int p, int fb, const int32_t* __restrict__ flag, int64_t* __restrict__ cnt,
                                double* __restrict__ A, double* __restrict__ B, int32_t* __restrict__ status) {
  const int r = blockIdx.x;
  const int nb = p - 1;
  const double* P = Pall + static_cast<int64_t>(r) * p;
  const unsigned long long* gs = acc + static_cast<int64_t>(r) * nb * 3;
  const double inv_two_fb = ldexp(1.0, -fb);
  const RowGrid g = row_grid(P, p);
  const bool uni = row_is_uniform(P, p, g, nullptr);
  for (int k = threadIdx.x; k < nb; k += blockDim.x) {
    const int64_t o = static_cast<int64_t>(r) * nb + k;
    const double c = static_cast<double>(gs[3 * k + 0]);
    const double S1 = static_cast<double>(gs[3 * k + 1]) * inv_two_fb;
    const double S2 = static_cast<double>(gs[3 * k + 2]) * inv_two_fb;
    cnt[o] = static_cast<int64_t>(gs[3 * k + 0]);
    if (uni) {
      const double e = grid_eta(P[k], g.P0, g.invD, k);
      A[o] = g.D * (S1 - c * e);
      B[o] = g.D * g.D * (S2 - 2.0 * e * S1 + c * e * e);
    } else {
      const double w = P[k + 1] - P[k];
      A[o] = S1 * w;
      B[o] = S2 * w * w;
    }
  }
  if (threadIdx.x == 0 && status) status[r] = flag[r] ? kStatusRange : kStatusOk;
}

}  // namespace

int bucket_fraction_bits(int64_t d) { return d < (int64_t(1) << 27) ? 36 : 32; }

int64_t minmax_chunk(int64_t d) { return d < 16384 ? d : 16384; }

cudaError_t launch_bf16_alphabet(const float* X, int n, int64_t d, int p_max, double* P, int32_t* p_len,
                                 int32_t* status, float* part, cudaStream_t st) {
  const int64_t chunk = minmax_chunk(d);
  const int nc = static_cast<int>((d + chunk - 1) / chunk);
  k_minmax_partial<<<dim3(nc, n), kGridThreads, 0, st>>>(X, d, chunk, nc, part);
  note_launch();
  k_bf16_finish<<<n, 256, 0, st>>>(part, nc, p_max, P, p_len, status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_uniform_grid(const float* X, int n, int64_t d, int p, double* P, int32_t* status,
                                float* part, cudaStream_t st) {
  const int64_t chunk = minmax_chunk(d);
  const int nc = static_cast<int>((d + chunk - 1) / chunk);
  k_minmax_partial<<<dim3(nc, n), kGridThreads, 0, st>>>(X, d, chunk, nc, part);
  note_launch();
  k_grid_finish<<<n, 128, 0, st>>>(part, nc, p, P, status);
  note_launch();
  return cudaGetLastError();
}

size_t bucket_smem_bytes(int p) { return static_cast<size_t>(p) * (8 * 2 + 4); }

int64_t bucket_chunk(int64_t d) {
  const int64_t c = static_cast<int64_t>(kBucketSub) * kBucketSubsPerCta;
  return d < c ? d : c;
}

// The wide kernel needs more than the default 48 KB of dynamic shared memory;
// the attribute is per device and is set once for each (thread-safe).
cudaError_t wide_smem_attribute(int dev) {
  static std::once_flag once[64];
  static cudaError_t result[64];
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev]() {
    result[dev] = cudaFuncSetAttribute(k_bucket_wide, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kWideSmem));
  });
  return result[dev];
}

cudaError_t launch_bucket(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                          double* A, double* B, int32_t* status, unsigned long long* acc,
                          int32_t* flag, cudaStream_t st) {
  const int fb = bucket_fraction_bits(d);
  cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(unsigned long long) * 3 * (p - 1) * static_cast<size_t>(n), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(flag, 0, sizeof(int32_t) * n, st);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t wide_items = static_cast<int64_t>(n) * ((d + kWideChunk - 1) / kWideChunk);
  if (p > kMaxP) {
    const int nc = static_cast<int>((d + kGenChunk - 1) / kGenChunk);
    k_bucket_general<<<dim3(nc, n), kGenThreads, 0, st>>>(X, d, P, p, fb, acc, flag);
  } else if (p - 1 <= kWideBuckets && d >= kWideChunk && wide_items >= sms) {
    e = wide_smem_attribute(dev);
    if (e != cudaSuccess) return e;
    k_bucket_wide<<<sms, kWideThreads, kWideSmem, st>>>(X, n, d, P, p, fb, acc, flag);
  } else {
    const int64_t full = static_cast<int64_t>(kBucketSub) * kBucketSubsPerCta;
    const int64_t chunk = fill_chunk(n, d, static_cast<int64_t>(sms) * kBucketCtasPerSm, full, 4, 4096);
    const int nc = static_cast<int>((d + chunk - 1) / chunk);
    // 37 KB of static and at most 10 KB of dynamic shared memory (p = 512): no attribute needed
    if (chunk == full)
      k_bucket<true><<<dim3(nc, n), kBucketThreads, bucket_smem_bytes(p), st>>>(X, d, P, p, fb, acc, flag, chunk);
    else
      k_bucket<false><<<dim3(nc, n), kBucketThreads, bucket_smem_bytes(p), st>>>(X, d, P, p, fb, acc, flag, chunk);
  }
  note_launch();
  k_bucket_finish<<<n, 256, 0, st>>>(acc, P, p, fb, flag, cnt, A, B, status);
  note_launch();
  return cudaGetLastError();
}

bool grid_bucket_fused_ok(int64_t d, int p) { return d >= 1 && d <= kFuseMaxD && p - 1 <= kFuseBuckets; }

cudaError_t launch_grid_bucket_fused(const float* X, int n, int64_t d, int p, double* P, int64_t* cnt, double* A,
                                     double* B, int32_t* status, cudaStream_t st) {
  static std::once_flag once[64];
  static cudaError_t result[64];
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev]() {
    result[dev] = cudaFuncSetAttribute(k_grid_bucket_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(fuse_smem_bytes(kFuseMaxD)));
  });
  if (result[dev] != cudaSuccess) return result[dev];
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = fuse_smem_bytes(d);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_grid_bucket_rows, kFuseThreads, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n, sms * std::max(per_sm, 1));
  k_grid_bucket_rows<<<grid, kFuseThreads, smem, st>>>(X, n, d, p, bucket_fraction_bits(d), P, cnt, A, B, status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace ecasq

// ---------------------------------------------------------------------------
// Bucketing for callers that cannot allocate device memory (see
// ecasq_bucket_noalloc in include/ecasq.h). The accumulators live in a fixed
// array in this module's device memory instead of a caller workspace. Every
// GPU that loads the library holds this array until the process exits; all
// calls on a device share it, so calls that overlap on that GPU race.

namespace ecasq {

namespace {
constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

size_t round256(size_t b) { return (b + 255) & ~size_t(255); }
}  // namespace

size_t bucket_noalloc_bytes(int n, int p) {
  return round256(sizeof(unsigned long long) * 3 * static_cast<size_t>(n) * (p - 1)) +
         round256(sizeof(int32_t) * static_cast<size_t>(n));
}

size_t bucket_noalloc_capacity() { return kNoallocScratchBytes; }

cudaError_t launch_bucket_noalloc(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt, double* A,
                                  double* B, int32_t* status, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* base = nullptr;
  {
    // Host code cannot use the array's name as a device address: resolve it
    // once per device, with that device current.
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess) return e;
      g_noalloc_ptr[dev] = ptr;
    }
    base = g_noalloc_ptr[dev];
  }
  unsigned char* b = static_cast<unsigned char*>(base);
  auto* acc = reinterpret_cast<unsigned long long*>(b);
  auto* flag = reinterpret_cast<int32_t*>(b + round256(sizeof(unsigned long long) * 3 * static_cast<size_t>(n) * (p - 1)));
  // launch_bucket clears the accumulators and flags on the stream before use,
  // so nothing carries over from the previous call.
  return launch_bucket(X, P, n, d, p, cnt, A, B, status, acc, flag, st);
}

}  // namespace ecasq
