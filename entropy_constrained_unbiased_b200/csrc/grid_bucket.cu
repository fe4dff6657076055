// Row statistics, uniform grid and bucketing of X onto the permissible set P.
//
// ECASQ summary (gist.science/pt/paper/2608.18147) §2.2 "Generalização": for an
// arbitrary permissible set P the solver costs O(p^2 s + d); the O(d) part is
// one pass that buckets every entry onto P and accumulates per-bucket
// statistics, from which every interval table is built without touching X
// again. Both kernels here are HBM-bound streams over X (4 bytes per entry).
#include <cuda_runtime.h>

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
// Bucketing. Sums are fixed point: an entry of bucket k with u = (x - P_k)/D_k,
// D_k = P_{k+1} - P_k, adds round(u * 2^36) to the first-moment sum and
// round(u^2 * 2^36) to the second. Integer sums make the result independent
// of the order in which entries are added.
//
// Only 32-bit shared-memory atomics are native on this GPU (64-bit and
// floating-point ones are emulated and collapse when lanes collide, which
// heavy-tailed inputs make the rule). So each 36-bit value is added as two
// 18-bit limbs to 32-bit counters. A limb is below 2^18 except the high limb
// of an entry exactly at the top of its bucket (2^18), so 2^13 entries per CTA
// keep every counter below 2^31. Per entry: one count and four limb additions,
// all return-less 32-bit atomics.

constexpr int kBucketThreads = 256;
constexpr int kFixBits = 36;
constexpr int kLimbBits = 18;
constexpr int64_t kBucketChunk = 8192;  // entries per CTA (see above)

__global__ void __launch_bounds__(kBucketThreads)
k_bucket(const float* __restrict__ X, int64_t d, int64_t chunk, const double* __restrict__ Pall, int p, int fb,
         unsigned long long* __restrict__ acc, int32_t* __restrict__ flag) {
  extern __shared__ __align__(16) unsigned char smem[];
  (void)fb;
  const int r = blockIdx.y;
  const int nb = p - 1;
  double* sP = reinterpret_cast<double*>(smem);                    // [p]
  double* sS = sP + p;                                             // [p] 2^36 / D_k
  unsigned int* hc = reinterpret_cast<unsigned int*>(sS + p);     // [p] count
  unsigned int* ha = hc + p;                                       // [2][p] first-moment limbs (lo, hi)
  unsigned int* hb = ha + 2 * p;                                   // [2][p] second-moment limbs
  float* sT = reinterpret_cast<float*>(hb + 2 * p);                // [p] exact fp32 thresholds
  __shared__ int s_bad;

  const double* P = Pall + static_cast<int64_t>(r) * p;
  const double two_f = 0x1p36;
  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    sP[k] = P[k];
    sS[k] = (k < nb) ? two_f / (P[k + 1] - P[k]) : 0.0;
    sT[k] = __double2float_ru(P[k]);
  }
  for (int k = threadIdx.x; k < 5 * p; k += blockDim.x) hc[k] = 0u;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();

  const float scale = static_cast<float>(static_cast<double>(p - 1) / (sP[p - 1] - sP[0]));
  const float top = __double2float_rd(sP[p - 1]);
  const double inv_two_f = 0x1p-36;
  const double magic = 0x1p52;  // v + 2^52 keeps round(v) in the low mantissa bits for 0 <= v < 2^52
  const unsigned int lmask = (1u << kLimbBits) - 1u;
  int bad = 0;

  auto one = [&](float xf) {
    const double x = static_cast<double>(xf);
    const int k = bucket_f32(xf, sT, top, p, scale);
    if (k < 0) {
      bad = 1;
      return;
    }
    const double u = (x - sP[k]) * sS[k];  // in [0, 2^36]
    const unsigned long long a = static_cast<unsigned long long>(__double_as_longlong(u + magic));
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(fma(u, u * inv_two_f, magic)));
    atomicAdd(hc + k, 1u);
    atomicAdd(ha + k, static_cast<unsigned int>(a) & lmask);
    atomicAdd(ha + p + k, static_cast<unsigned int>(a >> kLimbBits) & ((1u << (kFixBits + 1 - kLimbBits)) - 1u));
    atomicAdd(hb + k, static_cast<unsigned int>(b) & lmask);
    atomicAdd(hb + p + k, static_cast<unsigned int>(b >> kLimbBits) & ((1u << (kFixBits + 1 - kLimbBits)) - 1u));
  };

  const float* x = X + static_cast<int64_t>(r) * d;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int len = static_cast<int>((beg + chunk < d ? beg + chunk : d) - beg);
  const float* xc = x + beg;
  const bool vec = ((reinterpret_cast<uintptr_t>(xc) & 15u) == 0);
  int t = 0;
  if (vec) {
    const int nv = len >> 2;
    const float4* x4 = reinterpret_cast<const float4*>(xc);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const float4 v = __ldcs(x4 + i);
      one(v.x);
      one(v.y);
      one(v.z);
      one(v.w);
    }
    t = nv << 2;
  }
  for (int i = t + threadIdx.x; i < len; i += blockDim.x) one(__ldcs(xc + i));
  if (bad) s_bad = 1;
  __syncthreads();

  unsigned long long* gacc = acc + static_cast<int64_t>(r) * nb * 3;
  for (int k = threadIdx.x; k < nb; k += blockDim.x) {
    const unsigned int c = hc[k];
    if (c) {
      const unsigned long long sa = static_cast<unsigned long long>(ha[k]) +
                                    (static_cast<unsigned long long>(ha[p + k]) << kLimbBits);
      const unsigned long long sb = static_cast<unsigned long long>(hb[k]) +
                                    (static_cast<unsigned long long>(hb[p + k]) << kLimbBits);
      atomicAdd(gacc + 3 * k + 0, static_cast<unsigned long long>(c));
      atomicAdd(gacc + 3 * k + 1, sa);
      atomicAdd(gacc + 3 * k + 2, sb);
    }
  }
  if (threadIdx.x == 0 && s_bad) atomicOr(flag + r, 1);
}

// Fixed-point accumulators -> cnt (int64), A = sum y, B = sum y^2 (fp64).
__global__ void k_bucket_finish(const unsigned long long* __restrict__ acc, const double* __restrict__ Pall,
                                int p, int fb, const int32_t* __restrict__ flag, int64_t* __restrict__ cnt,
                                double* __restrict__ A, double* __restrict__ B, int32_t* __restrict__ status) {
  const int r = blockIdx.x;
  const int nb = p - 1;
  const double* P = Pall + static_cast<int64_t>(r) * p;
  const unsigned long long* g = acc + static_cast<int64_t>(r) * nb * 3;
  const double inv_two_fb = ldexp(1.0, -fb);
  for (int k = threadIdx.x; k < nb; k += blockDim.x) {
    const double D = P[k + 1] - P[k];
    const int64_t o = static_cast<int64_t>(r) * nb + k;
    cnt[o] = static_cast<int64_t>(g[3 * k + 0]);
    A[o] = static_cast<double>(g[3 * k + 1]) * inv_two_fb * D;
    B[o] = static_cast<double>(g[3 * k + 2]) * inv_two_fb * D * D;
  }
  if (threadIdx.x == 0 && status) status[r] = flag[r] ? kStatusRange : kStatusOk;
}

}  // namespace

int bucket_fraction_bits(int64_t d) {
  (void)d;
  return kFixBits;
}

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

size_t bucket_smem_bytes(int p) { return static_cast<size_t>(p) * (8 * 2 + 4 * 5 + 4); }

int64_t bucket_chunk(int64_t d) { return d < kBucketChunk ? d : kBucketChunk; }

cudaError_t launch_bucket(const float* X, const double* P, int n, int64_t d, int p, int64_t* cnt,
                          double* A, double* B, int32_t* status, unsigned long long* acc,
                          int32_t* flag, cudaStream_t st) {
  const int fb = bucket_fraction_bits(d);
  cudaError_t e = cudaMemsetAsync(acc, 0, sizeof(unsigned long long) * 3 * (p - 1) * static_cast<size_t>(n), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(flag, 0, sizeof(int32_t) * n, st);
  if (e != cudaSuccess) return e;
  const int64_t chunk = bucket_chunk(d);
  const int nc = static_cast<int>((d + chunk - 1) / chunk);
  const size_t smem = bucket_smem_bytes(p);
  // the attribute is per device: set it once for each device this process uses
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t ea = cudaFuncSetAttribute(k_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    if (ea != cudaSuccess) return ea;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  k_bucket<<<dim3(nc, n), kBucketThreads, smem, st>>>(X, d, chunk, P, p, fb, acc, flag);
  note_launch();
  k_bucket_finish<<<n, 256, 0, st>>>(acc, P, p, fb, flag, cnt, A, B, status);
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
