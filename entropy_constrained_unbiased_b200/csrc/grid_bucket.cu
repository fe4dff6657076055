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

// ---------------------------------------------------------------------------
// Bucketing. Sums are fixed point: an entry of bucket k with u = (x - P_k)/D_k,
// D_k = P_{k+1} - P_k, adds round(u * 2^fb) to the first-moment accumulator and
// round(u^2 * 2^fb) to the second; fb is chosen from d so that no 64-bit sum
// can overflow. Integer sums make the result independent of the order in
// which entries are added.
//
// Only 32-bit shared-memory atomics are native on this GPU, so the kernel
// groups entries by bucket with a counting sort per tile instead of adding
// 64-bit values atomically:
//   1. each thread buckets 8 entries and claims a slot in its bucket with a
//      32-bit atomic increment of the tile's bucket count;
//   2. warp 0 turns the counts into offsets (exclusive scan);
//   3. entries are scattered to their sorted position (u and the bucket id);
//   4. warps sweep the sorted tile 32 entries at a time with a segmented
//      inclusive scan (equal keys are contiguous); the last lane of each
//      segment adds the segment's sums to the warp's private accumulators.

constexpr int kBucketThreads = 256;
constexpr int kBucketWarps = kBucketThreads / kWarp;
constexpr int kPerThread = 8;                             // entries per thread per tile
constexpr int kTile = kBucketThreads * kPerThread;        // 2048

__global__ void __launch_bounds__(kBucketThreads)
k_bucket(const float* __restrict__ X, int64_t d, int64_t chunk, const double* __restrict__ Pall, int p, int fb,
         unsigned long long* __restrict__ acc, int32_t* __restrict__ flag) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int r = blockIdx.y;
  const int nb = p - 1;        // real buckets 0 .. p-2; key nb collects entries that add nothing
  double* sP = reinterpret_cast<double*>(smem);                                  // [p]
  double* sS = sP + p;                                                           // [p] 2^fb / D_k
  double* su = sS + p;                                                           // [kTile] sorted u * 2^fb
  unsigned long long* wa = reinterpret_cast<unsigned long long*>(su + kTile);    // [warps][p]
  unsigned long long* wb = wa + kBucketWarps * p;                                // [warps][p]
  unsigned long long* ccnt = wb + kBucketWarps * p;                              // [p]
  unsigned int* tcnt = reinterpret_cast<unsigned int*>(ccnt + p);                // [p]
  unsigned int* toff = tcnt + p;                                                 // [p]
  unsigned short* skey = reinterpret_cast<unsigned short*>(toff + p);            // [kTile]
  __shared__ int s_bad;

  const double* P = Pall + static_cast<int64_t>(r) * p;
  const double two_fb = ldexp(1.0, fb);
  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    sP[k] = P[k];
    sS[k] = (k < nb) ? two_fb / (P[k + 1] - P[k]) : 0.0;
    ccnt[k] = 0ull;
  }
  for (int k = threadIdx.x; k < kBucketWarps * p; k += blockDim.x) {
    wa[k] = 0ull;
    wb[k] = 0ull;
  }
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();

  const double scale = static_cast<double>(p - 1) / (sP[p - 1] - sP[0]);
  const double inv_two_fb = ldexp(1.0, -fb);
  const double magic = 0x1p52;  // v + 2^52 keeps round(v) in the low mantissa bits for 0 <= v < 2^52
  const unsigned long long low52 = (1ull << 52) - 1;
  const int lane = lane_id();
  const int w = warp_id();
  int bad = 0;

  const float* x = X + static_cast<int64_t>(r) * d;
  const int64_t beg = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t end = beg + chunk < d ? beg + chunk : d;
  const bool vec = ((reinterpret_cast<uintptr_t>(x + beg) & 15u) == 0);

  // Entry e of a thread in the tile starting at t0: position t0 + 4*(threadIdx.x + 256*(e/4)) + e%4.
  auto load_tile = [&](int64_t t0, float* xv) {
#pragma unroll
    for (int h = 0; h < kPerThread / 4; ++h) {
      const int64_t g = t0 + 4 * (threadIdx.x + static_cast<int64_t>(kBucketThreads) * h);
      const int cnt = g < end ? static_cast<int>(end - g < 4 ? end - g : 4) : 0;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (vec && cnt == 4) {
        v = __ldcs(reinterpret_cast<const float4*>(x + g));
      } else {
        if (cnt > 0) v.x = __ldcs(x + g);
        if (cnt > 1) v.y = __ldcs(x + g + 1);
        if (cnt > 2) v.z = __ldcs(x + g + 2);
        if (cnt > 3) v.w = __ldcs(x + g + 3);
      }
      xv[4 * h + 0] = v.x;
      xv[4 * h + 1] = v.y;
      xv[4 * h + 2] = v.z;
      xv[4 * h + 3] = v.w;
    }
  };
  auto valid = [&](int64_t t0, int e) {
    return t0 + 4 * (threadIdx.x + static_cast<int64_t>(kBucketThreads) * (e >> 2)) + (e & 3) < end;
  };

  float xv[kPerThread];
  if (beg < end) load_tile(beg, xv);
  for (int64_t t0 = beg; t0 < end; t0 += kTile) {
    for (int k = threadIdx.x; k < p; k += blockDim.x) tcnt[k] = 0u;
    int key[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      key[e] = nb;
      if (valid(t0, e)) {
        const int k = bucket_of(static_cast<double>(xv[e]), sP, p, scale);
        if (k < 0)
          bad = 1;
        else
          key[e] = k;
      }
    }
    __syncthreads();
    int slot[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) slot[e] = static_cast<int>(atomicAdd(tcnt + key[e], 1u));
    __syncthreads();
    if (w == 0) {  // exclusive scan of the tile's counts; per-CTA counts
      unsigned int run = 0;
      for (int base = 0; base < p; base += kWarp) {
        const int k = base + lane;
        const unsigned int c = (k < p) ? tcnt[k] : 0u;
        unsigned int incl = c;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const unsigned int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (k < p) {
          toff[k] = run + incl - c;
          ccnt[k] += c;
        }
        run += __shfl_sync(0xffffffffu, incl, kWarp - 1);
      }
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
      const int k = key[e];
      const int pos = static_cast<int>(toff[k]) + slot[e];
      su[pos] = (k < nb) ? (static_cast<double>(xv[e]) - sP[k]) * sS[k] : 0.0;
      skey[pos] = static_cast<unsigned short>(k);
    }
    __syncthreads();
    if (t0 + kTile < end) load_tile(t0 + kTile, xv);  // next tile in flight during the sweep
    const int nreal = static_cast<int>(toff[nb]);      // entries with a real bucket come first
    for (int base = w * kWarp; base < nreal; base += kBucketThreads) {
      const int pos = base + lane;
      int k = nb;
      unsigned long long a = 0, b = 0;
      if (pos < nreal) {
        k = skey[pos];
        const double u = su[pos];
        a = static_cast<unsigned long long>(__double_as_longlong(u + magic)) & low52;
        b = static_cast<unsigned long long>(__double_as_longlong(fma(u, u * inv_two_fb, magic))) & low52;
      }
#pragma unroll
      for (int o = 1; o < kWarp; o <<= 1) {
        const int ko = __shfl_up_sync(0xffffffffu, k, o);
        const unsigned long long ao = __shfl_up_sync(0xffffffffu, a, o);
        const unsigned long long bo = __shfl_up_sync(0xffffffffu, b, o);
        if (lane >= o && ko == k) {
          a += ao;
          b += bo;
        }
      }
      const int knext = __shfl_down_sync(0xffffffffu, k, 1);
      if (k < nb && (lane == kWarp - 1 || knext != k)) {
        wa[w * p + k] += a;
        wb[w * p + k] += b;
      }
    }
    __syncthreads();
  }
  if (bad) s_bad = 1;
  __syncthreads();

  unsigned long long* gacc = acc + static_cast<int64_t>(r) * nb * 3;
  for (int k = threadIdx.x; k < nb; k += blockDim.x) {
    const unsigned long long c = ccnt[k];
    if (c) {
      unsigned long long sa = 0, sb = 0;
#pragma unroll
      for (int q = 0; q < kBucketWarps; ++q) {
        sa += wa[q * p + k];
        sb += wb[q * p + k];
      }
      atomicAdd(gacc + 3 * k + 0, c);
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
  int lg = 0;
  while ((int64_t(1) << lg) < d + 1) ++lg;
  int fb = 63 - lg - 1;
  return fb > 50 ? 50 : fb;
}

int64_t minmax_chunk(int64_t d) { return d < 16384 ? d : 16384; }

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

size_t bucket_smem_bytes(int p) {
  return static_cast<size_t>(p) * 8 * 2 + static_cast<size_t>(kTile) * 8 +
         static_cast<size_t>(kBucketWarps) * p * 16 + static_cast<size_t>(p) * 8 + static_cast<size_t>(p) * 8 +
         static_cast<size_t>(kTile) * 2;
}

int64_t bucket_chunk(int64_t d) { return d < 32768 ? d : 32768; }

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
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(k_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    attr_set = true;
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
