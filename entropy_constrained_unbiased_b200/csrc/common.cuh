// Device-side helpers shared by the ECASQ kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ecasq {

constexpr int kWarp = 32;
constexpr int kMaxP = 512;    // largest alphabet of the exact solver and of the shared-memory kernels
constexpr int kMaxPWide = 65536;  // largest alphabet of bucketing, encoding and the approximation
constexpr int kMaxS = 255;    // largest code size

// Per-vector status codes written by the device (mirrors include/ecasq.h).
constexpr int32_t kStatusOk = 0;
constexpr int32_t kStatusArg = -1;
constexpr int32_t kStatusRange = -2;
constexpr int32_t kStatusBudget = 1;
constexpr int32_t kStatusStall = -4;  // a bounded device wait gave up (mirrors ECASQ_ERR_CUDA)

__device__ __forceinline__ int lane_id() { return threadIdx.x & (kWarp - 1); }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// log2 on the special-function unit (MUFU.LG2, flush-to-zero; |rel err| ~ 2^-22).
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
// as 1, 2, 3", SC'11). Each round maps the counter (c0,c1,c2,c3) with key
// (k0,k1) through two 32x32->64 multiplications:
//   (c0,c1,c2,c3) <- (hi(m1*c2) ^ c1 ^ k0, lo(m1*c2), hi(m0*c0) ^ c3 ^ k1, lo(m0*c0))
// and the key advances by the two Weyl increments between rounds.
struct Philox4x32 {
  static constexpr uint32_t kMulA = 0xD2511F53u;  // multiplier applied to c0
  static constexpr uint32_t kMulB = 0xCD9E8D57u;  // multiplier applied to c2
  static constexpr uint32_t kWeylA = 0x9E3779B9u; // golden-ratio increment of k0
  static constexpr uint32_t kWeylB = 0xBB67AE85u; // sqrt(3)-1 increment of k1

  __device__ __forceinline__ static uint4 block(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      const uint32_t lo0 = kMulA * c.x;
      const uint32_t hi0 = __umulhi(kMulA, c.x);
      const uint32_t lo1 = kMulB * c.z;
      const uint32_t hi1 = __umulhi(kMulB, c.z);
      c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
      k0 += kWeylA;
      k1 += kWeylB;
    }
    return c;
  }

  // The same generator with the ten round keys (k0 + r W_A, k1 + r W_B)
  // precomputed by the host and passed as kernel parameters, so that a round
  // is two 32x32->64 multiplications and two three-input XORs.
  struct RoundKeys {
    uint32_t k0[10], k1[10];
  };
  __host__ static RoundKeys round_keys(uint32_t k0, uint32_t k1) {
    RoundKeys K;
    for (int r = 0; r < 10; ++r) {
      K.k0[r] = k0 + static_cast<uint32_t>(r) * kWeylA;
      K.k1[r] = k1 + static_cast<uint32_t>(r) * kWeylB;
    }
    return K;
  }
  __device__ __forceinline__ static uint4 block(uint4 c, const RoundKeys& K) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
      const uint64_t p0 = static_cast<uint64_t>(kMulA) * c.x;
      const uint64_t p1 = static_cast<uint64_t>(kMulB) * c.z;
      c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ K.k0[r], static_cast<uint32_t>(p1),
                     static_cast<uint32_t>(p0 >> 32) ^ c.w ^ K.k1[r], static_cast<uint32_t>(p0));
    }
    return c;
  }
};

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Warp-wide argmin: smallest value, ties to the smallest index. All lanes get it.
template <typename T>
__device__ __forceinline__ void warp_argmin(T& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const T ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov < v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

// Return-less 32-bit additions to shared memory through 32-bit shared-window
// addresses (red.shared.add.u32), with a compile-time byte offset.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
template <int kOff = 0>
__device__ __forceinline__ void red_shared_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0+%2], %1;" ::"r"(addr), "r"(v), "n"(kOff) : "memory");
}
// +1: the hardware combines the lanes of a warp that hit the same counter.
template <int kOff = 0>
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0+%1], 1;" ::"r"(addr), "n"(kOff) : "memory");
}

// Untiled bulk copies global -> shared (cp.async.bulk, completion counted in
// bytes on an mbarrier; addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(mbar)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(mbar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of the given parity, giving up after `limit` attempts
// (each attempt may suspend the thread for a bounded time); true on success.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t mbar, uint32_t parity, int limit) {
  for (int i = 0; i < limit; ++i)
    if (mbar_try_wait(mbar, parity)) return true;
  return false;
}

// Triangle addressing of the pair tables (0 <= k < l < p):
//   column l holds the entries (k, l), k = 0 .. l-1, at col_off(l) + k;
//   row l holds the entries (l, j), j = l+1 .. p-1, at row_off(l, p) + (j - l - 1).
__host__ __device__ __forceinline__ int col_off(int l) { return (l * (l - 1)) >> 1; }
__host__ __device__ __forceinline__ int row_off(int l, int p) { return l * (p - 1) - ((l * (l - 1)) >> 1); }
__host__ __device__ __forceinline__ int tri_size(int p) { return (p * (p - 1)) >> 1; }

// Bucket of x with exact fp32 thresholds: T[k] is the smallest float >= P_k and
// top the largest float <= P_{p-1}, so for a float x, P_k <= x <=> T[k] <= x
// and x <= P_{p-1} <=> x <= top; the result is the largest k <= p-2 with
// P_k <= x, or -1 outside [P_0, P_{p-1}]. The fp32 guess is corrected by the
// exact comparisons.
__device__ __forceinline__ int bucket_f32(float x, const float* __restrict__ T, float top, int p, float scale) {
  if (!(x >= T[0]) || !(x <= top)) return -1;
  int k = static_cast<int>((x - T[0]) * scale);
  k = k < 0 ? 0 : (k > p - 2 ? p - 2 : k);
  while (k > 0 && x < T[k]) --k;
  while (k < p - 2 && x >= T[k + 1]) ++k;
  return k;
}


// Bucket of x on an increasing alphabet P (in shared memory): the largest
// k <= p-2 with P_k <= x. Starts from the uniform-grid guess and walks; -1 when
// x is outside [P_0, P_{p-1}] or NaN.
__device__ __forceinline__ int bucket_of(double x, const double* __restrict__ P, int p, double scale) {
  if (!(x >= P[0]) || !(x <= P[p - 1])) return -1;
  int k = static_cast<int>((x - P[0]) * scale);
  k = k < 0 ? 0 : (k > p - 2 ? p - 2 : k);
  while (k > 0 && P[k] > x) --k;
  while (k < p - 2 && P[k + 1] <= x) ++k;
  return k;
}


// Uniform-grid description of an alphabet row: P_k = P_0 + (k + eta_k) D with
// D = (P_{p-1} - P_0)/(p-1). A row counts as uniform when every |eta_k| is at
// most 2^-36 bucket widths; then the bucket of x follows from (x - P_0)/D
// computed directly, with an exact search only for entries very close to a
// grid point (bucketing and encoding use this).
constexpr double kEtaMax = 0x1p-36;

// eta_k = (P_k - P_0)/D - k with every operation rounded as written (the bucket
// kernel and the finish kernel must agree bit for bit).
__device__ __forceinline__ double grid_eta(double Pk, double P0, double invD, int k) {
  return __dsub_rn(__dmul_rn(__dsub_rn(Pk, P0), invD), static_cast<double>(k));
}

struct RowGrid {
  double P0, D, invD;
};

__device__ __forceinline__ RowGrid row_grid(const double* __restrict__ P, int p) {
  RowGrid g;
  g.P0 = P[0];
  const double span = __dsub_rn(P[p - 1], g.P0);
  g.D = __ddiv_rn(span, static_cast<double>(p - 1));
  g.invD = __ddiv_rn(1.0, g.D);
  return g;
}

// Whether the row takes the uniform fast path; called by every thread of the
// block (block-wide OR). eta_out (optional, shared) receives eta_k.
__device__ __forceinline__ bool row_is_uniform(const double* __restrict__ P, int p, const RowGrid& g, double* eta_out) {
  int bad = !(g.D > 0.0) || !isfinite(g.invD);
  for (int k = threadIdx.x; k < p; k += blockDim.x) {
    const double e = grid_eta(P[k], g.P0, g.invD, k);
    if (eta_out) eta_out[k] = e;
    if (!(fabs(e) <= kEtaMax)) bad = 1;
  }
  return !__syncthreads_or(bad);
}


}  // namespace ecasq
