// Space-efficient approximation of ECASQ on the surrogate entropy H(I,B), and
// the iterative refinement ("Entropy-Constrained Adaptive Stochastic
// Quantization (ECASQ)", gist.science/pt/paper/2608.18147, §2.3 and §2.4).
//
// H(I,B) is the entropy of the pair (interval index, rounding bit). An interval
// [P_a, P_c] of the code contributes h(L(a,c)) + h(R(a,c)) to it, so
//   MSE + lambda*H(I,B) = sum over intervals of w(a,c),
//   w(a,c) = V(a,c)/d + lambda*(h(L(a,c)) + h(R(a,c))),
// a sum of per-interval costs. Its exact minimiser over codes with P_0, P_{p-1}
// and at most s values is the layered shortest path
//   G_1(0) = 0,  G_i(c) = min_{a<c} G_{i-1}(a) + w(a,c),  J* = min_{2<=i<=s} G_i(p-1),
// O(p^2 s) time and O(p s) state per solve: no pair-state, no back-pointers.
//
// Refinement works on the exact objective MSE + lambda*H(X^) at the same lambda.
// The interior values are split by position mod 3 into three classes; moving a
// value changes only its two intervals and three masses, so a class moves at
// once. Each value binary-searches its open interval between its neighbours on
// the sign of the forward difference of its local cost and moves only on a
// strict decrease; classes run in the order 0, 1, 2, for up to `refine`
// iterations or until an iteration moves nothing.
//
// GPU layout (one CTA per vector, persistent over vectors):
//   * per vector, fp64 V, R, L of every pair a < c (column-major) and the
//     layer-precision terms V/d and h(L)+h(R) in a per-CTA global slab
//     (L2-resident); the latter in padded columns (16-byte aligned, starts
//     staggered over the banks);
//   * per solve, the cost table w(a,c) (same padded columns) and the layers
//     G_1..G_s in shared memory (global slab when they do not fit). Each
//     column's a range is split near its middle; a thread sweeps the lower part
//     of one column and the upper part of its mirror column (equal work per
//     thread) with 16-byte loads of the column and of G_{i-1}: four relaxations
//     per pair of loads, two packed f32x2 additions and two three-input minima
//     in fp32; the two parts' minima are merged after a barrier;
//   * the argmin is recovered afterwards by recomputing the sums in the same
//     precision (the minimum is one of them exactly), smallest a first;
//   * refinement and the fp64 evaluation read the fp64 tables, which are summed
//     in the order of a direct sum with every operation rounded as written (no
//     contraction), so every decision is taken on the same values as a plain
//     fp64 statement of the method.
// Alphabets beyond 512 values (k_approx_wide, further down) keep O(p) prefix
// sums instead of the tables and evaluate each pair cost once per solve in a
// tiled sweep that relaxes all layers with it.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {
namespace {

// Padded column layout of the cost table, in 16-byte vectors of kvec values:
// column x (entries a = 0 .. x-1) starts at vector cb[x], 16-byte aligned, and
// cb[x] = x (mod 8), so the eight columns a quarter-warp reads with one 16-byte
// load each lie on distinct banks. Returns cb[x+1] from cb[x].
__host__ __device__ __forceinline__ int next_column(int start, int x, int kvec) {
  const int end = start + (x + kvec - 1) / kvec;
  return end + (((x + 1) - end) & 7);
}

// Two IEEE round-to-nearest additions in one packed f32x2 instruction.
__device__ __forceinline__ float2 add_f32x2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Three-input minimum (exact).
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// -(mu/d) log2(mu/d), 0 for mu <= 0.
__device__ __forceinline__ double hmass(double mu, double dd) {
  if (!(mu > 0.0)) return 0.0;
  const double q = __ddiv_rn(mu, dd);
  return __dmul_rn(-q, log2(q));
}

template <typename T>
struct AOps;

template <>
struct AOps<float> {
  using Vec = float4;
  __device__ static float4 cost4(float4 v, float4 e, double lam) {
    const float l = static_cast<float>(lam);
    return make_float4(__fmaf_rn(l, e.x, v.x), __fmaf_rn(l, e.y, v.y), __fmaf_rn(l, e.z, v.z), __fmaf_rn(l, e.w, v.w));
  }
  __device__ static float inf() { return __int_as_float(0x7f800000); }
  // Layer-precision pair terms: V/d, and h(L) + h(R) with the MUFU log2 (the
  // fp32 layers resolve no more than that).
  __device__ static void terms(double V, double R, double L, double dd, double inv_d, float* vt, float* et) {
    *vt = static_cast<float>(V * inv_d);
    const float qr = static_cast<float>(R * inv_d), ql = static_cast<float>(L * inv_d);
    const float hr = qr > 0.0f ? -qr * lg2_approx(qr) : 0.0f;
    const float hl = ql > 0.0f ? -ql * lg2_approx(ql) : 0.0f;
    *et = hl + hr;
    (void)dd;
  }
  __device__ static float add(float a, float b) { return __fadd_rn(a, b); }
  __device__ static float cost(float v, float e, double lam) { return __fmaf_rn(static_cast<float>(lam), e, v); }
  __device__ static float vmin(float a, float b) { return fminf(a, b); }
  // Four relaxations: two packed additions, two three-input minima.
  __device__ static void relax(float4 g, float4 w, float& b0, float& b1) {
    const float2 s01 = add_f32x2(make_float2(g.x, g.y), make_float2(w.x, w.y));
    const float2 s23 = add_f32x2(make_float2(g.z, g.w), make_float2(w.z, w.w));
    b0 = min3f(b0, s01.x, s01.y);
    b1 = min3f(b1, s23.x, s23.y);
  }
};

template <>
struct AOps<double> {
  using Vec = double2;
  __device__ static double2 cost4(double2 v, double2 e, double lam) {
    return make_double2(__dadd_rn(v.x, __dmul_rn(lam, e.x)), __dadd_rn(v.y, __dmul_rn(lam, e.y)));
  }
  __device__ static double inf() { return __longlong_as_double(0x7ff0000000000000ll); }
  // fp64 pair terms in the order of the definitions.
  __device__ static void terms(double V, double R, double L, double dd, double inv_d, double* vt, double* et) {
    *vt = __ddiv_rn(V, dd);
    *et = __dadd_rn(hmass(L, dd), hmass(R, dd));
    (void)inv_d;
  }
  __device__ static double add(double a, double b) { return __dadd_rn(a, b); }
  __device__ static double cost(double v, double e, double lam) { return __dadd_rn(v, __dmul_rn(lam, e)); }
  __device__ static double vmin(double a, double b) { return fmin(a, b); }
  __device__ static void relax(double2 g, double2 w, double& b0, double& b1) {
    b0 = fmin(b0, __dadd_rn(g.x, w.x));
    b1 = fmin(b1, __dadd_rn(g.y, w.y));
  }
};

template <typename T>
struct ACtx {
  int p, S, tri;
  double dd;
  double *sP, *sN, *sA, *sB;
  int* sQ;
  double* fbuf;  // [warps][p] local costs of the refinement
  int* moved;    // refinement move counter (shared)
  int* msh;      // code size handed from the recovery warp to the block (shared)
  int pst;       // row stride of the layers (p rounded up to a 16-byte multiple)
  const int* cb; // [p+1] first 16-byte vector of each padded cost column (shared)
  T* vt;         // padded columns: V/d in the layer precision
  T* et;         // padded columns: h(L) + h(R) in the layer precision
  double* V;     // [tri] fp64 interval tables, pair (a, c) at col_off(c) + a
  double* R;
  double* L;
  T* cost;  // padded columns, w(a, x) at cb[x] * (16 / sizeof(T)) + a
  T* G;     // [(S+1) * pst]
  __device__ int at(int a, int e) const { return col_off(e) + a; }
};

struct AOut {
  int m;
  double mse, H, HIB, J;
};

// Per-vector tables in two passes.
// Pass 1, column by column (e = 1 .. p-1): thread a (< e) adds bucket e-1 to its
// running sums N, T1, T2 over a .. e-1 (ascending, the order of a direct sum),
// every operation rounded as written, and stores V, R, L of (a, e); the threads
// of one column write adjacent words. Needs blockDim.x >= p - 1.
// Pass 2, over all pairs evenly: the layer-precision terms V/d and h(L)+h(R)
// (fp64 as defined for fp64 layers; fp32 with the MUFU log2 for fp32 layers).
template <typename T>
__device__ void build_pair_terms(const ACtx<T>& c) {
  const int p = c.p, a = threadIdx.x;
  double N = 0.0, T1 = 0.0, T2 = 0.0;
  const double Pa = a < p ? c.sP[a] : 0.0;
  for (int e = 1; e < p; ++e) {
    if (a < e) {
      const int k = e - 1;
      const double dk = __dsub_rn(c.sP[k], Pa);
      const double nk = c.sN[k];
      N = __dadd_rn(N, nk);
      T1 = __dadd_rn(T1, __dadd_rn(c.sA[k], __dmul_rn(nk, dk)));
      T2 = __dadd_rn(T2, __dadd_rn(__dadd_rn(c.sB[k], __dmul_rn(__dmul_rn(2.0, dk), c.sA[k])),
                                   __dmul_rn(__dmul_rn(nk, dk), dk)));
      const double W = __dsub_rn(c.sP[e], Pa);
      double V = __dsub_rn(__dmul_rn(W, T1), T2);
      V = V < 0.0 ? 0.0 : V;
      const double R = W > 0.0 ? __ddiv_rn(T1, W) : 0.0;
      const int i = col_off(e) + a;
      c.V[i] = V;
      c.R[i] = R;
      c.L[i] = __dsub_rn(N, R);
    }
  }
  __syncthreads();
  constexpr int kVec = 16 / sizeof(T);
  const double inv_d = 1.0 / c.dd;
  for (int i = threadIdx.x; i < c.tri; i += blockDim.x) {
    // column e of entry i: col_off(e) <= i < col_off(e + 1)
    int e = static_cast<int>((1.0f + sqrtf(1.0f + 8.0f * static_cast<float>(i))) * 0.5f);
    while (col_off(e) > i) --e;
    while (col_off(e + 1) <= i) ++e;
    const int aa = i - col_off(e);
    const int o = c.cb[e] * kVec + aa;
    AOps<T>::terms(c.V[i], c.R[i], c.L[i], c.dd, inv_d, c.vt + o, c.et + o);
  }
}

// Local exact cost of the value at position t placed at index x (fp64): its two
// intervals and the three masses that depend on it.
template <typename T>
__device__ __forceinline__ double local_cost(const ACtx<T>& c, double lam, int a, int e, int x, double r_before,
                                             double l_after) {
  const int ia = c.at(a, x), ib = c.at(x, e);
  const double f = __ddiv_rn(__dadd_rn(c.V[ia], c.V[ib]), c.dd);
  const double mu_prev = __dadd_rn(r_before, c.L[ia]);
  const double mu_self = __dadd_rn(c.R[ia], c.L[ib]);
  const double mu_next = __dadd_rn(c.R[ib], l_after);
  const double hs = __dadd_rn(__dadd_rn(hmass(mu_prev, c.dd), hmass(mu_self, c.dd)), hmass(mu_next, c.dd));
  return __dadd_rn(f, __dmul_rn(lam, hs));
}

// Refinement of c.sQ[0..m-1] in place (all threads). A warp takes one value of
// the class; its lanes evaluate the local cost at every index of the open
// interval, then lane 0 runs the binary search over those stored costs (the
// same decisions a search computing them on demand takes) and the move test.
template <typename T>
__device__ void refine_code(const ACtx<T>& c, double lam, int m, int iters) {
  const int lane = lane_id(), warp = warp_id(), nw = blockDim.x / kWarp;
  int* Q = c.sQ;
  double* fb = c.fbuf + static_cast<size_t>(warp) * c.p;
  for (int it = 0; it < iters; ++it) {
    if (threadIdx.x == 0) *c.moved = 0;
    __syncthreads();
    for (int cls = 0; cls < 3; ++cls) {
      const int npos = (m - 2 - cls + 2) / 3;  // positions 1 + cls + 3j <= m - 2
      for (int j = warp; j < npos; j += nw) {
        const int t = 1 + cls + 3 * j;
        const int a = Q[t - 1], e = Q[t + 1];
        const double r_before = (t - 1 > 0) ? c.R[c.at(Q[t - 2], a)] : 0.0;
        const double l_after = (t + 1 < m - 1) ? c.L[c.at(e, Q[t + 2])] : 0.0;
        const int lo = a + 1, hi = e - 1;
        for (int x = lo + lane; x <= hi; x += kWarp) fb[x - lo] = local_cost(c, lam, a, e, x, r_before, l_after);
        __syncwarp();
        if (lane == 0) {
          int l = lo, h = hi;
          while (l < h) {
            const int mid = l + (h - l) / 2;
            if (fb[mid + 1 - lo] < fb[mid - lo])
              l = mid + 1;
            else
              h = mid;
          }
          if (l != Q[t] && fb[l - lo] < fb[Q[t] - lo]) {
            Q[t] = l;  // no other value of the class reads position t
            atomicAdd(c.moved, 1);
          }
        }
        __syncwarp();
      }
      __syncthreads();
    }
    if (*c.moved == 0) break;
    __syncthreads();
  }
}

// fp64 evaluation of c.sQ (warp 0). The lanes fetch the intervals' tables and
// take the logarithms in parallel; lane 0 then adds the terms in ascending
// order of t, the order of the definitions.
template <typename T>
__device__ void evaluate_code(const ACtx<T>& c, double lam, bool refined, int m, AOut* out) {
  const int lane = lane_id();
  double* tv = c.fbuf;           // V_t
  double* th = c.fbuf + c.S;     // h(mu_t)
  double* tl = c.fbuf + 2 * c.S; // h(L_t)
  double* tr = c.fbuf + 3 * c.S; // h(R_t)
  for (int t = lane; t < m; t += kWarp) {
    double u = 0.0;
    if (t > 0) u = __dadd_rn(u, c.R[c.at(c.sQ[t - 1], c.sQ[t])]);
    if (t + 1 < m) {
      const int i = c.at(c.sQ[t], c.sQ[t + 1]);
      const double L = c.L[i];
      u = __dadd_rn(u, L);
      tv[t] = c.V[i];
      tl[t] = hmass(L, c.dd);
      tr[t] = hmass(c.R[i], c.dd);
    }
    th[t] = hmass(u, c.dd);
  }
  __syncwarp();
  if (lane == 0) {
    double sv = 0.0, sh = 0.0, sib = 0.0;
    for (int t = 0; t < m; ++t) {
      if (t + 1 < m) sv = __dadd_rn(sv, tv[t]);
      sh = __dadd_rn(sh, th[t]);
      if (t + 1 < m) {
        sib = __dadd_rn(sib, tl[t]);
        sib = __dadd_rn(sib, tr[t]);
      }
    }
    out->m = m;
    out->mse = __ddiv_rn(sv, c.dd);
    out->H = sh;
    out->HIB = sib;
    out->J = __dadd_rn(out->mse, __dmul_rn(lam, refined ? sh : sib));
  }
  __syncwarp();
}

// min over a = a0 .. a1-1 of Gp[a] + col[a] (+inf for an empty range): scalar
// up to a 16-byte boundary, then pairs of 16-byte loads of the column and of
// the layer (a broadcast within a warp's common range), one more single load,
// then the scalar tail. Gp and col are 16-byte aligned at a = 0.
template <typename T>
__device__ __forceinline__ T sweep_min(const T* __restrict__ Gp, const T* __restrict__ col, int a0, int a1) {
  using O = AOps<T>;
  using V16 = typename AOps<T>::Vec;
  constexpr int kVec = 16 / sizeof(T);
  T b0 = O::inf(), b1 = O::inf(), b2 = O::inf(), b3 = O::inf();
  int a = a0;
  const int ah = min(a1, (a + kVec - 1) / kVec * kVec);
  for (; a < ah; ++a) b0 = O::vmin(b0, O::add(Gp[a], col[a]));
  const int av = a + (a1 - a) / (2 * kVec) * (2 * kVec);
  for (; a < av; a += 2 * kVec) {
    const V16 g0 = *reinterpret_cast<const V16*>(Gp + a);
    const V16 g1 = *reinterpret_cast<const V16*>(Gp + a + kVec);
    const V16 w0 = *reinterpret_cast<const V16*>(col + a);
    const V16 w1 = *reinterpret_cast<const V16*>(col + a + kVec);
    O::relax(g0, w0, b0, b1);
    O::relax(g1, w1, b2, b3);
  }
  if (a + kVec <= a1) {
    O::relax(*reinterpret_cast<const V16*>(Gp + a), *reinterpret_cast<const V16*>(col + a), b2, b3);
    a += kVec;
  }
  for (; a < a1; ++a) b1 = O::vmin(b1, O::add(Gp[a], col[a]));
  return O::vmin(O::vmin(b0, b1), O::vmin(b2, b3));
}

// Split point of column x in layer i (a = i-2 .. x-1): the 16-byte boundary at
// or below the middle, clamped to the column.
template <typename T>
__device__ __forceinline__ int column_split(int i, int x) {
  constexpr int kVec = 16 / sizeof(T);
  const int mid = ((i - 2 + x) >> 1) / kVec * kVec;
  return mid < i - 2 ? i - 2 : mid;
}

// One solve at lambda (all threads): cost table, layers, recovery of the code,
// refinement, evaluation. Leaves the code in c.sQ and the figures in *out.
// kSplit: each column's a range is shared by two threads (few vectors, one CTA
// per SM: the longest column is the critical path of a layer).
template <typename T, bool kSplit>
__device__ void approx_solve(const ACtx<T>& c, double lam, int refine, AOut* out) {
  using O = AOps<T>;
  const int p = c.p, S = c.S, tid = threadIdx.x, bd = blockDim.x;
  constexpr int kVec = 16 / sizeof(T);
  using V16 = typename AOps<T>::Vec;
  // Cost table w = V/d + lambda*(h(L)+h(R)) from the L2-resident pair terms
  // (same padded layout): 16-byte loads, several in flight per thread, so the
  // table arrives in about one L2 round trip. Padding words are computed too and
  // never read.
  {
    const int nvec = c.cb[p];
    const V16* vv = reinterpret_cast<const V16*>(c.vt);
    const V16* ev = reinterpret_cast<const V16*>(c.et);
    V16* cv = reinterpret_cast<V16*>(c.cost);
#pragma unroll 4
    for (int q = tid; q < nvec; q += bd) cv[q] = AOps<T>::cost4(vv[q], ev[q], lam);
  }
  for (int x = tid; x < p; x += bd) c.G[c.pst + x] = (x == 0) ? T(0) : O::inf();
  __syncthreads();
  if constexpr (kSplit) {
    // Layer i: G_i(x) = min over a = i-2 .. x-1 of G_{i-1}(a) + w(a, x). Column x
    // is split at a 16-byte boundary near its middle; thread t sweeps the lower
    // part of column i-1+t and the upper part of column p-1-t, so every thread
    // does about half of the longest column. The upper parts' minima go to row 0
    // of G (unused otherwise) and are merged after a barrier. A minimum is exact,
    // so the split changes no value.
    T* __restrict__ Gh = c.G;
    for (int i = 2; i <= S; ++i) {
      const T* __restrict__ Gp = c.G + (i - 1) * c.pst;
      T* __restrict__ Gc = c.G + i * c.pst;
      const int ncol = p - i + 1;
      for (int t = tid; t < ncol; t += bd) {
        const int x1 = i - 1 + t, x2 = p - 1 - t;
        Gc[x1] = sweep_min<T>(Gp, c.cost + c.cb[x1] * kVec, i - 2, column_split<T>(i, x1));
        Gh[x2] = sweep_min<T>(Gp, c.cost + c.cb[x2] * kVec, column_split<T>(i, x2), x2);
      }
      __syncthreads();
      for (int x = i - 1 + tid; x < p; x += bd) Gc[x] = O::vmin(Gc[x], Gh[x]);
      __syncthreads();
    }
  } else {
    // One thread per column: the whole a range of column x.
    for (int i = 2; i <= S; ++i) {
      const T* __restrict__ Gp = c.G + (i - 1) * c.pst;
      T* __restrict__ Gc = c.G + i * c.pst;
      for (int x = i - 1 + tid; x < p; x += bd) {
        // min over a = i-2 .. x-1 of G_{i-1}(a) + w(a, x): scalar up to a 16-byte
        // boundary, then four (fp32) or two (fp64) consecutive a per load of the
        // column and of the layer (a broadcast), then the scalar tail.
        const T* __restrict__ col = c.cost + c.cb[x] * kVec;
        T b0 = O::inf(), b1 = O::inf(), b2 = O::inf(), b3 = O::inf();
        int a = i - 2;
        const int ah = min(x, (a + kVec - 1) / kVec * kVec);
        for (; a < ah; ++a) b0 = O::vmin(b0, O::add(Gp[a], col[a]));
        const int av = a + (x - a) / (2 * kVec) * (2 * kVec);
        for (; a < av; a += 2 * kVec) {
          const V16 g0 = *reinterpret_cast<const V16*>(Gp + a);
          const V16 g1 = *reinterpret_cast<const V16*>(Gp + a + kVec);
          const V16 w0 = *reinterpret_cast<const V16*>(col + a);
          const V16 w1 = *reinterpret_cast<const V16*>(col + a + kVec);
          AOps<T>::relax(g0, w0, b0, b1);
          AOps<T>::relax(g1, w1, b2, b3);
        }
        for (; a < x; ++a) b1 = O::vmin(b1, O::add(Gp[a], col[a]));
        Gc[x] = O::vmin(O::vmin(b0, b1), O::vmin(b2, b3));
      }
      __syncthreads();
    }
  }
  if (warp_id() == 0) {
    const int lane = lane_id();
    T bv = O::inf();
    int bi = 0x7fffffff;
    for (int i = 2 + lane; i <= S; i += kWarp) {
      const T g = c.G[i * c.pst + p - 1];
      if (g < bv) {
        bv = g;
        bi = i;
      }
    }
    warp_argmin(bv, bi);
    int m;
    if (bi == 0x7fffffff) {  // no finite candidate (non-finite inputs): {P_0, P_{p-1}}
      m = 2;
      if (lane == 0) {
        c.sQ[0] = 0;
        c.sQ[1] = p - 1;
      }
    } else {
      // Recovery: the smallest a whose sum equals the layer's minimum (it is
      // one of them exactly); all chunks of the column are tested at once.
      m = bi;
      int x = p - 1;
      if (lane == 0) c.sQ[m - 1] = x;
      for (int i = m; i >= 2; --i) {
        const T target = c.G[i * c.pst + x];
        const T* Gp = c.G + (i - 1) * c.pst;
        const T* col = c.cost + c.cb[x] * kVec;
        int found = 0x7fffffff;
#pragma unroll 4
        for (int base = i - 2; base < x; base += kWarp) {
          const int a = base + lane;
          const bool hit = a < x && O::add(Gp[a], col[a]) == target;
          const unsigned msk = __ballot_sync(0xffffffffu, hit);
          if (msk && found == 0x7fffffff) found = base + __ffs(msk) - 1;
        }
        if (found == 0x7fffffff) found = i - 2;  // not reached: the minimum is one of the sums
        x = found;
        if (lane == 0) c.sQ[i - 2] = x;
      }
    }
    if (lane == 0) *c.msh = m;
  }
  __syncthreads();
  const int m = *c.msh;
  if (refine > 0) refine_code(c, lam, m, refine);
  if (warp_id() == 0) evaluate_code(c, lam, refine > 0, m, out);
  __syncthreads();
}

// Outputs of a row that needs no solve: a degenerate row (one value, status
// ok) or a rejected one (status st, empty codes).
__device__ void approx_fill_trivial(const ApproxArgs& a, int r, int32_t st) {
  const int so = a.s_out;
  const int qv = (st == kStatusOk) ? 0 : -1;
  const int ml = (st == kStatusOk) ? 1 : 0;
  if (a.mode == 0) {
    for (int t = 0; t < a.n_lambda; ++t) {
      const int64_t w = static_cast<int64_t>(r) * a.n_lambda + t;
      for (int q = threadIdx.x; q < so; q += blockDim.x) a.Q[w * so + q] = (q == 0) ? qv : -1;
      if (threadIdx.x == 0) {
        a.Q_len[w] = ml;
        a.obj[w] = a.mse[w] = a.H[w] = a.HIB[w] = 0.0;
      }
    }
  } else {
    for (int q = threadIdx.x; q < so; q += blockDim.x) {
      a.Q1[int64_t(r) * so + q] = (q == 0) ? qv : -1;
      a.Q2[int64_t(r) * so + q] = (q == 0) ? qv : -1;
    }
    if (threadIdx.x == 0) {
      a.Q1_len[r] = a.Q2_len[r] = ml;
      a.theta[r] = a.lam_lo[r] = a.lam_hi[r] = 0.0;
      a.H1[r] = a.H2[r] = a.HIB1[r] = a.HIB2[r] = a.mse1[r] = a.mse2[r] = 0.0;
    }
  }
  if (threadIdx.x == 0) a.status[r] = st;
}

// The per-row driver shared by the approximation kernels: each lambda of the
// row's list (mode 0), or the bisection on lambda with two-way time-sharing
// (mode 1, the constrained rate H(I,B) for the plain approximation and H(X^)
// once refined), writing the row's outputs. solve(lambda) leaves the code in
// sQ and its figures in s_out (all threads); bracket = (P_{p-1} - P_0)^2.
template <class Solve>
__device__ void approx_drive(const ApproxArgs& a, int r, const int* sQ, int* sQ1, int* sQ2, int S, double bracket,
                             AOut& s_out, Solve solve) {
  const int so = a.s_out;
  if (a.mode == 0) {
    for (int t = 0; t < a.n_lambda; ++t) {
      const int64_t w = static_cast<int64_t>(r) * a.n_lambda + t;
      solve(a.lambda[w]);
      for (int q = threadIdx.x; q < so; q += blockDim.x) a.Q[w * so + q] = (q < s_out.m) ? sQ[q] : -1;
      if (threadIdx.x == 0) {
        a.Q_len[w] = s_out.m;
        a.obj[w] = s_out.J;
        a.mse[w] = s_out.mse;
        a.H[w] = s_out.H;
        a.HIB[w] = s_out.HIB;
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) a.status[r] = kStatusOk;
  } else {
    // Bisection on lambda with two-way time-sharing; the constrained rate is
    // H(I,B) for the plain approximation and H(X^) once refined.
    const bool refined = a.refine > 0;
    double lo = 0.0;
    double hi = bracket;
    double H1 = 0, H2 = 0, B1 = 0, B2 = 0, M1 = 0, M2 = 0, r1 = 0, r2 = 0;
    int m1 = 0, m2 = 0;
    auto keep = [&](int* dst, int& m, double& Hk, double& Bk, double& Mk) {
      for (int q = threadIdx.x; q < S; q += blockDim.x) dst[q] = sQ[q];
      m = s_out.m;
      Hk = s_out.H;
      Bk = s_out.HIB;
      Mk = s_out.mse;
    };
    auto rate = [&]() { return refined ? s_out.H : s_out.HIB; };
    int32_t status = kStatusOk;
    double theta = 0.0;
    solve(0.0);
    keep(sQ1, m1, H1, B1, M1);
    r1 = rate();
    if (r1 <= a.budget) {
      keep(sQ2, m2, H2, B2, M2);
      hi = 0.0;
    } else {
      __syncthreads();
      solve(hi);
      keep(sQ2, m2, H2, B2, M2);
      r2 = rate();
      if (r2 > a.budget) {
        status = kStatusBudget;
      } else {
        for (int it = 0; it < a.steps; ++it) {
          const double mid = 0.5 * (lo + hi);
          __syncthreads();
          solve(mid);
          const double rr = rate();
          if (rr > a.budget) {
            lo = mid;
            r1 = rr;
            keep(sQ1, m1, H1, B1, M1);
          } else {
            hi = mid;
            r2 = rr;
            keep(sQ2, m2, H2, B2, M2);
          }
        }
        const double th = (a.budget - r2) / (r1 - r2);
        theta = th < 0.0 ? 0.0 : (th > 1.0 ? 1.0 : th);
      }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < so; q += blockDim.x) {
      a.Q1[int64_t(r) * so + q] = (q < m1) ? sQ1[q] : -1;
      a.Q2[int64_t(r) * so + q] = (q < m2) ? sQ2[q] : -1;
    }
    if (threadIdx.x == 0) {
      a.Q1_len[r] = m1;
      a.Q2_len[r] = m2;
      a.theta[r] = theta;
      a.lam_lo[r] = lo;
      a.lam_hi[r] = hi;
      a.H1[r] = H1;
      a.H2[r] = H2;
      a.HIB1[r] = B1;
      a.HIB2[r] = B2;
      a.mse1[r] = M1;
      a.mse2[r] = M2;
      a.status[r] = status;
    }
  }
}

template <typename T, bool kSmem, bool kSplit>
__global__ void __launch_bounds__(512, 1) k_approx(ApproxArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ AOut s_out;
  __shared__ int s_flag;
  __shared__ int s_misc[2];

  const int p = a.p, S = a.s;
  ACtx<T> c;
  c.p = p;
  c.S = S;
  c.tri = tri_size(p);
  c.dd = static_cast<double>(a.d);

  unsigned char* sp = smem;
  auto carve = [&sp](size_t bytes) {
    unsigned char* r = sp;
    sp += (bytes + 15) & ~size_t(15);
    return r;
  };
  c.sP = reinterpret_cast<double*>(carve(sizeof(double) * p));
  c.sN = reinterpret_cast<double*>(carve(sizeof(double) * p));
  c.sA = reinterpret_cast<double*>(carve(sizeof(double) * p));
  c.sB = reinterpret_cast<double*>(carve(sizeof(double) * p));
  c.sQ = reinterpret_cast<int*>(carve(sizeof(int) * S));
  int* sQ1 = reinterpret_cast<int*>(carve(sizeof(int) * S));
  int* sQ2 = reinterpret_cast<int*>(carve(sizeof(int) * S));
  int* cbs = reinterpret_cast<int*>(carve(sizeof(int) * (p + 1)));
  c.moved = &s_misc[0];
  c.msh = &s_misc[1];
  constexpr int kVec = 16 / sizeof(T);
  if (threadIdx.x == 0) {
    cbs[0] = 0;
    for (int x = 0; x < p; ++x) cbs[x + 1] = next_column(cbs[x], x, kVec);
  }
  __syncthreads();
  c.cb = cbs;
  c.pst = (p + kVec - 1) / kVec * kVec;

  // Global slab: [V/d][h(L)+h(R)] in T (padded columns), [V][R][L] in fp64,
  // then the cost table (whose space the refinement and the evaluation reuse)
  // and the layers when they are not in shared memory.
  unsigned char* gs = a.scratch + static_cast<size_t>(blockIdx.x) * a.scratch_per_cta;
  const size_t vb = (16 * static_cast<size_t>(cbs[p]) + 255) & ~size_t(255);
  const size_t db = (sizeof(double) * static_cast<size_t>(c.tri) + 255) & ~size_t(255);
  const size_t fb = sizeof(double) * p * (blockDim.x / kWarp);
  const size_t cbytes = (((vb > fb) ? vb : fb) + 255) & ~size_t(255);
  c.vt = reinterpret_cast<T*>(gs);
  c.et = reinterpret_cast<T*>(gs + vb);
  c.V = reinterpret_cast<double*>(gs + 2 * vb);
  c.R = reinterpret_cast<double*>(gs + 2 * vb + db);
  c.L = reinterpret_cast<double*>(gs + 2 * vb + 2 * db);
  unsigned char* big = kSmem ? sp : gs + 2 * vb + 3 * db;
  c.cost = reinterpret_cast<T*>(big);
  c.fbuf = reinterpret_cast<double*>(big);
  c.G = reinterpret_cast<T*>(big + cbytes);

  for (int r = blockIdx.x; r < a.n; r += gridDim.x) {
    const double* P = a.P + static_cast<int64_t>(r) * p;
    const int64_t bo = static_cast<int64_t>(r) * (p - 1);
    if (threadIdx.x == 0) s_flag = a.in_status ? a.in_status[r] : 0;
    for (int k = threadIdx.x; k < p; k += blockDim.x) {
      c.sP[k] = P[k];
      if (k < p - 1) {
        c.sN[k] = static_cast<double>(a.cnt[bo + k]);
        c.sA[k] = a.A[bo + k];
        c.sB[k] = a.B[bo + k];
      }
    }
    __syncthreads();
    const bool degenerate = (c.sP[0] == c.sP[p - 1]);
    int bad = 0;
    if (!degenerate)
      for (int k = threadIdx.x; k < p - 1; k += blockDim.x) bad |= !(c.sP[k] < c.sP[k + 1]);
    bad = __syncthreads_or(bad);
    const int32_t st = s_flag != 0 ? s_flag : (bad ? kStatusArg : kStatusOk);

    if (st != kStatusOk || degenerate) {
      approx_fill_trivial(a, r, st);
      __syncthreads();
      continue;
    }

    build_pair_terms(c);
    __syncthreads();

    approx_drive(a, r, c.sQ, sQ1, sQ2, S, (c.sP[p - 1] - c.sP[0]) * (c.sP[p - 1] - c.sP[0]), s_out,
                 [&](double lam) { approx_solve<T, kSplit>(c, lam, a.refine, &s_out); });
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// The approximation for large alphabets (p > 512, up to 65536 values: e.g.
// every BF16 value of a range, §5 "Generalidade"), in O(p) memory per vector
// besides the layers. The pair terms V, R, L of an interval [P_a, P_e] come
// from six prefix sums over the buckets, with u_k = P_k - P_0:
//   N  = sum n_k,
//   T1 = sum (x - P_a)   = SA + SNU - u_a N,
//   T2 = sum (x - P_a)^2 = SB + 2 SAU - 2 u_a SA + SNUU - 2 u_a SNU + u_a^2 N,
// over k = a .. e-1 (SA = sum A_k, SB = sum B_k, SNU = sum n_k u_k,
// SAU = sum A_k u_k, SNUU = sum n_k u_k^2; each a difference of two prefix
// sums), then V = W T1 - T2 (clamped at 0), R = T1 / W, L = N - R with
// W = P_e - P_a. The differences cancel: the relative error of T2 grows like
// (u_e / W)^2 times the fp64 unit, below 1e-7 for the alphabets this path
// serves, so the layers run in fp32 (their own resolution) with the cost
// w(a,e) = V/d + lambda (h(L) + h(R)) computed on the fly for every
// relaxation, and the recovery recomputes the same fp32 values. The
// refinement compares local costs from the same prefix terms in fp64; the
// reported figures of the final code (mse, H, H(I,B), objective) are direct
// fp64 sums over each interval's buckets in the order of the definitions.

// One end of an interval: the six prefix sums up to index k (buckets
// 0 .. k-1), P_k and u_k = P_k - P_0. A pair's terms are differences of its
// two ends' sums, so a column's end can be loaded once and reused.
struct WSide {
  double N, SA, SB, SNU, SAU, SNUU, P, u;
};

struct WCtx {
  int p, S, pst;
  double dd, inv_d;
  const double* P;  // [p] the row of the alphabet
  double* pre;      // [6][p] prefix sums N, SA, SB, SNU, SAU, SNUU (index k: buckets 0 .. k-1)
  double* nb;       // [p] bucket counts, A, B (for the direct sums)
  double* ab;
  double* bb;
  float* G;         // [(S+1) * pst] layers
  double* fbuf;     // [warps][p] local costs of the refinement
  int* sQ;
  int* moved;
  int* msh;
  int* found;
};

__device__ __forceinline__ WSide wside(const WCtx& c, int k) {
  const double* pr = c.pre;
  const int p = c.p;
  WSide w;
  w.N = pr[k];
  w.SA = pr[p + k];
  w.SB = pr[2 * p + k];
  w.SNU = pr[3 * p + k];
  w.SAU = pr[4 * p + k];
  w.SNUU = pr[5 * p + k];
  w.P = c.P[k];
  w.u = __dsub_rn(c.P[k], c.P[0]);
  return w;
}

__device__ __forceinline__ void wpair_sides(const WSide& sa, const WSide& se, double& V, double& R, double& L) {
  const double N = __dsub_rn(se.N, sa.N);
  const double SA = __dsub_rn(se.SA, sa.SA);
  const double SB = __dsub_rn(se.SB, sa.SB);
  const double SNU = __dsub_rn(se.SNU, sa.SNU);
  const double SAU = __dsub_rn(se.SAU, sa.SAU);
  const double SNUU = __dsub_rn(se.SNUU, sa.SNUU);
  const double ua = sa.u;
  const double W = __dsub_rn(se.P, sa.P);
  const double T1 = SA + SNU - ua * N;
  const double T2 = SB + 2.0 * SAU - 2.0 * ua * SA + SNUU - 2.0 * ua * SNU + ua * ua * N;
  V = fmax(W * T1 - T2, 0.0);
  R = W > 0.0 ? T1 / W : 0.0;
  L = N - R;
}

__device__ __forceinline__ void wpair(const WCtx& c, int a, int e, double& V, double& R, double& L) {
  wpair_sides(wside(c, a), wside(c, e), V, R, L);
}

// The layers' cost w(a, e) in fp32 (as the fp32 table path forms it).
__device__ __forceinline__ float wcost_sides(double inv_d, const WSide& sa, const WSide& se, float lamf) {
  double V, R, L;
  wpair_sides(sa, se, V, R, L);
  const float vt = static_cast<float>(V * inv_d);
  const float qr = static_cast<float>(R * inv_d), ql = static_cast<float>(L * inv_d);
  const float hr = qr > 0.0f ? -qr * lg2_approx(qr) : 0.0f;
  const float hl = ql > 0.0f ? -ql * lg2_approx(ql) : 0.0f;
  return __fmaf_rn(lamf, hl + hr, vt);
}

__device__ __forceinline__ float wcost(const WCtx& c, int a, int e, float lamf) {
  return wcost_sides(c.inv_d, wside(c, a), wside(c, e), lamf);
}

// Direct fp64 sums over buckets a .. e-1, every operation rounded as written,
// in the order of build_pair_terms (the oracle's tables).
__device__ void wpair_direct(const WCtx& c, int a, int e, double& V, double& R, double& L) {
  double N = 0.0, T1 = 0.0, T2 = 0.0;
  const double Pa = c.P[a];
  for (int k = a; k < e; ++k) {
    const double dk = __dsub_rn(c.P[k], Pa);
    const double nk = c.nb[k];
    N = __dadd_rn(N, nk);
    T1 = __dadd_rn(T1, __dadd_rn(c.ab[k], __dmul_rn(nk, dk)));
    T2 = __dadd_rn(T2, __dadd_rn(__dadd_rn(c.bb[k], __dmul_rn(__dmul_rn(2.0, dk), c.ab[k])), __dmul_rn(__dmul_rn(nk, dk), dk)));
  }
  const double W = __dsub_rn(c.P[e], Pa);
  V = __dsub_rn(__dmul_rn(W, T1), T2);
  V = V < 0.0 ? 0.0 : V;
  R = W > 0.0 ? __ddiv_rn(T1, W) : 0.0;
  L = __dsub_rn(N, R);
}

__device__ __forceinline__ double wlocal_cost(const WCtx& c, double lam, int a, int e, int x, double r_before,
                                              double l_after) {
  double Va, Ra, La, Vb, Rb, Lb;
  wpair(c, a, x, Va, Ra, La);
  wpair(c, x, e, Vb, Rb, Lb);
  const double f = __ddiv_rn(__dadd_rn(Va, Vb), c.dd);
  const double mu_prev = __dadd_rn(r_before, La);
  const double mu_self = __dadd_rn(Ra, Lb);
  const double mu_next = __dadd_rn(Rb, l_after);
  const double hs = __dadd_rn(__dadd_rn(hmass(mu_prev, c.dd), hmass(mu_self, c.dd)), hmass(mu_next, c.dd));
  return __dadd_rn(f, __dmul_rn(lam, hs));
}

// Refinement as refine_code, on the prefix terms.
__device__ void wrefine(const WCtx& c, double lam, int m, int iters) {
  const int lane = lane_id(), warp = warp_id(), nw = blockDim.x / kWarp;
  int* Q = c.sQ;
  double* fb = c.fbuf + static_cast<size_t>(warp) * c.p;
  for (int it = 0; it < iters; ++it) {
    if (threadIdx.x == 0) *c.moved = 0;
    __syncthreads();
    for (int cls = 0; cls < 3; ++cls) {
      const int npos = (m - 2 - cls + 2) / 3;
      for (int j = warp; j < npos; j += nw) {
        const int t = 1 + cls + 3 * j;
        const int a = Q[t - 1], e = Q[t + 1];
        double Vx, Rx, Lx;
        double r_before = 0.0, l_after = 0.0;
        if (t - 1 > 0) {
          wpair(c, Q[t - 2], a, Vx, Rx, Lx);
          r_before = Rx;
        }
        if (t + 1 < m - 1) {
          wpair(c, e, Q[t + 2], Vx, Rx, Lx);
          l_after = Lx;
        }
        const int lo = a + 1, hi = e - 1;
        for (int x = lo + lane; x <= hi; x += kWarp) fb[x - lo] = wlocal_cost(c, lam, a, e, x, r_before, l_after);
        __syncwarp();
        if (lane == 0) {
          int l = lo, h = hi;
          while (l < h) {
            const int mid = l + (h - l) / 2;
            if (fb[mid + 1 - lo] < fb[mid - lo])
              l = mid + 1;
            else
              h = mid;
          }
          if (l != Q[t] && fb[l - lo] < fb[Q[t] - lo]) {
            Q[t] = l;
            atomicAdd(c.moved, 1);
          }
        }
        __syncwarp();
      }
      __syncthreads();
    }
    if (*c.moved == 0) break;
    __syncthreads();
  }
}

// fp64 figures of c.sQ (warp 0), as evaluate_code, from direct sums.
__device__ void wevaluate(const WCtx& c, double lam, bool refined, int m, AOut* out) {
  const int lane = lane_id();
  double* tv = c.fbuf;
  double* th = c.fbuf + c.S;
  double* tl = c.fbuf + 2 * c.S;
  double* tr = c.fbuf + 3 * c.S;
  double* tR = c.fbuf + 4 * c.S;
  double* tL = c.fbuf + 5 * c.S;
  for (int t = lane; t + 1 < m; t += kWarp) {
    double V, R, L;
    wpair_direct(c, c.sQ[t], c.sQ[t + 1], V, R, L);
    tv[t] = V;
    tR[t] = R;
    tL[t] = L;
    tl[t] = hmass(L, c.dd);
    tr[t] = hmass(R, c.dd);
  }
  __syncwarp();
  for (int t = lane; t < m; t += kWarp) {
    double u = 0.0;
    if (t > 0) u = __dadd_rn(u, tR[t - 1]);
    if (t + 1 < m) u = __dadd_rn(u, tL[t]);
    th[t] = hmass(u, c.dd);
  }
  __syncwarp();
  if (lane == 0) {
    double sv = 0.0, sh = 0.0, sib = 0.0;
    for (int t = 0; t < m; ++t) {
      if (t + 1 < m) sv = __dadd_rn(sv, tv[t]);
      sh = __dadd_rn(sh, th[t]);
      if (t + 1 < m) {
        sib = __dadd_rn(sib, tl[t]);
        sib = __dadd_rn(sib, tr[t]);
      }
    }
    out->m = m;
    out->mse = __ddiv_rn(sv, c.dd);
    out->H = sh;
    out->HIB = sib;
    out->J = __dadd_rn(out->mse, __dmul_rn(lam, refined ? sh : sib));
  }
  __syncwarp();
}

// Tiled layers (S - 1 <= kS layers after the first). Every pair cost w(a, x)
// is computed once per solve and relaxes all layers: G_i(x) depends only on
// G_{i-1}(a), a < x, so once the columns left of an X-tile of kWT columns are
// final in every layer, the pairs (a, x) with a in an earlier A-tile of kWA
// rows relax layers 2 .. S together. The warps share the earlier A-tiles (lane =
// column x, whose end of the pair terms stays in registers for the whole
// X-tile; the A-tile's ends and layer values staged in shared memory and read
// as broadcasts), their partial minima are merged, and warp 0 runs the
// diagonal block (a, x in the same tile, a < x; its pair costs computed by all
// warps) layer by layer. A minimum does not depend on the order of its terms,
// so every G_i(x) equals the one the layer-by-layer sweep gives; below the
// first reachable column (x < i - 1) the layer holds +inf.
constexpr int kWT = 32;  // columns of an X-tile (one per lane)
constexpr int kWA = 16;  // rows of an A-tile

// Layers kept per lane by the tiled sweep for a code of S values (0: the
// layer-by-layer sweep, S > 33).
__host__ __device__ inline int wide_tile_layers(int S) {
  return S - 1 <= 8 ? 8 : (S - 1 <= 16 ? 16 : (S - 1 <= 32 ? 32 : 0));
}

constexpr int kWideApproxThreads = 512;

// Dynamic shared memory of k_approx_wide: the three codes, then the tiled
// sweep's staging, partial minima, block costs, diagonal block and A-tile ends.
__host__ __device__ inline size_t wide_smem_head(int S) {
  return (sizeof(int) * 3 * static_cast<size_t>(S) + 15) & ~size_t(15);
}
__host__ __device__ inline size_t wide_smem_bytes(int S) {
  const size_t kS = static_cast<size_t>(wide_tile_layers(S));
  const size_t nw = kWideApproxThreads / kWarp;
  return wide_smem_head(S) +
         (kS ? sizeof(float) * (nw * kWA * kS + nw * kS * kWT + nw * kWA * kWT + kWT * kWT) + sizeof(WSide) * nw * kWA
             : 0);
}

template <int kS>
__device__ __noinline__ void wide_layers_tiled(const WCtx& cx, float lamf) {
  // the context in registers: a reference would be re-read from local memory
  // after every shared-memory store
  const WCtx c = cx;
  const int p = c.p, S = c.S, pst = c.pst, tid = threadIdx.x, bd = blockDim.x;
  const int lane = lane_id(), warp = warp_id(), nw = bd / kWarp;
  const double inv_d = c.inv_d;
  float* __restrict__ G = c.G;
  // the tiles, carved here from the dynamic shared array (after the three
  // codes) so that every access compiles to a shared-memory instruction:
  // staged layer values [warps][kWA][kS], partial minima [warps][kS][kWT], block
  // costs [warps][kWA][kWT], the diagonal block's costs [kWT][kWT], the A-tile
  // ends [warps][kWA]
  extern __shared__ __align__(16) unsigned char smem[];
  float* tG = reinterpret_cast<float*>(smem + wide_smem_head(S));
  float* tpart = tG + static_cast<size_t>(nw) * kWA * kS;
  float* tw = tpart + static_cast<size_t>(nw) * kS * kWT;
  float* tdiag = tw + static_cast<size_t>(nw) * kWA * kWT;
  WSide* tside = reinterpret_cast<WSide*>(tdiag + kWT * kWT);
  const float inf = __int_as_float(0x7f800000);
  for (int i = 1; i <= S; ++i)
    for (int x = tid; x < p; x += bd) G[i * pst + x] = (i == 1 && x == 0) ? 0.0f : inf;
  __syncthreads();
  float* gs = tG + static_cast<size_t>(warp) * kWA * kS;       // [kWA][kS]
  float* ws = tw + static_cast<size_t>(warp) * kWA * kWT;      // [kWA][kWT]
  float* part = tpart + static_cast<size_t>(warp) * kS * kWT;  // [kS][kWT]
  WSide* as = tside + static_cast<size_t>(warp) * kWA;         // [kWA]
  const int ntile = (p + kWT - 1) / kWT;
  for (int xt = 0; xt < ntile; ++xt) {
    const int x0 = xt * kWT, x = x0 + lane;
    const bool xin = x < p;
    const WSide xs = wside(c, xin ? x : p - 1);
#pragma unroll
    for (int q = 0; q < kS; ++q) part[q * kWT + lane] = inf;
    for (int at = warp; at < xt * (kWT / kWA); at += nw) {
      const int a0 = at * kWA;
      // the A-tile's ends and gs[j][q] = G_{q+1}(a0 + j) (layers past S - 1
      // are not read), then the block's costs ws[j][lane] = w(a0 + j, x); the
      // partial minima stay in shared memory between blocks so that the cost
      // evaluation has the registers
      if (lane < kWA) as[lane] = wside(c, a0 + lane);
#pragma unroll
      for (int e = lane; e < kWA * kS; e += kWarp) {  // consecutive lanes, consecutive words
        const int j = e / kS, q = e % kS;
        gs[e] = (q + 1 <= S - 1) ? G[(q + 1) * pst + a0 + j] : inf;
      }
      __syncwarp();
      for (int j = 0; j < kWA; ++j) ws[j * kWT + lane] = xin ? wcost_sides(inv_d, as[j], xs, lamf) : 0.0f;
      __syncwarp();
      float best[kS];
#pragma unroll
      for (int q = 0; q < kS; ++q) best[q] = part[q * kWT + lane];
      // two rows at a time: eight relaxations are four packed additions and
      // four three-input minima
#pragma unroll 1
      for (int j = 0; j < kWA; j += 2) {
        const float w0 = ws[j * kWT + lane], w1 = ws[(j + 1) * kWT + lane];
        const float2 ww0 = make_float2(w0, w0), ww1 = make_float2(w1, w1);
        const float4* g0 = reinterpret_cast<const float4*>(gs + j * kS);
        const float4* g1 = reinterpret_cast<const float4*>(gs + (j + 1) * kS);
#pragma unroll
        for (int q4 = 0; q4 < kS / 4; ++q4) {
          const float4 ga = g0[q4], gb = g1[q4];
          const float2 a01 = add_f32x2(make_float2(ga.x, ga.y), ww0);
          const float2 a23 = add_f32x2(make_float2(ga.z, ga.w), ww0);
          const float2 b01 = add_f32x2(make_float2(gb.x, gb.y), ww1);
          const float2 b23 = add_f32x2(make_float2(gb.z, gb.w), ww1);
          best[4 * q4 + 0] = min3f(best[4 * q4 + 0], a01.x, b01.x);
          best[4 * q4 + 1] = min3f(best[4 * q4 + 1], a01.y, b01.y);
          best[4 * q4 + 2] = min3f(best[4 * q4 + 2], a23.x, b23.x);
          best[4 * q4 + 3] = min3f(best[4 * q4 + 3], a23.y, b23.y);
        }
      }
#pragma unroll
      for (int q = 0; q < kS; ++q) part[q * kWT + lane] = best[q];
      __syncwarp();
    }
    // the diagonal block's costs wd[j][lane] = w(x0 + j, x), +inf unless j < lane
    for (int j = warp; j < kWT; j += nw)
      tdiag[j * kWT + lane] = (xin && j < lane) ? wcost_sides(inv_d, wside(c, x0 + j), xs, lamf) : inf;
    __syncthreads();
    if (warp == 0) {
      const float* wd = tdiag;
      float prev = xin ? G[pst + x] : inf;  // layer i - 1 at this column
      for (int i = 2; i <= S; ++i) {
        float b = inf;
        for (int w = 0; w < nw; ++w) b = fminf(b, tpart[(static_cast<size_t>(w) * kS + (i - 2)) * kWT + lane]);
        for (int j = 0; j < kWT; ++j) {
          const float gj = __shfl_sync(0xffffffffu, prev, j);
          b = fminf(b, __fadd_rn(gj, wd[j * kWT + lane]));
        }
        if (xin) G[i * pst + x] = b;
        prev = b;
      }
    }
    __syncthreads();
  }
}

__device__ void approx_solve_wide(const WCtx& c, double lam, int refine, AOut* out) {
  const int p = c.p, S = c.S, tid = threadIdx.x, bd = blockDim.x;
  const float inf = __int_as_float(0x7f800000);
  const float lamf = static_cast<float>(lam);
  const int kS = wide_tile_layers(S);
  if (kS == 8) {
    wide_layers_tiled<8>(c, lamf);
  } else if (kS == 16) {
    wide_layers_tiled<16>(c, lamf);
  } else if (kS == 32) {
    wide_layers_tiled<32>(c, lamf);
  } else {
    for (int x = tid; x < p; x += bd) c.G[c.pst + x] = (x == 0) ? 0.0f : inf;
    __syncthreads();
    for (int i = 2; i <= S; ++i) {
      const float* __restrict__ Gp = c.G + (i - 1) * c.pst;
      float* __restrict__ Gc = c.G + i * c.pst;
      for (int x = i - 1 + tid; x < p; x += bd) {
        float best = inf;
        for (int a = i - 2; a < x; ++a) best = fminf(best, __fadd_rn(Gp[a], wcost(c, a, x, lamf)));
        Gc[x] = best;
      }
      __syncthreads();
    }
  }
  if (warp_id() == 0) {
    const int lane = lane_id();
    float bv = inf;
    int bi = 0x7fffffff;
    for (int i = 2 + lane; i <= S; i += kWarp) {
      const float g = c.G[i * c.pst + p - 1];
      if (g < bv) {
        bv = g;
        bi = i;
      }
    }
    warp_argmin(bv, bi);
    if (lane == 0) {
      c.sQ[0] = 0;
      c.sQ[1] = p - 1;  // no finite candidate (non-finite inputs): {P_0, P_{p-1}}
      if (bi != 0x7fffffff) c.sQ[bi - 1] = p - 1;
      *c.msh = (bi == 0x7fffffff) ? -2 : bi;
    }
  }
  __syncthreads();
  // Recovery, all threads: at layer i the value before c_i = x is the smallest
  // a < x whose sum G_{i-1}(a) + w(a, x) equals G_i(x) (the minimum is one of
  // the sums, recomputed with the same operations).
  const int mr = *c.msh;
  if (mr > 0) {
    int x = p - 1;
    for (int i = mr; i >= 2; --i) {
      const float target = c.G[i * c.pst + x];
      const float* Gp = c.G + (i - 1) * c.pst;
      if (tid == 0) *c.found = 0x7fffffff;
      __syncthreads();
      const WSide xs = wside(c, x);
      for (int a = i - 2 + tid; a < x; a += bd) {
        if (__fadd_rn(Gp[a], wcost_sides(c.inv_d, wside(c, a), xs, lamf)) == target) {
          atomicMin(c.found, a);
          break;
        }
      }
      __syncthreads();
      const int f = *c.found;
      x = (f == 0x7fffffff) ? i - 2 : f;  // not reached: the minimum is one of the sums
      if (tid == 0) c.sQ[i - 2] = x;
      __syncthreads();  // every thread has read found before it is reset
    }
  }
  __syncthreads();
  const int m = mr > 0 ? mr : 2;
  if (refine > 0) wrefine(c, lam, m, refine);
  if (warp_id() == 0) wevaluate(c, lam, refine > 0, m, out);
  __syncthreads();
}

__global__ void __launch_bounds__(kWideApproxThreads, 1) k_approx_wide(ApproxArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ AOut s_out;
  __shared__ int s_flag;
  __shared__ int s_misc[3];
  __shared__ double s_tot[6][kWideApproxThreads / kWarp];
  const int p = a.p, S = a.s, tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  constexpr int kNW = kWideApproxThreads / kWarp;
  WCtx c;
  c.p = p;
  c.S = S;
  c.pst = (p + 3) & ~3;
  c.dd = static_cast<double>(a.d);
  c.inv_d = 1.0 / c.dd;
  c.sQ = reinterpret_cast<int*>(smem);
  int* sQ1 = c.sQ + S;
  int* sQ2 = sQ1 + S;
  c.moved = &s_misc[0];
  c.msh = &s_misc[1];
  c.found = &s_misc[2];
  unsigned char* gs = a.scratch + static_cast<size_t>(blockIdx.x) * a.scratch_per_cta;
  auto take = [&gs](size_t bytes) {
    unsigned char* r = gs;
    gs += (bytes + 255) & ~size_t(255);
    return r;
  };
  c.pre = reinterpret_cast<double*>(take(sizeof(double) * 6 * static_cast<size_t>(p)));
  c.nb = reinterpret_cast<double*>(take(sizeof(double) * p));
  c.ab = reinterpret_cast<double*>(take(sizeof(double) * p));
  c.bb = reinterpret_cast<double*>(take(sizeof(double) * p));
  c.G = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(S + 1) * c.pst));
  c.fbuf = reinterpret_cast<double*>(take(sizeof(double) * static_cast<size_t>(kNW) * p));

  for (int r = blockIdx.x; r < a.n; r += gridDim.x) {
    const double* P = a.P + static_cast<int64_t>(r) * p;
    const int64_t bo = static_cast<int64_t>(r) * (p - 1);
    c.P = P;
    if (tid == 0) s_flag = a.in_status ? a.in_status[r] : 0;
    for (int k = tid; k < p - 1; k += kWideApproxThreads) {
      c.nb[k] = static_cast<double>(a.cnt[bo + k]);
      c.ab[k] = a.A[bo + k];
      c.bb[k] = a.B[bo + k];
    }
    __syncthreads();
    const bool degenerate = (P[0] == P[p - 1]);
    int bad = 0;
    if (!degenerate)
      for (int k = tid; k < p - 1; k += kWideApproxThreads) bad |= !(P[k] < P[k + 1]);
    bad = __syncthreads_or(bad);
    const int32_t st = s_flag != 0 ? s_flag : (bad ? kStatusArg : kStatusOk);
    if (st != kStatusOk || degenerate) {
      approx_fill_trivial(a, r, st);
      __syncthreads();
      continue;
    }
    // prefix sums: each thread scans a contiguous chunk of buckets, then the
    // chunk totals are scanned across the block
    {
      const int nbk = p - 1;
      const int chunk = (nbk + kWideApproxThreads - 1) / kWideApproxThreads;
      const int k0 = tid * chunk, k1 = min(k0 + chunk, nbk);
      const double P0 = P[0];
      double t[6] = {0, 0, 0, 0, 0, 0};
      for (int k = k0; k < k1; ++k) {
        const double u = P[k] - P0, n = c.nb[k], A = c.ab[k];
        t[0] += n;
        t[1] += A;
        t[2] += c.bb[k];
        t[3] += n * u;
        t[4] += A * u;
        t[5] += n * u * u;
      }
      double inc[6];
#pragma unroll
      for (int j = 0; j < 6; ++j) {
        double v = t[j];
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += y;
        }
        inc[j] = v;
        if (lane == kWarp - 1) s_tot[j][warp] = v;
      }
      __syncthreads();
      if (warp == 0) {
#pragma unroll
        for (int j = 0; j < 6; ++j) {
          double v = lane < kNW ? s_tot[j][lane] : 0.0;
#pragma unroll
          for (int o = 1; o < kWarp; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
          }
          if (lane < kNW) s_tot[j][lane] = v;  // inclusive over warps
        }
      }
      __syncthreads();
      double run[6];
#pragma unroll
      for (int j = 0; j < 6; ++j) run[j] = (inc[j] - t[j]) + (warp > 0 ? s_tot[j][warp - 1] : 0.0);
      if (tid == 0)
        for (int j = 0; j < 6; ++j) c.pre[j * p] = 0.0;
      for (int k = k0; k < k1; ++k) {
        const double u = P[k] - P0, n = c.nb[k], A = c.ab[k];
        run[0] += n;
        run[1] += A;
        run[2] += c.bb[k];
        run[3] += n * u;
        run[4] += A * u;
        run[5] += n * u * u;
#pragma unroll
        for (int j = 0; j < 6; ++j) c.pre[j * p + k + 1] = run[j];
      }
    }
    __syncthreads();
    approx_drive(a, r, c.sQ, sQ1, sQ2, S, (P[p - 1] - P[0]) * (P[p - 1] - P[0]), s_out,
                 [&](double lam) { approx_solve_wide(c, lam, a.refine, &s_out); });
    __syncthreads();
  }
}

template <typename T, bool kSmem, bool kSplit>
void* approx_kernel_ptr() {
  return reinterpret_cast<void*>(&k_approx<T, kSmem, kSplit>);
}

template <typename T, bool kSmem>
void* approx_fn_split(bool split) {
  return split ? approx_kernel_ptr<T, kSmem, true>() : approx_kernel_ptr<T, kSmem, false>();
}

void* approx_fn(bool fp64, bool smem, bool split) {
  return fp64 ? (smem ? approx_fn_split<double, true>(split) : approx_fn_split<double, false>(split))
              : (smem ? approx_fn_split<float, true>(split) : approx_fn_split<float, false>(split));
}

size_t al16(size_t b) { return (b + 15) & ~size_t(15); }
size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

bool approx_plan(int n, int p, int s, bool fp64, ApproxPlan* plan) {
  if (p < 2 || p > kMaxPWide || s < 2 || n < 1) return false;
  const int S = s < p ? s : p;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int sms = 0, optin = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  plan->wide = p > kMaxP;
  if (plan->wide) {
    // large alphabets: fp32 layers only, one CTA per SM, O(p) slab per CTA
    if (fp64) return false;
    const size_t pst = static_cast<size_t>((p + 3) & ~3);
    plan->fp64 = false;
    plan->smem = false;
    plan->split = false;
    plan->threads = kWideApproxThreads;
    plan->smem_bytes = wide_smem_bytes(S);
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(&k_approx_wide),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(plan->smem_bytes)) !=
        cudaSuccess)
      return false;
    plan->scratch_per_cta = al256(8 * 6 * static_cast<size_t>(p)) + 3 * al256(8 * static_cast<size_t>(p)) +
                            al256(4 * static_cast<size_t>(S + 1) * pst) +
                            al256(8 * static_cast<size_t>(kWideApproxThreads / kWarp) * p);
    plan->ctas = n < sms ? n : sms;
    return true;
  }
  const size_t tsz = fp64 ? 8 : 4;
  const int kvec = static_cast<int>(16 / tsz);
  int ncv = 0;
  for (int x = 0; x < p; ++x) ncv = next_column(ncv, x, kvec);
  const size_t vb = al256(16 * static_cast<size_t>(ncv));
  const size_t db = al256(8 * static_cast<size_t>(tri_size(p)));
  plan->fp64 = fp64;
  // Table pass 1 gives each thread one a: threads >= p - 1.
  plan->threads = p <= 128 ? 128 : (p <= 256 ? 256 : 512);
  const size_t fb = 8 * static_cast<size_t>(p) * (plan->threads / 32);
  const size_t cbytes = al256(vb > fb ? vb : fb);
  const int pst = (p + kvec - 1) / kvec * kvec;
  const size_t small = al16(8 * p) * 4 + al16(4 * S) * 3 + al16(4 * static_cast<size_t>(p + 1));
  const size_t big = cbytes + al16(tsz * static_cast<size_t>(S + 1) * pst);
  plan->smem = small + big + 1024 <= static_cast<size_t>(optin);
  plan->smem_bytes = small + (plan->smem ? big : 0);
  plan->scratch_per_cta = al256(2 * vb + 3 * db + (plan->smem ? 0 : big));
  // Split columns when no SM holds more than one vector: then a layer waits on
  // its longest column; with several CTAs per SM the others hide that wait and
  // the split's extra loads and barrier only cost.
  plan->split = n <= sms;
  void* fn = approx_fn(fp64, plan->smem, plan->split);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(plan->smem_bytes)) !=
      cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, plan->threads, plan->smem_bytes) != cudaSuccess ||
      per_sm < 1)
    return false;
  const int ctas = sms * per_sm;
  plan->ctas = n < ctas ? n : ctas;
  return true;
}

cudaError_t launch_approx(const ApproxPlan& plan, ApproxArgs args, cudaStream_t st) {
  void* kargs[] = {&args};
  void* fn = plan.wide ? reinterpret_cast<void*>(&k_approx_wide) : approx_fn(plan.fp64, plan.smem, plan.split);
  cudaError_t e = cudaLaunchKernel(fn, dim3(plan.ctas), dim3(plan.threads), kargs, plan.smem_bytes, st);
  note_launch();
  return e;
}

int64_t approx_pair_layers(int p, int s) {
  const int S = s < p ? s : p;
  int64_t t = 0;
  for (int i = 2; i <= S; ++i)
    for (int x = i - 1; x <= p - 1; ++x) t += x - (i - 2);
  return t;
}

}  // namespace ecasq
