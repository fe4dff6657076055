// The exact ECASQ dynamic programme on B200.
//
// ECASQ summary (gist.science/pt/paper/2608.18147):
//   §2.1 "Relaxação Lagrangiana": minimise MSE(Q,X) + lambda * H(X^).
//   §2.2 "Programação Dinâmica Ótima": the ASQ DP does not extend because the
//        entropy term of a value depends on both neighbours, so the state is a
//        PAIR of consecutive values, dp_OPT(i, l, j); the direct programme costs
//        O(d^3 s) time over the entries, O(p^3 s) over a permissible set P;
//        "Algoritmo de Hirschberg": divide and conquer that keeps only two DP
//        layers, O(d^2) (here O(p^2)) memory.
//
// Recurrence evaluated here (i = number of values up to and including P_l,
// counting c_1 = P_0; m = mu/d the normalised mass of a value):
//   F_1(0, j) = V(0,j)/(lambda d) + h(L(0,j)/d)
//   F_i(l, j) = V(l,j)/(lambda d) + min_{k} [ F_{i-1}(k,l) + h((R(k,l) + L(l,j))/d) ]
//   J*/lambda = min_{i,k} F_i(k, p-1) + h(R(k,p-1)/d),   h(m) = -m log2 m.
// The whole programme is scaled by 1/lambda, so one (k,l,j) triple is one add,
// one MUFU log2 and one FMA plus the running minimum. lambda = 0 is the
// separable MSE-only programme (the minimum over k no longer depends on j).
//
// Design (this file):
//   * one CTA per vector, persistent over every solve of that vector (all
//     lambdas, or the whole bisection), so the pair tables are built once;
//     with the tables in the global slab and at most one vector per two SMs,
//     a cluster of two CTAs shares each vector: they split every layer's tasks
//     through one counter in rank 0's shared memory and synchronise at cluster
//     barriers;
//   * the tables and the two live DP layers sit in shared memory when they fit
//     (fp32, p <= 128) and in a per-CTA global (L2-resident) slab otherwise;
//   * a DP layer is split into tasks of 32 lanes; a lane owns 4 outputs
//     (l, j0..j0+3) of one row and sweeps k down the column of l in two
//     interleaved streams; tasks are decoded in closed form from their index,
//     longest rows first, and taken by warps from a shared counter; with the
//     tables in the global slab a warp prefetches its next task's column and
//     rows into L2 while it runs the current one;
//   * store mode keeps every layer's values in a per-CTA global slab (no
//     back-pointers); the backtrack recomputes the argmin of the few states on
//     the optimal path;
//     Hirschberg mode keeps none: a forward pass finds the optimum and its last
//     pair, then the code is recovered by divide and conquer, joining a forward
//     pass over the left part with a pass over the reflected alphabet
//     (P'_k = -P_{p-1-k}) for the right part;
//   * the fp64 evaluation of the chosen code and the bisection run in the same
//     kernel.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / kWarp;
constexpr int kTJ = 4;  // outputs (l, j0 .. j0+3) per lane
constexpr int kNQ = 2;  // interleaved k-streams per output (kTJ * kNQ independent min chains per lane)

template <typename T>
struct Arith;

template <>
struct Arith<float> {
  // Added to every mass so that log2 never sees 0 inside the sweep:
  // h(2^-100) ~ 8e-29, far below fp32 resolution of any objective.
  static constexpr float kEps = 0x1p-100f;
  __device__ static float inf() { return __int_as_float(0x7f800000); }
  __device__ static float nlog(float m) { return -m * lg2_approx(m); }
  __device__ static float fold(float g, float m) { return fmaf(-m, lg2_approx(m), g); }
  __device__ static float vmin(float a, float b) { return fminf(a, b); }
};

template <>
struct Arith<double> {
  static constexpr double kEps = 0.0;
  __device__ static double inf() { return __longlong_as_double(0x7ff0000000000000ll); }
  __device__ static double nlog(double m) { return m > 0.0 ? -m * log2(m) : 0.0; }
  __device__ static double fold(double g, double m) { return m > 0.0 ? fma(-m, log2(m), g) : g; }
  __device__ static double vmin(double a, double b) { return fmin(a, b); }
};

// Barrier of the CTAs that share a vector: the block itself, or the whole
// thread-block cluster (release/acquire at cluster scope, so the layer values
// the other CTAs wrote to the global slab are visible after it).
template <int kCL>
__device__ __forceinline__ void csync() {
  if constexpr (kCL > 1)
    cooperative_groups::this_cluster().sync();
  else
    __syncthreads();
}

// One entry of a live DP layer: the layer value G = F(k, l) and a = R(k, l)/d
// (+ eps) side by side, so one 8- (16-) byte shared load feeds a whole k step.
// a is written once per vector into both ping-pong layers.
template <typename T>
struct alignas(2 * sizeof(T)) GA {
  T g, a;
};

// Layouts. The live DP layers (with a) are stored by COLUMN: entry (k, l),
// k < l, sits at cb[l] + k, so a lane sweeping k for its row l walks
// consecutive addresses (one pointer, immediate offsets). Column starts are
// padded so that cb[l] = l (mod 16): lanes that hold 16 consecutive rows l
// then read 16 distinct 8-byte bank pairs at every k. b = L/d and V/d are read
// once per output and stay in the row-triangle layout (row_off(l) + j - l - 1).
__host__ __device__ inline int next_colbase(int prev_base, int prev_col) {
  int c = prev_base + prev_col;  // column prev_col holds prev_col entries
  const int want = (prev_col + 1) & 15;
  c += (want - (c & 15) + 16) & 15;
  return c;
}
__host__ __device__ inline int layer_elems(int p) {
  int c = 0;
  for (int l = 0; l < p; ++l) c = next_colbase(c, l);
  return c;
}

// Groups of kTJ outputs of a layer, counted from the last row upward (rows
// e0-1, e0-2, ...; a row with n outputs holds ceil(n/4) groups). The rows with
// 1 .. n outputs hold G(n) = 2m(m+1) + r(m+1) groups, n = 4m + r; a group index
// inverts G with one square root.
__host__ __device__ inline int groups_upto(int n) {
  const int m = n >> 2, r = n & 3;
  return 2 * m * (m + 1) + r * (m + 1);
}
__device__ inline void decode_group(int q, int e0, int& l, int& j0, int& nv) {
  int n = static_cast<int>(sqrtf(8.f * q + 4.f) - 2.f);
  n = n < 1 ? 1 : n;
  while (groups_upto(n) <= q) ++n;
  while (n > 1 && groups_upto(n - 1) > q) --n;
  l = e0 - n;
  j0 = l + 1 + kTJ * (q - groups_upto(n - 1));
  nv = min(kTJ, e0 - j0 + 1);
}

// The tables a pass reads: two ping-pong layer buffers (with a) and b, V/d.
template <typename T>
struct Tables {
  GA<T>* buf0;
  GA<T>* buf1;
  T* rowB;
  T* rowV;
  __device__ __forceinline__ GA<T>* layer(int t) const { return (t & 1) ? buf1 : buf0; }
};

template <typename T>
struct Ctx {
  int p, S, tri;
  double dd;
  Tables<T> fw;  // the alphabet as given
  Tables<T> rf;  // the reflected alphabet (Hirschberg mode)
  const int* cb;              // [p+1] padded column starts (shared memory)
  T* fst;                     // [S][tri] layer values F_i(l, j) (store mode; row triangle)
  double *sP, *sN, *sA, *sB;  // [p] alphabet and bucket statistics
  double *sR, *sL;            // [S] evaluation scratch
  T* rmin;                    // [p] row minima (lambda = 0)
  int* rarg;                  // [p]
  int* ctr;                   // [S] task counters (rank 0's, in a cluster)
  int* sQ;                    // [S] code of the last solve
  int* stk;                   // [2S] Hirschberg segment stack
  bool hirschberg;
};

struct SolveOut {
  double mse, H, J;
  int m;
  int bestI, bestK;
  int jx, jy;  // Hirschberg join result
  int nstk;
};

// ---- tables --------------------------------------------------------------------
// For every pair a < c, sums over the buckets a .. c-1 (ascending), with
// delta_k = P_k - P_a:  N = sum n_k, T1 = sum (A_k + n_k delta_k),
// T2 = sum (B_k + 2 delta_k A_k + n_k delta_k^2); W = P_c - P_a;
// V = W T1 - T2 (>= 0), R = T1 / W, L = N - R. One thread per a, running in c.
template <typename T>
__device__ __forceinline__ void build_tables(const Ctx<T>& c) {
  const int p = c.p;
  for (int a = threadIdx.x; a < p - 1; a += blockDim.x) {
    double N = 0.0, T1 = 0.0, T2 = 0.0;
    const double Pa = c.sP[a];
    const int ro = row_off(a, p) - a - 1;
    for (int cc = a + 1; cc < p; ++cc) {
      const int k = cc - 1;
      const double dk = c.sP[k] - Pa;
      const double nk = c.sN[k];
      N += nk;
      T1 += c.sA[k] + nk * dk;
      T2 += c.sB[k] + 2.0 * dk * c.sA[k] + nk * dk * dk;
      const double W = c.sP[cc] - Pa;
      double V = W * T1 - T2;
      V = V > 0.0 ? V : 0.0;
      const double R = T1 / W;
      double L = N - R;
      L = L > 0.0 ? L : 0.0;
      const T av = static_cast<T>(R / c.dd) + Arith<T>::kEps;
      c.fw.buf0[c.cb[cc] + a].a = av;
      c.fw.buf1[c.cb[cc] + a].a = av;
      c.fw.rowB[ro + cc] = static_cast<T>(L / c.dd);
      c.fw.rowV[ro + cc] = static_cast<T>(V / c.dd);
    }
  }
}

// Reflected tables, from the forward ones: with r(x) = p-1-x,
//   R'(k', l') = L(r(l'), r(k')),  L'(l', j') = R(r(j'), r(l')),  V'(l', j') = V(r(j'), r(l')).
template <typename T>
__device__ __forceinline__ void build_reflected(const Ctx<T>& c) {
  const int p = c.p;
  for (int l = 1 + threadIdx.x / kWarp; l < p; l += blockDim.x / kWarp) {
    for (int k = lane_id(); k < l; k += kWarp) {
      const int rl = p - 1 - l, rk = p - 1 - k;  // rl < rk
      const T av = c.fw.rowB[row_off(rl, p) + rk - rl - 1] + Arith<T>::kEps;
      c.rf.buf0[c.cb[l] + k].a = av;
      c.rf.buf1[c.cb[l] + k].a = av;
      // (k, l) as a row pair of the reflected problem: row k, column l.
      const int e = row_off(k, p) + l - k - 1;
      const int rl2 = p - 1 - l, rk2 = p - 1 - k;  // original interval [rl2, rk2]
      c.rf.rowB[e] = c.fw.buf0[c.cb[rk2] + rl2].a;
      c.rf.rowV[e] = c.fw.rowV[row_off(rl2, p) + rk2 - rl2 - 1];
    }
  }
}

// ---- one pass of DP layers ------------------------------------------------------
// Layers 1 .. T over the values s0 .. e0: layer t holds F_t(l, j), the best cost
// of t values from s0 up to l, followed by j. Layer 1 is row s0 alone; its
// value's mass adds `extra` (the share from a fixed left neighbour; < 0 when
// s0 has none). With last_only the last layer is computed for j = e0 only.
struct Pass {
  int s0, e0, T;
  bool last_only;
  double extra;
  bool store_f;  // keep every layer's values for the backtrack
  bool finalize;
};

template <typename T>
__device__ __forceinline__ void finalize_layer(const Ctx<T>& c, const Tables<T>& tb, int i, int s0, int e0,
                                               const GA<T>* G, bool sep, T* bestE, int* bestI, int* bestK) {
  // Best (E, i, k) over the finished layer i: E = F_i(k, e0) + h(R(k, e0)/d).
  // Warp 0 only. Strict '<' over layers in ascending order keeps the smaller code.
  const int kb = (i == 1) ? s0 : s0 + i - 1;
  const int ke = (i == 1) ? s0 : e0 - 1;
  T best = Arith<T>::inf();
  int arg = 0x7fffffff;
  const GA<T>* col = G + c.cb[e0];
  for (int k = kb + lane_id(); k <= ke; k += kWarp) {
    const GA<T> ga = col[k];
    T e = ga.g;
    if (!sep) e += Arith<T>::nlog(ga.a);
    if (e < best) {
      best = e;
      arg = k;
    }
  }
  warp_argmin(best, arg);
  if (lane_id() == 0 && best < *bestE) {
    *bestE = best;
    *bestI = i;
    *bestK = arg;
  }
  (void)tb;
}

// One task of a layer: 32 groups, one per lane. The lane owns the outputs
// (l, j0 .. j0+nv-1) and sweeps k = kmin .. l-1 down its column in kNQ
// interleaved streams (each output and stream keeps its own running minimum,
// so consecutive updates do not wait on one another). The k range common to
// the warp runs unpredicated; the rest masks the layer value to +inf past the
// lane's own column. Only the minimum is kept: the backtrack recomputes the
// argmin of the few states on the optimal path from the stored layers (fsi).
template <typename T, int kUnroll>
__device__ __forceinline__ void run_task(const Ctx<T>& c, const Tables<T>& tb, int l, int j0, int nv, bool active,
                                         int kmin, const GA<T>* __restrict__ Gp, GA<T>* __restrict__ Gc,
                                         T* __restrict__ fsi, T invl) {
  const int p = c.p;
  if (!active) {
    l = kmin + 1;  // inactive lanes sweep an in-range column and write nothing
    nv = 0;
  }
  const int lmin = __reduce_min_sync(0xffffffffu, active ? l : 0x7fffffff);
  const int lmax = __reduce_max_sync(0xffffffffu, active ? l : 0);
  const int ro = row_off(l, p) - l - 1;
  T b[kTJ];
#pragma unroll
  for (int u = 0; u < kTJ; ++u) b[u] = (u < nv) ? tb.rowB[ro + j0 + u] : T(0);
  const GA<T>* __restrict__ col = Gp + c.cb[l];

  T best[kTJ][kNQ];
#pragma unroll
  for (int u = 0; u < kTJ; ++u)
#pragma unroll
    for (int s = 0; s < kNQ; ++s) best[u][s] = Arith<T>::inf();
  int k = kmin;
#pragma unroll kUnroll
  for (; k + kNQ <= lmin; k += kNQ) {
#pragma unroll
    for (int s = 0; s < kNQ; ++s) {
      const GA<T> ga = col[k + s];
#pragma unroll
      for (int u = 0; u < kTJ; ++u) best[u][s] = Arith<T>::vmin(best[u][s], Arith<T>::fold(ga.g, ga.a + b[u]));
    }
  }
#pragma unroll 1
  for (; k < lmax; ++k) {
    GA<T> ga = col[k];
    ga.g = (k < l) ? ga.g : Arith<T>::inf();
#pragma unroll
    for (int u = 0; u < kTJ; ++u) best[u][0] = Arith<T>::vmin(best[u][0], Arith<T>::fold(ga.g, ga.a + b[u]));
  }
#pragma unroll
  for (int u = 0; u < kTJ; ++u) {
    T bu = best[u][0];
#pragma unroll
    for (int s = 1; s < kNQ; ++s) bu = Arith<T>::vmin(bu, best[u][s]);
    if (u < nv) {
      const int e = ro + j0 + u;
      const T f = tb.rowV[e] * invl + bu;
      Gc[c.cb[j0 + u] + l].g = f;
      if (fsi) fsi[e] = f;
    }
  }
}

// Prefetch of a task's column of the previous layer (128-byte lines) and of
// the b and V/d rows its outputs read (tables in the global slab).
template <typename T>
__device__ __forceinline__ void prefetch_task(const Ctx<T>& c, const Tables<T>& tb, int l, int j0, int kmin,
                                              const GA<T>* Gp) {
  const uintptr_t beg = reinterpret_cast<uintptr_t>(Gp + c.cb[l] + kmin) & ~uintptr_t(127);
  const uintptr_t end = reinterpret_cast<uintptr_t>(Gp + c.cb[l] + l);
  for (uintptr_t a = beg; a < end; a += 128) asm volatile("prefetch.L2 [%0];" ::"l"(a));
  const int ro = row_off(l, c.p) - l - 1;
  asm volatile("prefetch.L2 [%0];" ::"l"(tb.rowB + ro + j0));
  asm volatile("prefetch.L2 [%0];" ::"l"(tb.rowV + ro + j0));
}

// Runs the pass; all threads. Leaves layer T in tb.layer(T).
// With a cluster, the CTAs split each layer's tasks (one counter, in rank 0)
// and compute everything else redundantly from the same data. With the tables
// in the global slab (kSlab), a warp decodes its next task before running the
// current one and prefetches that task's column and rows into L2.
template <typename T, int kUnroll, int kCL, bool kSlab>
__device__ __forceinline__ void run_pass(const Ctx<T>& c, const Tables<T>& tb, const Pass& ps, bool sep, T invl,
                                         SolveOut* out, T* bestE) {
  const int p = c.p, tri = c.tri;
  const int s0 = ps.s0, e0 = ps.e0;
  const int tid = threadIdx.x;
  const int warp = warp_id(), lane = lane_id();
  if constexpr (kCL > 1) {
    csync<kCL>();  // the other CTAs have finished reading what this pass rewrites
    if (cooperative_groups::this_cluster().block_rank() == 0)
      for (int t = tid; t < c.S; t += blockDim.x) c.ctr[t] = 0;
  } else {
    for (int t = tid; t < c.S; t += blockDim.x) c.ctr[t] = 0;
  }
  {  // layer 1: row s0
    GA<T>* G1 = tb.layer(1);
    const T extra = ps.extra > 0.0 ? static_cast<T>(ps.extra) : T(0);
    const int ro = row_off(s0, p) - s0 - 1;
    const int jb = (ps.T == 1 && ps.last_only) ? e0 : s0 + 1;
    for (int j = jb + tid; j <= e0; j += blockDim.x) {
      const int e = ro + j;
      T f = tb.rowV[e] * invl;
      if (!sep) f += Arith<T>::nlog(tb.rowB[e] + extra + Arith<T>::kEps);
      G1[c.cb[j] + s0].g = f;
    }
  }
  csync<kCL>();
  for (int t = 2; t <= ps.T; ++t) {
    const GA<T>* Gp = tb.layer(t - 1);
    GA<T>* Gc = tb.layer(t);
    T* fsi = ps.store_f ? c.fst + static_cast<size_t>(t) * tri : nullptr;
    const bool last = ps.last_only && t == ps.T;
    const int r0 = s0 + t - 1;  // first row of the layer
    if (ps.finalize && warp == 0) finalize_layer(c, tb, t - 1, s0, e0, Gp, sep, bestE, &out->bestI, &out->bestK);
    if (t == 2) {
      // Only k = s0 precedes the second value.
      for (int l = r0 + warp; l <= e0 - 1; l += kWarps) {
        const GA<T> ga = Gp[c.cb[l] + s0];  // (s0, l)
        const int ro = row_off(l, p) - l - 1;
        for (int j = (last ? e0 : l + 1) + lane; j <= e0; j += kWarp) {
          const int e = ro + j;
          const T v = sep ? ga.g : Arith<T>::fold(ga.g, ga.a + tb.rowB[e]);
          const T f = tb.rowV[e] * invl + v;
          Gc[c.cb[j] + l].g = f;
          if (fsi) fsi[e] = f;
        }
      }
    } else if (sep) {
      const int kmin = s0 + t - 2;
      for (int l = r0 + warp; l <= e0 - 1; l += kWarps) {
        T best = Arith<T>::inf();
        int arg = kmin;
        for (int k = kmin + lane; k < l; k += kWarp) {
          const T v = Gp[c.cb[l] + k].g;
          if (v < best) {
            best = v;
            arg = k;
          }
        }
        warp_argmin(best, arg);
        if (lane == 0) {
          c.rmin[l] = best;
          c.rarg[l] = arg;
        }
      }
      __syncthreads();
      for (int l = r0 + warp; l <= e0 - 1; l += kWarps) {
        const int ro = row_off(l, p) - l - 1;
        const T rm = c.rmin[l];
        for (int j = (last ? e0 : l + 1) + lane; j <= e0; j += kWarp) {
          const int e = ro + j;
          const T f = tb.rowV[e] + rm;
          Gc[c.cb[j] + l].g = f;
          if (fsi) fsi[e] = f;
        }
      }
    } else if (r0 <= e0 - 1) {
      const int kmin = s0 + t - 2;
      const int ng = last ? (e0 - r0) : groups_upto(e0 - r0);
      const int nt = (ng + kWarp - 1) / kWarp;
      // Tasks in index order are the longest rows first. The next task index
      // is fetched before the current task runs.
      if constexpr (kSlab) {
        auto decode = [&](int tk, int& l, int& j0, int& nv) {
          const int q = tk * kWarp + lane;
          l = 0;
          j0 = 0;
          nv = 0;
          if (q < ng) {
            if (last) {
              l = e0 - 1 - q;
              j0 = e0;
              nv = 1;
            } else {
              decode_group(q, e0, l, j0, nv);
            }
          }
        };
        int tn = 0;
        if (lane == 0) tn = atomicAdd(c.ctr + t, 1);
        tn = __shfl_sync(0xffffffffu, tn, 0);
        int nl = 0, nj0 = 0, nnv = 0;
        if (tn < nt) {
          decode(tn, nl, nj0, nnv);
          if (nnv > 0) prefetch_task(c, tb, nl, nj0, kmin, Gp);
        }
        while (tn < nt) {
          const int l = nl, j0 = nj0, nv = nnv;
          if (lane == 0) tn = atomicAdd(c.ctr + t, 1);
          tn = __shfl_sync(0xffffffffu, tn, 0);
          if (tn < nt) {
            decode(tn, nl, nj0, nnv);
            if (nnv > 0) prefetch_task(c, tb, nl, nj0, kmin, Gp);
          }
          run_task<T, kUnroll>(c, tb, l, j0, nv, nv > 0, kmin, Gp, Gc, fsi, invl);
        }
      } else {
        int tn = 0;
        if (lane == 0) tn = atomicAdd(c.ctr + t, 1);
        tn = __shfl_sync(0xffffffffu, tn, 0);
        while (tn < nt) {
          const int tk = tn;
          if (lane == 0) tn = atomicAdd(c.ctr + t, 1);
          tn = __shfl_sync(0xffffffffu, tn, 0);
          const int q = tk * kWarp + lane;
          const bool act = q < ng;
          int l = 0, j0 = 0, nv = 0;
          if (act) {
            if (last) {
              l = e0 - 1 - q;
              j0 = e0;
              nv = 1;
            } else {
              decode_group(q, e0, l, j0, nv);
            }
          }
          run_task<T, kUnroll>(c, tb, l, j0, nv, act, kmin, Gp, Gc, fsi, invl);
        }
      }
    }
    csync<kCL>();
  }
  if (ps.finalize && warp == 0)
    finalize_layer(c, tb, ps.T, s0, e0, tb.layer(ps.T), sep, bestE, &out->bestI, &out->bestK);
  __syncthreads();
}

// Hirschberg join: the split pair (x, y) minimising
//   F(x, y) + F'(r(y), r(x)) - V(x, y)/(lambda d)
// over x in [xlo, xhi], y in [x+1, yhi] (y = yhi only when fixed); ties go to
// the smaller x, then the smaller y. All threads; result in out->jx, out->jy.
template <typename T>
__device__ __forceinline__ void join(const Ctx<T>& c, const GA<T>* Ff, const GA<T>* Fb, int xlo, int xhi, int yhi,
                                     bool yfixed, T invl, SolveOut* out, T* wbest, int* warg) {
  const int p = c.p;
  const int warp = warp_id(), lane = lane_id();
  T best = Arith<T>::inf();
  int arg = 0x7fffffff;
  for (int x = xlo + warp; x <= xhi; x += kWarps) {
    const int ro = row_off(x, p) - x - 1;
    const int rx = p - 1 - x;
    for (int y = (yfixed ? yhi : x + 1) + lane; y <= yhi; y += kWarp) {
      const T v = Ff[c.cb[y] + x].g + Fb[c.cb[rx] + (p - 1 - y)].g - c.fw.rowV[ro + y] * invl;
      const int id = x * p + y;
      if (v < best || (v == best && id < arg)) {
        best = v;
        arg = id;
      }
    }
  }
  warp_argmin(best, arg);
  if (lane == 0) {
    wbest[warp] = best;
    warg[warp] = arg;
  }
  __syncthreads();
  if (warp == 0) {
    best = lane < kWarps ? wbest[lane] : Arith<T>::inf();
    arg = lane < kWarps ? warg[lane] : 0x7fffffff;
    warp_argmin(best, arg);
    if (lane == 0) {
      if (arg == 0x7fffffff) arg = xlo * p + (yfixed ? yhi : xlo + 1);  // non-finite values only
      out->jx = arg / p;
      out->jy = arg % p;
    }
  }
  __syncthreads();
}

// fp64 evaluation of the code in c.sQ from the bucket statistics (warp 0).
template <typename T>
__device__ __forceinline__ void evaluate(const Ctx<T>& c, double lam, SolveOut* out) {
  if (warp_id() != 0) return;
  const int lane = lane_id();
  const int m = out->m;
  double vs = 0.0;
  for (int t = lane; t < m - 1; t += kWarp) {
    const int a = c.sQ[t], cc = c.sQ[t + 1];
    double N = 0.0, T1 = 0.0, T2 = 0.0;
    const double Pa = c.sP[a];
    for (int k = a; k < cc; ++k) {
      const double dk = c.sP[k] - Pa;
      const double nk = c.sN[k];
      N += nk;
      T1 += c.sA[k] + nk * dk;
      T2 += c.sB[k] + 2.0 * dk * c.sA[k] + nk * dk * dk;
    }
    const double W = c.sP[cc] - Pa;
    double V = W * T1 - T2;
    V = V > 0.0 ? V : 0.0;
    const double R = T1 / W;
    c.sR[t] = R;
    c.sL[t] = N - R;
    vs += V;
  }
  __syncwarp();
  double hs = 0.0;
  for (int t = lane; t < m; t += kWarp) {
    const double mu = (t > 0 ? c.sR[t - 1] : 0.0) + (t < m - 1 ? c.sL[t] : 0.0);
    if (mu > 0.0) {
      const double q = mu / c.dd;
      hs -= q * log2(q);
    }
  }
  vs = warp_sum(vs);
  hs = warp_sum(hs);
  if (lane == 0) {
    out->mse = vs / c.dd;
    out->H = hs;
    out->J = out->mse + lam * hs;
  }
}

// One full solve at lambda (all threads). Leaves the code in c.sQ and the fp64
// evaluation in *out (shared).
template <typename T, int kUnroll, int kCL, bool kSlab>
__device__ __forceinline__ void solve(const Ctx<T>& c, double lam, SolveOut* out, T* bestE, T* wbest, int* warg) {
  const int p = c.p, S = c.S, tri = c.tri;
  // Below kMinLambda the entropy terms vanish under the precision of T and
  // 1/lambda would overflow it: the layers then run the MSE-only programme
  // (the code is still evaluated in fp64 at the true lambda).
  const double kMinLambda = sizeof(T) == 4 ? 1e-30 : 1e-290;
  const bool sep = !(lam > kMinLambda);
  const T invl = sep ? T(1) : static_cast<T>(1.0 / lam);
  const int tid = threadIdx.x;

  if (tid == 0) {
    *bestE = Arith<T>::inf();
    out->bestI = -1;
    out->bestK = -1;
  }
  __syncthreads();
  // The whole alphabet, from c_1 = P_0; the last layer needs only j = p-1.
  Pass full{0, p - 1, S - 1, true, -1.0, !c.hirschberg, true};
  run_pass<T, kUnroll, kCL, kSlab>(c, c.fw, full, sep, invl, out, bestE);

  if (tid == 0 && out->bestI < 1) {  // no finite candidate (non-finite inputs): fall back to {P_0, P_{p-1}}
    out->bestI = 1;
    out->bestK = 0;
  }
  __syncthreads();
  const int bi = out->bestI;
  if (tid == 0) {
    c.sQ[bi] = p - 1;
    c.sQ[bi - 1] = out->bestK;
    c.sQ[0] = 0;
    out->m = bi + 1;
    out->nstk = 0;
    if (c.hirschberg && bi + 1 - 3 >= 1) {
      // Segments (lo, hi): c[lo] (with c[lo-1] when lo >= 1) and the pair
      // (c[hi], c[hi+1]) are known; c[lo+1 .. hi-1] are not.
      c.stk[0] = 0;
      c.stk[1] = bi - 1;
      out->nstk = 1;
    }
  }
  if (!c.hirschberg && warp_id() == 0) {
    // Backtrack from (c_bi, c_{bi+1}) = (bestK, p-1): at layer ii the value
    // before c_ii is the smallest k reaching min_k fold(F_{ii-1}(k, c_ii),
    // R(k, c_ii)/d + L(c_ii, c_{ii+1})/d) (sep: min_k F_{ii-1}(k, c_ii)),
    // recomputed with the operations of the layer sweep; layer 2 has k = 0.
    const int lane = lane_id();
    int l = out->bestK, j = p - 1;
    for (int ii = bi; ii >= 2; --ii) {
      int kk = 0;
      if (ii > 2) {
        const T bb = c.fw.rowB[row_off(l, p) + j - l - 1];
        const T* Fp = c.fst + static_cast<size_t>(ii - 1) * tri;
        T best = Arith<T>::inf();
        int arg = 0x7fffffff;
        for (int k = ii - 2 + lane; k < l; k += kWarp) {
          const T g = Fp[row_off(k, p) + l - k - 1];
          const T v = sep ? g : Arith<T>::fold(g, c.fw.buf0[c.cb[l] + k].a + bb);
          if (v < best) {
            best = v;
            arg = k;
          }
        }
        warp_argmin(best, arg);
        kk = (arg == 0x7fffffff) ? ii - 2 : arg;  // all +inf only for non-finite inputs
      }
      if (lane == 0) c.sQ[ii - 2] = kk;
      j = l;
      l = kk;
    }
  }
  __syncthreads();

  while (c.hirschberg && out->nstk > 0) {
    const int top = out->nstk - 1;
    const int lo = c.stk[2 * top], hi = c.stk[2 * top + 1];
    __syncthreads();
    if (tid == 0) out->nstk = top;
    const int n = hi - lo - 1;          // unknown values c[lo+1 .. hi-1]
    const int mid = lo + (n + 1) / 2;   // split pair (c[mid], c[mid+1]); c[mid] unknown
    const int qlo = c.sQ[lo], qhi = c.sQ[hi], qnext = c.sQ[hi + 1];
    // Forward: values c[lo] .. c[mid], next c[mid+1], all <= c[hi].
    double extra_f = -1.0;
    if (lo >= 1) extra_f = static_cast<double>(c.fw.buf0[c.cb[qlo] + c.sQ[lo - 1]].a);  // R(c[lo-1], c[lo])/d
    Pass fwp{qlo, qhi, mid - lo + 1, mid + 1 == hi, extra_f, false, false};
    run_pass<T, kUnroll, kCL, kSlab>(c, c.fw, fwp, sep, invl, out, bestE);
    // Reflected: values c[hi] .. c[mid+1] (reflected), next c[mid]; the mass of
    // c[hi] takes L(c[hi], c[hi+1]) from its right neighbour.
    const double extra_b = static_cast<double>(c.fw.rowB[row_off(qhi, p) + qnext - qhi - 1]);
    Pass bwp{p - 1 - qhi, p - 1 - qlo, hi - mid, false, extra_b, false, false};
    run_pass<T, kUnroll, kCL, kSlab>(c, c.rf, bwp, sep, invl, out, bestE);
    const int xlo = qlo + (mid - lo), xhi = qhi - (hi - mid);
    const int yhi = qhi - (hi - mid - 1);
    join(c, c.fw.layer(fwp.T), c.rf.layer(bwp.T), xlo, xhi, yhi, mid + 1 == hi, invl, out, wbest, warg);
    if (tid == 0) {
      c.sQ[mid] = out->jx;
      c.sQ[mid + 1] = out->jy;
      int ns = out->nstk;
      if (mid - lo - 1 >= 1) {
        c.stk[2 * ns] = lo;
        c.stk[2 * ns + 1] = mid;
        ++ns;
      }
      if (hi - mid - 2 >= 1) {
        c.stk[2 * ns] = mid + 1;
        c.stk[2 * ns + 1] = hi;
        ++ns;
      }
      out->nstk = ns;
    }
    __syncthreads();
  }

  evaluate(c, lam, out);
  __syncthreads();
}

template <typename T, bool kSmemTables, int kCL>
__global__ void __launch_bounds__(kThreads, 1) k_dp(DpArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ SolveOut s_out;
  __shared__ T s_bestE;
  __shared__ int s_flag;
  __shared__ T s_wbest[kWarps];
  __shared__ int s_warg[kWarps];

  // k-loop unroll of the layer tasks: the tables in the global slab (L2) want
  // more loads in flight; the shared-memory variant has no registers to spare.
  constexpr int kUnrollK = kSmemTables ? 4 : 8;
  const int p = a.p, S = a.s;
  const int tri = tri_size(p);
  Ctx<T> c;
  c.p = p;
  c.S = S;
  c.tri = tri;
  c.dd = static_cast<double>(a.d);
  c.hirschberg = a.hirschberg != 0;

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
  c.sR = reinterpret_cast<double*>(carve(sizeof(double) * S));
  c.sL = reinterpret_cast<double*>(carve(sizeof(double) * S));
  c.rmin = reinterpret_cast<T*>(carve(sizeof(T) * p));
  c.rarg = reinterpret_cast<int*>(carve(sizeof(int) * p));
  c.ctr = reinterpret_cast<int*>(carve(sizeof(int) * S));
  c.sQ = reinterpret_cast<int*>(carve(sizeof(int) * S));
  int* sQ1 = reinterpret_cast<int*>(carve(sizeof(int) * S));
  int* sQ2 = reinterpret_cast<int*>(carve(sizeof(int) * S));
  c.stk = reinterpret_cast<int*>(carve(sizeof(int) * 2 * S));
  int* cbs = reinterpret_cast<int*>(carve(sizeof(int) * (p + 1)));
  if (threadIdx.x == 0) {
    int cc = 0;
    for (int l = 0; l < p; ++l) {
      cbs[l] = cc;
      cc = next_colbase(cc, l);
    }
    cbs[p] = cc;
  }
  c.cb = cbs;
  // CTAs of one cluster share a vector, its slab and rank 0's task counters.
  if constexpr (kCL > 1) c.ctr = cooperative_groups::this_cluster().map_shared_rank(c.ctr, 0);

  unsigned char* gs = a.scratch + static_cast<size_t>(blockIdx.x / kCL) * a.scratch_per_cta;
  c.fst = reinterpret_cast<T*>(gs);
  if (!c.hirschberg) gs += (sizeof(T) * static_cast<size_t>(S) * tri + 255) & ~size_t(255);
  const size_t tb = (sizeof(T) * static_cast<size_t>(tri) + 15) & ~size_t(15);
  const size_t gb = (2 * sizeof(T) * static_cast<size_t>(layer_elems(p)) + 15) & ~size_t(15);
  unsigned char* big = kSmemTables ? sp : gs;
  c.fw.buf0 = reinterpret_cast<GA<T>*>(big);
  c.fw.buf1 = reinterpret_cast<GA<T>*>(big + gb);
  c.fw.rowB = reinterpret_cast<T*>(big + 2 * gb);
  c.fw.rowV = reinterpret_cast<T*>(big + 2 * gb + tb);
  unsigned char* big2 = big + 2 * gb + 2 * tb;  // reflected tables (Hirschberg mode, global slab only)
  c.rf.buf0 = reinterpret_cast<GA<T>*>(big2);
  c.rf.buf1 = reinterpret_cast<GA<T>*>(big2 + gb);
  c.rf.rowB = reinterpret_cast<T*>(big2 + 2 * gb);
  c.rf.rowV = reinterpret_cast<T*>(big2 + 2 * gb + tb);
  __syncthreads();  // cb visible to all threads

  const int s_out_stride = a.s_out;
  for (int r = blockIdx.x / kCL; r < a.n; r += gridDim.x / kCL) {
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
    // P must be strictly increasing; P_0 == P_{p-1} is the constant vector.
    const bool degenerate = (c.sP[0] == c.sP[p - 1]);
    int bad = 0;
    if (!degenerate)
      for (int k = threadIdx.x; k < p - 1; k += blockDim.x) bad |= !(c.sP[k] < c.sP[k + 1]);
    bad = __syncthreads_or(bad);
    int32_t st = s_flag != 0 ? s_flag : (bad ? kStatusArg : kStatusOk);

    if (st != kStatusOk || degenerate) {
      // Invalid row: -1 codes. Constant row: Q = {P_0}, zero cost.
      const int qv = (st == kStatusOk) ? 0 : -1;
      const int ml = (st == kStatusOk) ? 1 : 0;
      if (a.mode == 0) {
        for (int t = 0; t < a.n_lambda; ++t) {
          const int64_t w = static_cast<int64_t>(r) * a.n_lambda + t;
          for (int q = threadIdx.x; q < s_out_stride; q += blockDim.x) a.Q[w * s_out_stride + q] = (q == 0) ? qv : -1;
          if (threadIdx.x == 0) {
            a.Q_len[w] = ml;
            a.obj[w] = a.mse[w] = a.H[w] = 0.0;
          }
        }
      } else {
        for (int q = threadIdx.x; q < s_out_stride; q += blockDim.x) {
          a.Q1[int64_t(r) * s_out_stride + q] = (q == 0) ? qv : -1;
          a.Q2[int64_t(r) * s_out_stride + q] = (q == 0) ? qv : -1;
        }
        if (threadIdx.x == 0) {
          a.Q1_len[r] = a.Q2_len[r] = ml;
          a.theta[r] = a.lam_lo[r] = a.lam_hi[r] = 0.0;
          a.H1[r] = a.H2[r] = a.mse1[r] = a.mse2[r] = 0.0;
        }
      }
      if (threadIdx.x == 0) a.status[r] = st;
      __syncthreads();
      continue;
    }

    if constexpr (kCL > 1) csync<kCL>();  // the other CTAs are done with the previous vector's tables
    build_tables(c);
    __syncthreads();
    if (c.hirschberg) {
      build_reflected(c);
      __syncthreads();
    }

    if (a.mode == 0) {
      for (int t = 0; t < a.n_lambda; ++t) {
        const int64_t w = static_cast<int64_t>(r) * a.n_lambda + t;
        const double lam = a.lambda[w];
        solve<T, kUnrollK, kCL, !kSmemTables>(c, lam, &s_out, &s_bestE, s_wbest, s_warg);
        for (int q = threadIdx.x; q < s_out_stride; q += blockDim.x)
          a.Q[w * s_out_stride + q] = (q < s_out.m) ? c.sQ[q] : -1;
        if (threadIdx.x == 0) {
          a.Q_len[w] = s_out.m;
          a.obj[w] = s_out.J;
          a.mse[w] = s_out.mse;
          a.H[w] = s_out.H;
        }
        __syncthreads();
      }
      if (threadIdx.x == 0) a.status[r] = kStatusOk;
    } else {
      // Bisection on lambda with two-way time-sharing.
      double lo = 0.0;
      double hi = (c.sP[p - 1] - c.sP[0]) * (c.sP[p - 1] - c.sP[0]);
      double H1 = 0, H2 = 0, M1 = 0, M2 = 0;
      int m1 = 0, m2 = 0;
      auto keep = [&](int* dst, int& m, double& Hk, double& Mk) {
        for (int q = threadIdx.x; q < S; q += blockDim.x) dst[q] = c.sQ[q];
        m = s_out.m;
        Hk = s_out.H;
        Mk = s_out.mse;
      };
      int32_t status = kStatusOk;
      double theta = 0.0;
      solve<T, kUnrollK, kCL, !kSmemTables>(c, 0.0, &s_out, &s_bestE, s_wbest, s_warg);
      keep(sQ1, m1, H1, M1);
      if (s_out.H <= a.budget) {
        keep(sQ2, m2, H2, M2);
        hi = 0.0;
      } else {
        __syncthreads();
        solve<T, kUnrollK, kCL, !kSmemTables>(c, hi, &s_out, &s_bestE, s_wbest, s_warg);
        keep(sQ2, m2, H2, M2);
        if (s_out.H > a.budget) {
          status = kStatusBudget;
        } else {
          for (int it = 0; it < a.steps; ++it) {
            const double mid = 0.5 * (lo + hi);
            __syncthreads();
            solve<T, kUnrollK, kCL, !kSmemTables>(c, mid, &s_out, &s_bestE, s_wbest, s_warg);
            if (s_out.H > a.budget) {
              lo = mid;
              keep(sQ1, m1, H1, M1);
            } else {
              hi = mid;
              keep(sQ2, m2, H2, M2);
            }
          }
          double th = (a.budget - H2) / (H1 - H2);
          theta = th < 0.0 ? 0.0 : (th > 1.0 ? 1.0 : th);
        }
      }
      __syncthreads();
      for (int q = threadIdx.x; q < s_out_stride; q += blockDim.x) {
        a.Q1[int64_t(r) * s_out_stride + q] = (q < m1) ? sQ1[q] : -1;
        a.Q2[int64_t(r) * s_out_stride + q] = (q < m2) ? sQ2[q] : -1;
      }
      if (threadIdx.x == 0) {
        a.Q1_len[r] = m1;
        a.Q2_len[r] = m2;
        a.theta[r] = theta;
        a.lam_lo[r] = lo;
        a.lam_hi[r] = hi;
        a.H1[r] = H1;
        a.H2[r] = H2;
        a.mse1[r] = M1;
        a.mse2[r] = M2;
        a.status[r] = status;
      }
    }
    __syncthreads();
  }
  // rank 0's task counters stay alive until no CTA of the cluster can reach them
  if constexpr (kCL > 1) cooperative_groups::this_cluster().sync();
}

template <typename T, bool kSmem, int kCL>
void* dp_kernel_ptr() {
  return reinterpret_cast<void*>(&k_dp<T, kSmem, kCL>);
}

// Tables in shared memory run one CTA per vector; tables in the global slab can
// run a cluster of two CTAs per vector when there are few vectors.
void* dp_fn(bool fp64, bool smem, int cluster) {
  if (smem) return fp64 ? dp_kernel_ptr<double, true, 1>() : dp_kernel_ptr<float, true, 1>();
  if (cluster == 2) return fp64 ? dp_kernel_ptr<double, false, 2>() : dp_kernel_ptr<float, false, 2>();
  return fp64 ? dp_kernel_ptr<double, false, 1>() : dp_kernel_ptr<float, false, 1>();
}

size_t small_smem(int p, int S, size_t tsz) {
  auto al = [](size_t b) { return (b + 15) & ~size_t(15); };
  return al(8 * p) * 4 + al(8 * S) * 2 + al(tsz * p) + al(4 * p) + al(4 * S) * 4 + al(8 * S) + al(4 * (p + 1));
}

size_t table_bytes(int p, size_t tsz) {
  const size_t tb = (tsz * tri_size(p) + 15) & ~size_t(15);
  const size_t gb = (2 * tsz * static_cast<size_t>(layer_elems(p)) + 15) & ~size_t(15);
  return 2 * gb + 2 * tb;
}

}  // namespace

int64_t dp_triples(int p, int s) {
  const int S = s < p ? s : p;
  int64_t t = 0;
  for (int i = 2; i <= S - 1; ++i) {
    const bool last = (i == S - 1);
    for (int l = i - 1; l <= p - 2; ++l) {
      const int64_t K = (i == 2) ? 1 : (l - i + 2);
      const int64_t NJ = last ? 1 : (p - 1 - l);
      t += K * NJ;
    }
  }
  return t;
}

bool dp_plan(int n, int p, int s, bool fp64, bool hirschberg, DpPlan* plan) {
  if (p < 2 || p > kMaxP || s < 2 || n < 1) return false;
  const int S = s < p ? s : p;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int sms = 0, optin = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t tsz = fp64 ? 8 : 4;
  const size_t small = small_smem(p, S, tsz);
  const size_t big = table_bytes(p, tsz);
  plan->fp64 = fp64;
  plan->hirschberg = hirschberg;
  plan->threads = kThreads;
  plan->smem_tables = !hirschberg && (small + big + 1024 <= static_cast<size_t>(optin));
  plan->smem_bytes = small + (plan->smem_tables ? big : 0);
  const size_t bp = hirschberg ? 0 : (tsz * static_cast<size_t>(S) * tri_size(p) + 255) & ~size_t(255);
  const size_t slab = plan->smem_tables ? 0 : (hirschberg ? 2 * big : big);
  plan->scratch_per_cta = (bp + slab + 255) & ~size_t(255);
  // Two CTAs per vector when the tables are in the global slab and the
  // vectors alone would leave more than half of the SMs idle.
  plan->cluster = (!plan->smem_tables && 2 * n <= sms) ? 2 : 1;
  void* fn = dp_fn(fp64, plan->smem_tables, plan->cluster);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(plan->smem_bytes)) !=
      cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, plan->smem_bytes) != cudaSuccess ||
      per_sm < 1)
    return false;
  const int slots = sms * per_sm / plan->cluster;  // vectors in flight
  plan->ctas = plan->cluster * (n < slots ? n : slots);
  return true;
}

cudaError_t launch_dp(const DpPlan& plan, DpArgs args, cudaStream_t st) {
  args.hirschberg = plan.hirschberg ? 1 : 0;
  void* fn = dp_fn(plan.fp64, plan.smem_tables, plan.cluster);
  void* kargs[] = {&args};
  cudaError_t e;
  if (plan.cluster > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(plan.ctas);
    cfg.blockDim = dim3(plan.threads);
    cfg.dynamicSmemBytes = plan.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = plan.cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelExC(&cfg, fn, kargs);
  } else {
    e = cudaLaunchKernel(fn, dim3(plan.ctas), dim3(plan.threads), kargs, plan.smem_bytes, st);
  }
  note_launch();
  return e;
}

}  // namespace ecasq
