// The exact ECASQ dynamic programme on B200.
//
// ECASQ summary (gist.science/pt/paper/2608.18147):
//   §2.1 "Relaxação Lagrangiana": minimise MSE(Q,X) + lambda * H(X^).
//   §2.2 "Programação Dinâmica Ótima": the ASQ DP does not extend because the
//        entropy term of a value depends on both neighbours, so the state is a
//        PAIR of consecutive values, dp_OPT(i, l, j); the direct programme costs
//        O(d^3 s) time over the entries, O(p^3 s) over a permissible set P.
//
// Recurrence evaluated here (i = number of values up to and including P_l,
// counting c_1 = P_0; m = mu/d the normalised mass of a value):
//   F_1(0, j) = V(0,j)/(lambda d) + h(L(0,j)/d)
//   F_i(l, j) = V(l,j)/(lambda d) + min_{k} [ F_{i-1}(k,l) + h((R(k,l) + L(l,j))/d) ]
//   J*/lambda = min_{i,k} F_i(k, p-1) + h(R(k,p-1)/d),   h(m) = -m log2 m.
// The whole programme is scaled by 1/lambda, so one (k,l,j) triple is one add,
// one MUFU log2 and one FMA plus the running argmin. lambda = 0 is the
// separable MSE-only programme (the minimum over k no longer depends on j).
//
// Design (this file):
//   * one CTA per vector, persistent over every solve of that vector (all
//     lambdas, or the whole bisection), so the pair tables are built once;
//   * the tables and the two live DP layers sit in shared memory when they fit
//     (fp32, p <= 128) and in a per-CTA global (L2-resident) slab otherwise;
//   * one DP layer is a list of tasks (row l, a block of <= 64 j, a k-split of
//     1..32 lanes) in descending cost order, taken by warps from a shared
//     counter; each lane keeps 2 j in registers and sweeps k with broadcast
//     loads; k-splits merge with a warp-shuffle argmin;
//   * back-pointers go to a per-CTA global slab; the backtrack, the fp64
//     evaluation of the chosen code and the bisection run in the same kernel.
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

// A group descriptor names up to kTJ outputs (l, j0 .. j0 + n - 1) of one layer:
// l in bits 0..9, j0 in bits 10..19, n - 1 in bits 20..22.
__host__ __device__ inline uint32_t pack_group(int l, int j0, int n) {
  return static_cast<uint32_t>(l) | (static_cast<uint32_t>(j0) << 10) | (static_cast<uint32_t>(n - 1) << 20);
}
__host__ __device__ inline int max_groups(int p) { return p * ((p + kTJ - 1) / kTJ + 1); }

template <typename T>
struct Arith;

template <>
struct Arith<float> {
  // Added to every R/d so that a mass is never 0 inside the sweep:
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

// One entry of a live DP layer: the layer value G = F_{i-1}(k, l) and
// a = R(k, l)/d + eps side by side, so one 8- (16-) byte shared load feeds a
// whole k step. a is written once per vector into both ping-pong layers.
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

// cb[0..p]: padded column starts; cb[p] = elements of one layer buffer.
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

template <typename T>
struct Ctx {
  int p, S, tri;
  double dd;
  GA<T>* ga0;  // DP layers of even / odd i (with a), column layout
  GA<T>* ga1;
  const int* cb;  // [p+1] padded column starts (shared memory)
  __device__ __forceinline__ GA<T>* layer(int i) const { return (i & 1) ? ga1 : ga0; }
  T* rowB;     // L(l,j)/d
  T* rowV;     // V(l,j)/d
  uint16_t* bp;  // [S][tri] back-pointers
  double *sP, *sN, *sA, *sB;  // [p] alphabet and bucket statistics
  double *sR, *sL;            // [S] evaluation scratch
  T* rmin;                    // [p] row minima (lambda = 0)
  int* rarg;                  // [p]
  int* ctr;                   // [S] task counters
  int* sQ;                    // [S] code of the last solve
  const uint32_t* groups;  // [S][max_groups] group descriptors per layer
  const int32_t* ngroups;  // [S]
  int max_groups;
};

struct SolveOut {
  double mse, H, J;
  int m;
  int bestI, bestK;
};

// ---- table build -------------------------------------------------------------
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
      c.ga0[c.cb[cc] + a].a = av;
      c.ga1[c.cb[cc] + a].a = av;
      c.rowB[ro + cc] = static_cast<T>(L / c.dd);
      c.rowV[ro + cc] = static_cast<T>(V / c.dd);
    }
  }
}

// ---- one layer ---------------------------------------------------------------

// Best (E, i, k) over the finished layer i: E = F_i(k, p-1) + h(R(k,p-1)/d).
// Warp 0 only. Strict '<' over layers in ascending order keeps the smaller code.
template <typename T>
__device__ __forceinline__ void finalize_layer(const Ctx<T>& c, int i, const GA<T>* G, bool sep, T* bestE,
                                               int* bestI, int* bestK) {
  const int p = c.p;
  const int kb = (i == 1) ? 0 : i - 1;
  const int ke = (i == 1) ? 0 : p - 2;
  T best = Arith<T>::inf();
  int arg = 0x7fffffff;
  const GA<T>* col = G + c.cb[p - 1];
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
}

// One task of layer i >= 3: 32 group descriptors, one per lane. Lane L owns
// the outputs (l, j0 .. j0+n-1) and sweeps k = i-2 .. l-1 down its column in
// kNQ interleaved streams (each output and stream keeps its own running
// minimum, so consecutive updates do not wait on one another). The k range
// common to the warp runs unpredicated; the rest masks the layer value to +inf
// past the lane's own column.
template <typename T>
__device__ __forceinline__ void run_task(const Ctx<T>& c, uint32_t desc, bool active, int i,
                                         const GA<T>* __restrict__ Gp, GA<T>* __restrict__ Gc,
                                         uint16_t* __restrict__ bpi, T invl) {
  const int p = c.p;
  const int kmin = i - 2;
  const int l = active ? static_cast<int>(desc & 1023) : kmin + 1;  // inactive lanes: any in-range row
  const int j0 = static_cast<int>((desc >> 10) & 1023);
  const int nv = active ? static_cast<int>((desc >> 20) & 7) + 1 : 0;
  const int lmin = __reduce_min_sync(0xffffffffu, active ? l : 0x7fffffff);
  const int lmax = __reduce_max_sync(0xffffffffu, active ? l : 0);
  const int ro = row_off(l, p) - l - 1;
  T b[kTJ];
#pragma unroll
  for (int u = 0; u < kTJ; ++u) b[u] = (u < nv) ? c.rowB[ro + j0 + u] : T(0);
  const GA<T>* __restrict__ col = Gp + c.cb[l];

  T best[kTJ][kNQ];
  int arg[kTJ][kNQ];
#pragma unroll
  for (int u = 0; u < kTJ; ++u)
#pragma unroll
    for (int s = 0; s < kNQ; ++s) {
      best[u][s] = Arith<T>::inf();
      arg[u][s] = kmin;
    }
  int k = kmin;
#pragma unroll 2
  for (; k + kNQ <= lmin; k += kNQ) {
#pragma unroll
    for (int s = 0; s < kNQ; ++s) {
      const GA<T> ga = col[k + s];
#pragma unroll
      for (int u = 0; u < kTJ; ++u) {
        const T v = Arith<T>::fold(ga.g, ga.a + b[u]);
        // The running minimum is one min op per step; the argmin follows it.
        const bool lt = v < best[u][s];
        best[u][s] = Arith<T>::vmin(best[u][s], v);
        arg[u][s] = lt ? k : arg[u][s];
      }
    }
  }
#pragma unroll 1
  for (; k < lmax; ++k) {
    GA<T> ga = col[k];
    ga.g = (k < l) ? ga.g : Arith<T>::inf();
#pragma unroll
    for (int u = 0; u < kTJ; ++u) {
      const T v = Arith<T>::fold(ga.g, ga.a + b[u]);
      const bool lt = v < best[u][0];
      best[u][0] = Arith<T>::vmin(best[u][0], v);
      arg[u][0] = lt ? k : arg[u][0];
    }
  }
  // Stream s holds base indices (it saw k = base + s); the tail updated stream
  // 0 with true indices. Merge with the tie rule (smaller k wins).
#pragma unroll
  for (int u = 0; u < kTJ; ++u) {
#pragma unroll
    for (int s = 1; s < kNQ; ++s) {
      const int ks = arg[u][s] + s;
      if (best[u][s] < best[u][0] || (best[u][s] == best[u][0] && ks < arg[u][0])) {
        best[u][0] = best[u][s];
        arg[u][0] = ks;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kTJ; ++u) {
    if (u < nv) {
      const int e = ro + j0 + u;
      Gc[c.cb[j0 + u] + l].g = c.rowV[e] * invl + best[u][0];
      bpi[e] = static_cast<uint16_t>(arg[u][0]);
    }
  }
}

// One full solve at lambda (all threads). Leaves the code in c.sQ and the fp64
// evaluation in *out (shared).
template <typename T>
__device__ __forceinline__ void solve(const Ctx<T>& c, double lam, SolveOut* out, T* bestE) {
  const int p = c.p, S = c.S, tri = c.tri;
  // Below kMinLambda the entropy terms vanish under the precision of T and
  // 1/lambda would overflow it: the layers then run the MSE-only programme
  // (the code is still evaluated in fp64 at the true lambda).
  const double kMinLambda = sizeof(T) == 4 ? 1e-30 : 1e-290;
  const bool sep = !(lam > kMinLambda);
  const T invl = sep ? T(1) : static_cast<T>(1.0 / lam);
  const int tid = threadIdx.x;
  const int warp = warp_id(), lane = lane_id();

  for (int t = tid; t < S; t += blockDim.x) c.ctr[t] = 0;
  if (tid == 0) {
    *bestE = Arith<T>::inf();
    out->bestI = -1;
    out->bestK = -1;
  }
  // Layer 1: F_1(0, j) (row 0), written to buffer 1.
  {
    GA<T>* G1 = c.ga1;
    for (int j = 1 + tid; j < p; j += blockDim.x) {
      const int e = j - 1;
      T f = c.rowV[e] * invl;
      if (!sep) f += Arith<T>::nlog(c.rowB[e] + Arith<T>::kEps);
      G1[c.cb[j]].g = f;
    }
  }
  __syncthreads();
  for (int i = 2; i <= S - 1; ++i) {
    const GA<T>* Gp = c.layer(i - 1);
    GA<T>* Gc = c.layer(i);
    uint16_t* bpi = c.bp + static_cast<size_t>(i) * tri;
    const bool last = (i == S - 1);
    if (warp == 0) finalize_layer(c, i - 1, Gp, sep, bestE, &out->bestI, &out->bestK);
    if (i == 2) {
      // Only k = c_1 = 0 precedes the second value.
      for (int l = 1 + warp; l <= p - 2; l += kWarps) {
        const GA<T> ga = Gp[c.cb[l]];  // (0, l)
        const int ro = row_off(l, p) - l - 1;
        for (int j = (last ? p - 1 : l + 1) + lane; j <= p - 1; j += kWarp) {
          const int e = ro + j;
          const T v = sep ? ga.g : Arith<T>::fold(ga.g, ga.a + c.rowB[e]);
          Gc[c.cb[j] + l].g = c.rowV[e] * invl + v;
        }
      }
    } else if (sep) {
      const int kmin = i - 2;
      for (int l = i - 1 + warp; l <= p - 2; l += kWarps) {
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
      for (int l = i - 1 + warp; l <= p - 2; l += kWarps) {
        const int ro = row_off(l, p) - l - 1;
        const T rm = c.rmin[l];
        const uint16_t ra = static_cast<uint16_t>(c.rarg[l]);
        for (int j = (last ? p - 1 : l + 1) + lane; j <= p - 1; j += kWarp) {
          const int e = ro + j;
          Gc[c.cb[j] + l].g = c.rowV[e] + rm;
          bpi[e] = ra;
        }
      }
    } else {
      // Tasks in descending cost: higher rows have longer k sweeps.
      const uint32_t* pl = c.groups + static_cast<size_t>(i) * c.max_groups;
      const int np = c.ngroups[i];
      const int nt = (np + kWarp - 1) / kWarp;
      // The next task's index and descriptor are fetched before the current
      // task runs, so their latency hides behind the sweep.
      auto fetch = [&](int& t, uint32_t& d, bool& act) {
        int tt = 0;
        if (lane == 0) tt = atomicAdd(c.ctr + i, 1);
        t = __shfl_sync(0xffffffffu, tt, 0);
        const int q = (nt - 1 - t) * kWarp + lane;
        act = (t < nt) && q < np;
        d = act ? pl[q] : 0u;
      };
      int t;
      uint32_t d;
      bool act;
      fetch(t, d, act);
      while (t < nt) {
        int tn;
        uint32_t dn;
        bool an;
        fetch(tn, dn, an);
        run_task(c, d, act, i, Gp, Gc, bpi, invl);
        t = tn;
        d = dn;
        act = an;
      }
    }
    __syncthreads();
  }
  if (warp == 0) finalize_layer(c, S - 1, c.layer(S - 1), sep, bestE, &out->bestI, &out->bestK);
  __syncthreads();

  // Backtrack: c_{i+1} = p-1, c_i = k, c_{ii-1} = bp_ii(c_ii, c_{ii+1}), c_1 = 0.
  if (tid == 0) {
    if (out->bestI < 1) {  // no finite candidate (non-finite inputs): fall back to {P_0, P_{p-1}}
      out->bestI = 1;
      out->bestK = 0;
    }
    const int bi = out->bestI;
    int l = out->bestK, j = p - 1;
    c.sQ[bi] = p - 1;
    c.sQ[bi - 1] = l;
    for (int ii = bi; ii >= 2; --ii) {
      const int kk = (ii == 2) ? 0 : static_cast<int>(c.bp[static_cast<size_t>(ii) * tri + row_off(l, p) + j - l - 1]);
      c.sQ[ii - 2] = kk;
      j = l;
      l = kk;
    }
    out->m = bi + 1;
  }
  __syncthreads();

  // fp64 evaluation of the code from the bucket statistics.
  if (warp == 0) {
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
  __syncthreads();
}

template <typename T, bool kSmemTables>
__global__ void __launch_bounds__(kThreads, 1) k_dp(DpArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ SolveOut s_out;
  __shared__ T s_bestE;
  __shared__ int s_flag;

  const int p = a.p, S = a.s;
  const int tri = tri_size(p);
  Ctx<T> c;
  c.p = p;
  c.S = S;
  c.tri = tri;
  c.dd = static_cast<double>(a.d);
  c.groups = a.tasks;
  c.ngroups = a.ntasks;
  c.max_groups = a.max_tasks;

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

  unsigned char* gs = a.scratch + static_cast<size_t>(blockIdx.x) * a.scratch_per_cta;
  c.bp = reinterpret_cast<uint16_t*>(gs);
  gs += (sizeof(uint16_t) * static_cast<size_t>(S) * tri + 255) & ~size_t(255);
  const size_t tb = (sizeof(T) * static_cast<size_t>(tri) + 15) & ~size_t(15);
  const size_t gb = (2 * sizeof(T) * static_cast<size_t>(layer_elems(p)) + 15) & ~size_t(15);
  unsigned char* big = kSmemTables ? sp : gs;
  c.ga0 = reinterpret_cast<GA<T>*>(big);
  c.ga1 = reinterpret_cast<GA<T>*>(big + gb);
  c.rowB = reinterpret_cast<T*>(big + 2 * gb);
  c.rowV = reinterpret_cast<T*>(big + 2 * gb + tb);
  __syncthreads();  // cb visible to all threads

  const int s_out_stride = a.s_out;
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

    build_tables(c);
    __syncthreads();

    if (a.mode == 0) {
      for (int t = 0; t < a.n_lambda; ++t) {
        const int64_t w = static_cast<int64_t>(r) * a.n_lambda + t;
        const double lam = a.lambda[w];
        solve(c, lam, &s_out, &s_bestE);
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
      solve(c, 0.0, &s_out, &s_bestE);
      keep(sQ1, m1, H1, M1);
      if (s_out.H <= a.budget) {
        keep(sQ2, m2, H2, M2);
        hi = 0.0;
      } else {
        __syncthreads();
        solve(c, hi, &s_out, &s_bestE);
        keep(sQ2, m2, H2, M2);
        if (s_out.H > a.budget) {
          status = kStatusBudget;
        } else {
          for (int it = 0; it < a.steps; ++it) {
            const double mid = 0.5 * (lo + hi);
            __syncthreads();
            solve(c, mid, &s_out, &s_bestE);
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
}

// ---- schedule ----------------------------------------------------------------
// Group descriptors of layer i >= 3 in row-major order (rows l = i-1 .. p-2,
// j ascending in groups of kTJ; the last layer has only j = p-1). One CTA per
// layer, one thread per row; a row's first group index is the sum of the group
// counts of the rows before it.
__global__ void k_schedule(int p, int S, int max_groups_, uint32_t* groups, int32_t* ngroups) {
  const int i = blockIdx.x;
  if (i < 3) {
    if (threadIdx.x == 0) ngroups[i] = 0;
    return;
  }
  const bool last = (i == S - 1);
  auto row_groups = [&](int l) { return last ? 1 : (p - 1 - l + kTJ - 1) / kTJ; };
  uint32_t* out = groups + static_cast<size_t>(i) * max_groups_;
  for (int l = i - 1 + threadIdx.x; l <= p - 2; l += blockDim.x) {
    int o = 0;
    for (int r = i - 1; r < l; ++r) o += row_groups(r);
    if (last) {
      out[o] = pack_group(l, p - 1, 1);
    } else {
      for (int j = l + 1; j <= p - 1; j += kTJ) out[o++] = pack_group(l, j, min(kTJ, p - j));
    }
  }
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int r = i - 1; r <= p - 2; ++r) tot += row_groups(r);
    ngroups[i] = tot;
  }
}

template <typename T, bool kSmem>
void* dp_kernel_ptr() {
  return reinterpret_cast<void*>(&k_dp<T, kSmem>);
}

size_t small_smem(int p, int S, size_t tsz) {
  auto al = [](size_t b) { return (b + 15) & ~size_t(15); };
  return al(8 * p) * 4 + al(8 * S) * 2 + al(tsz * p) + al(4 * p) + al(4 * S) * 4 + al(4 * (p + 1));
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

size_t dp_schedule_bytes(int p, int s) {
  const int S = s < p ? s : p;
  return ((sizeof(uint32_t) * static_cast<size_t>(max_groups(p)) * S + 255) & ~size_t(255)) +
         ((sizeof(int32_t) * S + 255) & ~size_t(255));
}

bool dp_plan(int n, int p, int s, bool fp64, DpPlan* plan) {
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
  plan->threads = kThreads;
  plan->smem_tables = (small + big + 1024 <= static_cast<size_t>(optin));
  plan->smem_bytes = small + (plan->smem_tables ? big : 0);
  const size_t bp = (sizeof(uint16_t) * static_cast<size_t>(S) * tri_size(p) + 255) & ~size_t(255);
  plan->scratch_per_cta = (bp + (plan->smem_tables ? 0 : big) + 255) & ~size_t(255);
  plan->max_tasks = max_groups(p);
  void* fn = fp64 ? (plan->smem_tables ? dp_kernel_ptr<double, true>() : dp_kernel_ptr<double, false>())
                  : (plan->smem_tables ? dp_kernel_ptr<float, true>() : dp_kernel_ptr<float, false>());
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(plan->smem_bytes)) !=
      cudaSuccess)
    return false;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, plan->smem_bytes) != cudaSuccess ||
      per_sm < 1)
    return false;
  const int ctas = sms * per_sm;
  plan->ctas = n < ctas ? n : ctas;
  return true;
}

cudaError_t launch_dp(const DpPlan& plan, DpArgs args, uint32_t* tasks, int32_t* ntasks, cudaStream_t st) {
  const int S = args.s;
  args.tasks = tasks;
  args.ntasks = ntasks;
  args.max_tasks = plan.max_tasks;
  k_schedule<<<S, 128, 0, st>>>(args.p, S, plan.max_tasks, tasks, ntasks);
  note_launch();
  void* fn = plan.fp64 ? (plan.smem_tables ? dp_kernel_ptr<double, true>() : dp_kernel_ptr<double, false>())
                       : (plan.smem_tables ? dp_kernel_ptr<float, true>() : dp_kernel_ptr<float, false>());
  void* kargs[] = {&args};
  cudaError_t e = cudaLaunchKernel(fn, dim3(plan.ctas), dim3(plan.threads), kargs, plan.smem_bytes, st);
  note_launch();
  return e;
}

}  // namespace ecasq
