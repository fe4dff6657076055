// Lossless entropy coder for the emitted indices ("Entropy-Constrained Adaptive
// Stochastic Quantization (ECASQ)", gist.science/pt/paper/2608.18147, §1
// "Contexto": the quantizer's output is entropy-coded, frequent values getting
// shorter bit strings; H(X^) is what such a coder approaches). Static-model rANS
// (Duda, "Asymmetric numeral systems", arXiv:1311.2540):
//   * one model per vector and time-sharing part, from the encoder's histogram:
//     f_i = max(1, floor(c_i M / n)) for the symbols that occur, M = 2^15; the
//     shortfall to M goes to the most frequent symbol (lowest index on ties), an
//     excess is taken from the largest frequencies first, none below 1. The part
//     of an entry is not coded: both sides recompute it from the seed;
//   * state x in [2^16, 2^32), 16-bit words: before coding a symbol (f, c), if
//     x >= 2^17 f the low half is emitted; then x <- floor(x/f) M + x mod f + c;
//   * one warp per segment of 32 x 512 entries, one state per lane: step t
//     codes entries 32t .. 32t+31. The encoder runs the steps backwards; in a
//     step the lanes that renormalise push their word onto the segment's word
//     stack in lane order (ballot + popcount give the slots); the final states
//     follow as (low, high) pairs. The decoder pops them in reverse.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "kernels.cuh"

namespace ecasq {
namespace {

constexpr int kScale = 15;
constexpr uint32_t kM = 1u << kScale;
constexpr uint32_t kLow = 1u << 16;
constexpr int kSteps = 512;
constexpr int64_t kSeg = int64_t(kWarp) * kSteps;
constexpr int64_t kSegCap = int64_t(kWarp) * kSteps + 2 * kWarp;
constexpr int kWarpsPerBlock = 4;

// Quantised model of hist[0..s) into f[0..s), cum[0..s] (shared), one warp.
__device__ void build_model(const int64_t* __restrict__ cnt, int s, uint32_t* f, uint32_t* cum) {
  const int lane = lane_id();
  long long total = 0;
  for (int i = lane; i < s; i += kWarp) total += cnt[i];
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  long long sum = 0;
  for (int i = lane; i < s; i += kWarp) {
    uint32_t v = 0;
    if (cnt[i] > 0) {
      const long long q = (cnt[i] * static_cast<long long>(kM)) / total;
      v = q < 1 ? 1u : static_cast<uint32_t>(q);
    }
    f[i] = v;
    sum += v;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  __syncwarp();
  long long diff = static_cast<long long>(kM) - sum;
  if (total > 0 && diff > 0) {
    // most frequent symbol, lowest index on ties
    long long bc = -1;
    int bi = 0x7fffffff;
    for (int i = lane; i < s; i += kWarp)
      if (cnt[i] > bc) {
        bc = cnt[i];
        bi = i;
      }
    for (int o = 16; o > 0; o >>= 1) {
      const long long oc = __shfl_xor_sync(0xffffffffu, bc, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oc > bc || (oc == bc && oi < bi)) {
        bc = oc;
        bi = oi;
      }
    }
    if (lane == 0) f[bi] += static_cast<uint32_t>(diff);
  }
  // An excess needs some frequency above 1 (s frequencies of 1 sum to less
  // than M); each round takes from the largest one and either ends the excess or
  // brings that frequency to 1, so s rounds suffice.
  for (int round = 0; total > 0 && diff < 0 && round < s; ++round) {
    __syncwarp();
    uint32_t bf = 0;
    int bi = 0x7fffffff;
    for (int i = lane; i < s; i += kWarp)
      if (f[i] > 1 && f[i] > bf) {
        bf = f[i];
        bi = i;
      }
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t of = __shfl_xor_sync(0xffffffffu, bf, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (of > bf || (of == bf && oi < bi)) {
        bf = of;
        bi = oi;
      }
    }
    if (bi == 0x7fffffff) break;  // not reached (see above)
    const long long take = min(static_cast<long long>(bf) - 1, -diff);
    __syncwarp();
    if (lane == 0) f[bi] -= static_cast<uint32_t>(take);
    diff += take;
  }
  __syncwarp();
  // cum = exclusive prefix sum of f, in chunks of 32
  uint32_t carry = 0;
  for (int i0 = 0; i0 < s; i0 += kWarp) {
    const int i = i0 + lane;
    const uint32_t v = i < s ? f[i] : 0u;
    uint32_t incl = v;
    for (int o = 1; o < kWarp; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (i < s) cum[i] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, kWarp - 1);
  }
  if (lane == 0) cum[s] = carry;
  __syncwarp();
}

// mode of a row: 0 every entry in part 0, 1 every entry in part 1, 2 mixed.
__device__ __forceinline__ int row_mode(int two_codes, const double* theta, int r, double* th) {
  *th = 0.0;
  if (!two_codes) return 0;
  const double t = theta ? theta[r] : 0.0;
  *th = t;
  if (t > 0.0 && t < 1.0) return 2;
  return t >= 1.0 ? 0 : 1;
}

// A warp's two models (parts 0 and 1), in dynamic shared memory sized by s.
struct WarpModel {
  // floor(x / f) = umulhi64(x, rcp) for x < 2^32, f in [2, 2^15]:
  // rcp = ceil(2^47 / f) * 2^17; the product overestimates x/f by less than
  // x / 2^47 < 2^-15 <= 1/f, which never crosses the next integer.
  unsigned long long* rcp;  // [2s]
  uint32_t* f;              // [2s]
  uint32_t* cum;            // [2(s+1)]
};

// Bytes of one warp's models (16-byte multiple).
__host__ __device__ inline size_t warp_model_bytes(int s) {
  return (sizeof(unsigned long long) * 2 * s + sizeof(uint32_t) * 2 * s + sizeof(uint32_t) * 2 * (s + 1) + 15) &
         ~size_t(15);
}

__device__ __forceinline__ WarpModel warp_model(unsigned char* base, int s, int warp) {
  unsigned char* b = base + warp_model_bytes(s) * warp;
  WarpModel m;
  m.rcp = reinterpret_cast<unsigned long long*>(b);
  m.f = reinterpret_cast<uint32_t*>(b + sizeof(unsigned long long) * 2 * s);
  m.cum = m.f + 2 * s;
  return m;
}

constexpr int kChunk = 32;  // steps staged at a time

// The decoder's staged chunk: the parts of kChunk steps (so that the serial
// state updates do not wait on Philox) and the decoded symbols, written back
// to the row in one coalesced pass.
struct WarpStage {
  uint8_t sym[kChunk * kWarp];
  uint32_t part[kChunk];  // bit j of word t: part of lane j at step t_lo + t
};

__device__ void model_reciprocals(const WarpModel& m, int s) {
  for (int i = lane_id(); i < 2 * s; i += kWarp) {
    const unsigned long long f = m.f[i];
    m.rcp[i] = f >= 2 ? (((1ull << 47) + f - 1) / f) << 17 : 0ull;
  }
  __syncwarp();
}

// Parts of steps t_lo .. t_hi-1 for the decoder (lane j draws the 8 Philox
// blocks of step t_lo + j).
__device__ void stage_chunk(int64_t base, int t_lo, int t_hi, uint32_t row, uint32_t k0, uint32_t k1, int mode,
                            double th, WarpStage& st) {
  const int lane = lane_id();
  const int64_t e_lo = base + static_cast<int64_t>(t_lo) * kWarp;
  if (lane < t_hi - t_lo) {
    uint32_t bits = mode == 1 ? 0xffffffffu : 0u;
    if (mode == 2) {
      const int64_t e0 = e_lo + static_cast<int64_t>(lane) * kWarp;
      // u < theta with u = word * 2^-32 is word < ceil(theta * 2^32): theta * 2^32
      // is exact in fp64 and the word is an integer.
      const uint64_t cut = static_cast<uint64_t>(ceil(th * 0x1p32));
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const uint4 w = Philox4x32::block(make_uint4(static_cast<uint32_t>((e0 >> 2) + b), row, 1u, 0u), k0, k1);
        bits |= (static_cast<uint64_t>(w.x) < cut ? 0u : 1u) << (4 * b);
        bits |= (static_cast<uint64_t>(w.y) < cut ? 0u : 1u) << (4 * b + 1);
        bits |= (static_cast<uint64_t>(w.z) < cut ? 0u : 1u) << (4 * b + 2);
        bits |= (static_cast<uint64_t>(w.w) < cut ? 0u : 1u) << (4 * b + 3);
      }
    }
    st.part[lane] = bits;
  }
  __syncwarp();
}

// The encoder's staged chunk: per entry the index of its (part, symbol) pair,
// part * s + symbol, into the packed model; per step the parts' bit word.
struct EncStage {
  uint16_t code[kChunk * kWarp];
  uint32_t part[kChunk];
};

// Parts (lane j draws the 8 Philox blocks of step t_lo + j) and the pair
// indices of steps t_lo .. t_hi-1. A symbol >= s sets *bad and is coded as
// s - 1 (the row's status reports it).
__device__ void stage_codes(const uint8_t* __restrict__ xrow, int64_t d, int64_t base, int t_lo, int t_hi,
                            uint32_t row, uint32_t k0, uint32_t k1, int mode, double th, int s, EncStage& st,
                            int* bad) {
  const int lane = lane_id();
  const int64_t e_lo = base + static_cast<int64_t>(t_lo) * kWarp;
  const int n_ent = (t_hi - t_lo) * kWarp;
  uint8_t v[kChunk];
#pragma unroll
  for (int k = 0; k < kChunk; ++k) {  // all 32 loads of a lane in flight first
    const int i = k * kWarp + lane;
    v[k] = (i < n_ent && e_lo + i < d) ? xrow[e_lo + i] : 0;
  }
  if (lane < t_hi - t_lo) {
    uint32_t bits = mode == 1 ? 0xffffffffu : 0u;
    if (mode == 2) {
      const int64_t e0 = e_lo + static_cast<int64_t>(lane) * kWarp;
      // u < theta with u = word * 2^-32 is word < ceil(theta * 2^32): theta * 2^32
      // is exact in fp64 and the word is an integer.
      const uint64_t cut = static_cast<uint64_t>(ceil(th * 0x1p32));
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const uint4 w = Philox4x32::block(make_uint4(static_cast<uint32_t>((e0 >> 2) + b), row, 1u, 0u), k0, k1);
        bits |= (static_cast<uint64_t>(w.x) < cut ? 0u : 1u) << (4 * b);
        bits |= (static_cast<uint64_t>(w.y) < cut ? 0u : 1u) << (4 * b + 1);
        bits |= (static_cast<uint64_t>(w.z) < cut ? 0u : 1u) << (4 * b + 2);
        bits |= (static_cast<uint64_t>(w.w) < cut ? 0u : 1u) << (4 * b + 3);
      }
    }
    st.part[lane] = bits;
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < kChunk; ++k) {
    const int i = k * kWarp + lane;
    int sym = v[k];
    if (i < n_ent && e_lo + i < d && sym >= s) {
      *bad = 1;
      sym = s - 1;
    }
    const int part = (k < t_hi - t_lo) ? static_cast<int>((st.part[k] >> lane) & 1u) : 0;
    st.code[i] = static_cast<uint16_t>(part * s + sym);
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kWarp * kWarpsPerBlock) k_rans_encode(
    const uint8_t* __restrict__ idx, const int64_t* __restrict__ hist, const double* __restrict__ theta,
    int two_codes, int n, int64_t d, int s, uint64_t seed, int64_t nseg, uint16_t* __restrict__ words,
    int32_t* __restrict__ seg_len, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char rsm[];
  __shared__ EncStage ss[kWarpsPerBlock];
  const int warp = warp_id(), lane = lane_id();
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (unit >= static_cast<int64_t>(n) * nseg) return;  // warp-uniform
  const int r = static_cast<int>(unit / nseg);
  const int64_t g = unit % nseg;
  const WarpModel m = warp_model(rsm, s, warp);
  EncStage& st = ss[warp];
  build_model(hist + static_cast<int64_t>(r) * 2 * s, s, m.f, m.cum);
  build_model(hist + static_cast<int64_t>(r) * 2 * s + s, s, m.f + s, m.cum + s + 1);
  model_reciprocals(m, s);
  // pack each pair's frequency and cumulative start into one word of m.f:
  // f | c << 16 (both below 2^16), so a step reads one word and the reciprocal
  for (int i = lane_id(); i < 2 * s; i += kWarp) {
    const int part = i >= s ? 1 : 0, sym = i - part * s;
    m.f[i] |= m.cum[part * (s + 1) + sym] << 16;
  }
  __syncwarp();
  double th;
  const int mode = row_mode(two_codes, theta, r, &th);
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const int64_t base = g * kSeg;
  const int64_t len = min(kSeg, d - base);
  const int steps = static_cast<int>((len + kWarp - 1) / kWarp);
  const int len32 = static_cast<int>(len);
  const uint8_t* xrow = idx + static_cast<int64_t>(r) * d;
  uint16_t* out = words + unit * kSegCap;
  uint32_t x = kLow;
  int top = 0, bad = 0;
  for (int ch = (steps - 1) / kChunk; ch >= 0; --ch) {
    const int t_lo = ch * kChunk, t_hi = min(steps, t_lo + kChunk);
    __syncwarp();  // the previous chunk's reads are done
    stage_codes(xrow, d, base, t_lo, t_hi, static_cast<uint32_t>(r), k0, k1, mode, th, s, st, &bad);
    for (int t = t_hi - 1; t >= t_lo; --t) {
      const bool live = t * kWarp + lane < len32;
      const uint32_t code = st.code[(t - t_lo) * kWarp + lane];
      const uint32_t fc = m.f[code];
      const unsigned long long rc = m.rcp[code];
      const uint32_t c = fc >> 16;
      uint32_t f = fc & 0xFFFFu;
      if (live && f == 0) bad = 1;
      f = f == 0 ? 1u : f;
      // x >= 2^17 f  <=>  floor(x / 2^17) >= f
      const bool need = live && (x >> 17) >= f;
      const unsigned mask = __ballot_sync(0xffffffffu, need);
      if (need) {
        out[top + __popc(mask & ((1u << lane) - 1u))] = static_cast<uint16_t>(x & 0xFFFFu);
        x >>= 16;
      }
      top += __popc(mask);
      if (live) {
        // floor(x * rc / 2^64) for x < 2^32, from the halves of rc
        const uint32_t rlo = static_cast<uint32_t>(rc), rhi = static_cast<uint32_t>(rc >> 32);
        const unsigned long long hi = static_cast<unsigned long long>(x) * rhi + __umulhi(x, rlo);
        const uint32_t q = f == 1 ? x : static_cast<uint32_t>(hi >> 32);
        x = (q << kScale) + (x - q * f) + c;
      }
    }
  }
  out[top + 2 * lane] = static_cast<uint16_t>(x & 0xFFFFu);
  out[top + 2 * lane + 1] = static_cast<uint16_t>(x >> 16);
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0) {
    seg_len[unit] = top + 2 * kWarp;
    if (bad) atomicExch(status + r, kStatusArg);
  }
}

__global__ void __launch_bounds__(kWarp * kWarpsPerBlock) k_rans_decode(
    const uint16_t* __restrict__ words, const int32_t* __restrict__ seg_len, const int64_t* __restrict__ hist,
    const double* __restrict__ theta, int two_codes, int n, int64_t d, int s, uint64_t seed, int64_t nseg,
    uint8_t* __restrict__ idx, int32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char rsm[];
  __shared__ WarpStage ss[kWarpsPerBlock];
  const int warp = warp_id(), lane = lane_id();
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * kWarpsPerBlock + warp;
  if (unit >= static_cast<int64_t>(n) * nseg) return;  // warp-uniform
  const int r = static_cast<int>(unit / nseg);
  const int64_t g = unit % nseg;
  const WarpModel m = warp_model(rsm, s, warp);
  WarpStage& st = ss[warp];
  build_model(hist + static_cast<int64_t>(r) * 2 * s, s, m.f, m.cum);
  build_model(hist + static_cast<int64_t>(r) * 2 * s + s, s, m.f + s, m.cum + s + 1);
  double th;
  const int mode = row_mode(two_codes, theta, r, &th);
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const int64_t base = g * kSeg;
  const int64_t len = min(kSeg, d - base);
  const int steps = static_cast<int>((len + kWarp - 1) / kWarp);
  const int len32 = static_cast<int>(len);
  const uint16_t* in = words + unit * kSegCap;
  uint8_t* xrow = idx + static_cast<int64_t>(r) * d;
  int top = seg_len[unit];
  int bad = (top < 2 * kWarp || top > kSegCap) ? 1 : 0;
  uint32_t x = kLow;
  if (!bad) {
    top -= 2 * kWarp;
    x = static_cast<uint32_t>(in[top + 2 * lane]) | (static_cast<uint32_t>(in[top + 2 * lane + 1]) << 16);
  }
  for (int ch = 0; ch * kChunk < steps && !bad; ++ch) {
    const int t_lo = ch * kChunk, t_hi = min(steps, t_lo + kChunk);
    __syncwarp();
    stage_chunk(base, t_lo, t_hi, static_cast<uint32_t>(r), k0, k1, mode, th, st);
    for (int t = t_lo; t < t_hi; ++t) {
      const bool live = t * kWarp + lane < len32;
      const int part = (st.part[t - t_lo] >> lane) & 1;
      bool need = false;
      int fail = 0;
      if (live) {
        const uint32_t slot = x & (kM - 1u);
        const uint32_t* cp = m.cum + part * (s + 1);
        if (slot >= cp[s]) {
          fail = 1;
        } else {
          // largest i with cp[i] <= slot: the symbol whose interval holds slot
          int lo = 0, hi = s;
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cp[mid] <= slot)
              lo = mid;
            else
              hi = mid;
          }
          st.sym[(t - t_lo) * kWarp + lane] = static_cast<uint8_t>(lo);
          x = m.f[part * s + lo] * (x >> kScale) + slot - cp[lo];
          need = x < kLow;
        }
      }
      const unsigned mask = __ballot_sync(0xffffffffu, need);
      const int nn = __popc(mask);
      bad = __reduce_or_sync(0xffffffffu, fail) | (top - nn < 0 ? 1 : 0);
      if (bad) break;
      top -= nn;
      if (need) x = (x << 16) | in[top + __popc(mask & ((1u << lane) - 1u))];
    }
    __syncwarp();
    if (!bad) {
      const int n_ent = (t_hi - t_lo) * kWarp;
      const int64_t e_lo = base + static_cast<int64_t>(t_lo) * kWarp;
      for (int i = lane; i < n_ent; i += kWarp)
        if (e_lo + i < d) xrow[e_lo + i] = st.sym[i];
    }
  }
  if (!bad && top != 0) bad = 1;
  if (lane == 0 && bad) atomicExch(status + r, kStatusArg);
}

}  // namespace

int64_t rans_segments(int64_t d) { return (d + kSeg - 1) / kSeg; }
int64_t rans_segment_words() { return kSegCap; }

cudaError_t launch_rans_encode(const uint8_t* idx, const int64_t* hist, const double* theta, int two_codes, int n,
                               int64_t d, int s, uint64_t seed, uint16_t* words, int32_t* seg_len, int32_t* status,
                               cudaStream_t st) {
  const int64_t nseg = rans_segments(d);
  const int64_t units = static_cast<int64_t>(n) * nseg;
  cudaMemsetAsync(status, 0, sizeof(int32_t) * n, st);
  const int64_t blocks = (units + kWarpsPerBlock - 1) / kWarpsPerBlock;
  k_rans_encode<<<static_cast<unsigned>(blocks), kWarp * kWarpsPerBlock, warp_model_bytes(s) * kWarpsPerBlock, st>>>(idx, hist, theta, two_codes, n, d,
                                                                                   s, seed, nseg, words, seg_len,
                                                                                   status);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_rans_decode(const uint16_t* words, const int32_t* seg_len, const int64_t* hist, const double* theta,
                               int two_codes, int n, int64_t d, int s, uint64_t seed, uint8_t* idx, int32_t* status,
                               cudaStream_t st) {
  const int64_t nseg = rans_segments(d);
  const int64_t units = static_cast<int64_t>(n) * nseg;
  cudaMemsetAsync(status, 0, sizeof(int32_t) * n, st);
  const int64_t blocks = (units + kWarpsPerBlock - 1) / kWarpsPerBlock;
  k_rans_decode<<<static_cast<unsigned>(blocks), kWarp * kWarpsPerBlock, warp_model_bytes(s) * kWarpsPerBlock, st>>>(words, seg_len, hist, theta,
                                                                                   two_codes, n, d, s, seed, nseg, idx,
                                                                                   status);
  note_launch();
  return cudaGetLastError();
}

}  // namespace ecasq
