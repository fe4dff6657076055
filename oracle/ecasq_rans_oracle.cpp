// ECASQ oracle, part 3: the lossless entropy coder for the emitted indices.
//
// TEST INFRASTRUCTURE ONLY, like ecasq_oracle.cpp (same library, same rules):
// nothing on the product path includes, links or calls it.
//
// Source: "Entropy-Constrained Adaptive Stochastic Quantization (ECASQ)"
// technical summary (gist.science/pt/paper/2608.18147), §1 "Contexto": the
// quantizer's output goes through a lossless entropy coder that gives frequent
// values shorter bit strings; H(X^) is what such a coder approaches. The page
// names no coder; this is range-variant asymmetric numeral systems (rANS, Duda,
// "Asymmetric numeral systems", arXiv:1311.2540) with a static model.
//
// Readings where the page leaves a step open:
//   * one model per vector and time-sharing part (the codes Q1, Q2), from the
//     encoder's histogram; the part of an entry is not coded: the decoder
//     recomputes it from the seed exactly as the encoder drew it;
//   * model: probabilities quantised to M = 2^15: f_i = max(1, floor(c_i M / n))
//     for every symbol that occurs; the shortfall to M goes to the most frequent
//     symbol (lowest index on ties); an excess is taken from the largest
//     frequencies first (lowest index on ties), none below 1;
//   * state x in [2^16, 2^32), 16-bit renormalisation: before coding a symbol
//     with frequency f, if x >= 2^17 f emit the low 16 bits and shift; then
//     x <- floor(x / f) * M + (x mod f) + c (c = cumulative frequency);
//   * 32 interleaved states per segment of 32 x 512 entries: step t covers the
//     entries 32t .. 32t+31 of the segment, state j takes entry 32t + j. The
//     encoder runs the steps from last to first; in each step the states that
//     renormalise push their word in ascending j onto one word stack; after the
//     first step every state pushes its low and high halves (j ascending). The
//     decoder pops the states, then runs the steps forward: decode, then the
//     states below 2^16 pop their words (the block the encoder pushed for that
//     step, ascending j).

#include <algorithm>
#include <cstdint>
#include <vector>

extern "C" {
void eo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
int eo_threads();
}

namespace {

constexpr int kScale = 15;
constexpr uint32_t kM = 1u << kScale;
constexpr uint32_t kLow = 1u << 16;
constexpr int kLanes = 32;
constexpr int kSteps = 512;
constexpr int64_t kSeg = int64_t(kLanes) * kSteps;
constexpr int64_t kSegCap = int64_t(kLanes) * kSteps + 2 * kLanes;  // 16-bit words

uint32_t philox_u32(uint64_t seed, int64_t j, uint32_t row, uint32_t stream) {
  uint32_t ctr[4] = {uint32_t(uint64_t(j) >> 2), row, stream, 0u};
  uint32_t key[2] = {uint32_t(seed), uint32_t(seed >> 32)};
  uint32_t out[4];
  eo_philox4x32_10(ctr, key, out);
  return out[j & 3];
}

// Time-sharing part of entry j: the rule of the encoder.
int part_of(int64_t j, uint32_t row, uint64_t seed, int two_codes, const double* theta) {
  if (!two_codes) return 0;
  const double th = theta ? theta[row] : 0.0;
  if (th > 0.0 && th < 1.0) return (double(philox_u32(seed, j, row, 1u)) * 0x1p-32 < th) ? 0 : 1;
  return th >= 1.0 ? 0 : 1;
}

}  // namespace

extern "C" {

int64_t eo_rans_segment_words() { return kSegCap; }
int64_t eo_rans_segments(int64_t d) { return (d + kSeg - 1) / kSeg; }

// Quantised model of one histogram (s symbols): f [s], cum [s+1].
void eo_rans_model(const int64_t* cnt, int s, uint32_t* f, uint32_t* cum) {
  int64_t total = 0;
  for (int i = 0; i < s; ++i) total += cnt[i];
  for (int i = 0; i < s; ++i) f[i] = 0;
  if (total > 0) {
    int64_t sum = 0;
    for (int i = 0; i < s; ++i) {
      if (cnt[i] == 0) continue;
      int64_t v = (cnt[i] * int64_t(kM)) / total;
      f[i] = uint32_t(v < 1 ? 1 : v);
      sum += f[i];
    }
    int64_t diff = int64_t(kM) - sum;
    if (diff > 0) {
      int best = 0;
      for (int i = 1; i < s; ++i)
        if (cnt[i] > cnt[best]) best = i;
      f[best] += uint32_t(diff);
    }
    while (diff < 0) {
      int best = -1;
      for (int i = 0; i < s; ++i)
        if (f[i] > 1 && (best < 0 || f[i] > f[best])) best = i;
      const int64_t take = std::min<int64_t>(int64_t(f[best]) - 1, -diff);
      f[best] -= uint32_t(take);
      diff += take;
    }
  }
  cum[0] = 0;
  for (int i = 0; i < s; ++i) cum[i + 1] = cum[i] + f[i];
}

// Encode one vector's indices. words: [segments][kSegCap], seg_len: [segments].
// Returns 0, or -1 when an index has zero frequency in its part's model.
int eo_rans_encode_row(const uint8_t* idx, int64_t d, int s, const int64_t* hist, const double* theta,
                       int two_codes, uint64_t seed, uint32_t row, uint16_t* words, int32_t* seg_len) {
  std::vector<uint32_t> f(2 * s), cum(2 * (s + 1));
  eo_rans_model(hist, s, f.data(), cum.data());
  eo_rans_model(hist + s, s, f.data() + s, cum.data() + s + 1);
  const int64_t nseg = eo_rans_segments(d);
  for (int64_t g = 0; g < nseg; ++g) {
    const int64_t base = g * kSeg, len = std::min<int64_t>(kSeg, d - base);
    const int64_t steps = (len + kLanes - 1) / kLanes;
    uint16_t* w = words + g * kSegCap;
    int64_t top = 0;
    uint32_t x[kLanes];
    for (int j = 0; j < kLanes; ++j) x[j] = kLow;
    for (int64_t t = steps - 1; t >= 0; --t) {
      uint32_t fs[kLanes], cs[kLanes];
      bool live[kLanes];
      for (int j = 0; j < kLanes; ++j) {
        const int64_t e = base + t * kLanes + j;
        live[j] = e < d;
        if (!live[j]) continue;
        const int part = part_of(e, row, seed, two_codes, theta);
        const int sym = idx[e];
        if (sym >= s) return -1;
        fs[j] = f[part * s + sym];
        cs[j] = cum[part * (s + 1) + sym];
        if (fs[j] == 0) return -1;
      }
      for (int j = 0; j < kLanes; ++j)  // renormalise: push in ascending j
        if (live[j] && uint64_t(x[j]) >= (uint64_t(kLow >> kScale) << 16) * fs[j]) {
          w[top++] = uint16_t(x[j] & 0xFFFFu);
          x[j] >>= 16;
        }
      for (int j = 0; j < kLanes; ++j)
        if (live[j]) x[j] = ((x[j] / fs[j]) << kScale) + (x[j] % fs[j]) + cs[j];
    }
    for (int j = 0; j < kLanes; ++j) {
      w[top++] = uint16_t(x[j] & 0xFFFFu);
      w[top++] = uint16_t(x[j] >> 16);
    }
    seg_len[g] = int32_t(top);
  }
  return 0;
}

// Decode one vector. Returns 0, or -1 on a malformed stream.
int eo_rans_decode_row(const uint16_t* words, const int32_t* seg_len, int64_t d, int s, const int64_t* hist,
                       const double* theta, int two_codes, uint64_t seed, uint32_t row, uint8_t* idx) {
  std::vector<uint32_t> f(2 * s), cum(2 * (s + 1));
  eo_rans_model(hist, s, f.data(), cum.data());
  eo_rans_model(hist + s, s, f.data() + s, cum.data() + s + 1);
  const int64_t nseg = eo_rans_segments(d);
  for (int64_t g = 0; g < nseg; ++g) {
    const int64_t base = g * kSeg, len = std::min<int64_t>(kSeg, d - base);
    const int64_t steps = (len + kLanes - 1) / kLanes;
    const uint16_t* w = words + g * kSegCap;
    int64_t top = seg_len[g];
    if (top < 2 * kLanes || top > kSegCap) return -1;
    uint32_t x[kLanes];
    top -= 2 * kLanes;
    for (int j = 0; j < kLanes; ++j) x[j] = uint32_t(w[top + 2 * j]) | (uint32_t(w[top + 2 * j + 1]) << 16);
    for (int64_t t = 0; t < steps; ++t) {
      bool need[kLanes];
      int nneed = 0;
      for (int j = 0; j < kLanes; ++j) {
        need[j] = false;
        const int64_t e = base + t * kLanes + j;
        if (e >= d) continue;
        const int part = part_of(e, row, seed, two_codes, theta);
        const uint32_t slot = x[j] & (kM - 1);
        const uint32_t* cp = cum.data() + part * (s + 1);
        int sym = -1;
        for (int i = 0; i < s; ++i)
          if (cp[i] <= slot && slot < cp[i + 1]) {
            sym = i;
            break;
          }
        if (sym < 0) return -1;
        idx[e] = uint8_t(sym);
        x[j] = f[part * s + sym] * (x[j] >> kScale) + slot - cp[sym];
        need[j] = x[j] < kLow;
        nneed += need[j];
      }
      top -= nneed;  // the block pushed for this step, ascending j
      if (top < 0) return -1;
      int64_t k = top;
      for (int j = 0; j < kLanes; ++j)
        if (need[j]) x[j] = (x[j] << 16) | w[k++];
    }
    if (top != 0) return -1;
  }
  return 0;
}

int eo_rans_encode_batch(const uint8_t* idx, int n, int64_t d, int s, const int64_t* hist, const double* theta,
                         int two_codes, uint64_t seed, uint16_t* words, int32_t* seg_len, int32_t* status) {
  const int64_t nseg = eo_rans_segments(d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r)
    status[r] = eo_rans_encode_row(idx + int64_t(r) * d, d, s, hist + int64_t(r) * 2 * s, theta, two_codes, seed,
                                   uint32_t(r), words + int64_t(r) * nseg * kSegCap, seg_len + int64_t(r) * nseg);
  return eo_threads();
}

int eo_rans_decode_batch(const uint16_t* words, const int32_t* seg_len, int n, int64_t d, int s,
                         const int64_t* hist, const double* theta, int two_codes, uint64_t seed, uint8_t* idx,
                         int32_t* status) {
  const int64_t nseg = eo_rans_segments(d);
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r)
    status[r] = eo_rans_decode_row(words + int64_t(r) * nseg * kSegCap, seg_len + int64_t(r) * nseg, d, s,
                                   hist + int64_t(r) * 2 * s, theta, two_codes, seed, uint32_t(r),
                                   idx + int64_t(r) * d);
  return eo_threads();
}

}  // extern "C"
