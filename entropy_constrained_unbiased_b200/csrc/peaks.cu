// Throughput microbenchmarks for the roofline denominators of the DP kernel:
// MUFU lg2 results/s and FP32 FFMA/s on the current device. Measurement
// tooling for bench.py (libecasq_peaks.so); not part of the solver.
#include <cuda_runtime.h>

#include <cstdint>

namespace {

constexpr int kChains = 8;
constexpr int kIters = 4096;

__global__ void __launch_bounds__(256) k_lg2(float* out, float seed) {
  float x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = seed + 0.25f * c + 1e-3f * threadIdx.x;
  for (int it = 0; it < kIters; ++it) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
      float y;
      asm volatile("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x[c]));
      x[c] = y + 1.5f;  // stays in [0.5, 2): lg2 maps it back into [-1, 1)
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) acc += x[c];
  if (acc == 12345.678f) out[threadIdx.x] = acc;
}

__global__ void __launch_bounds__(256) k_ffma(float* out, float seed) {
  float x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = seed + 0.25f * c + 1e-3f * threadIdx.x;
  const float a = 0.999f, b = 1e-4f;
  for (int it = 0; it < kIters; ++it) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = fmaf(x[c], a, b);
  }
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) acc += x[c];
  if (acc == 12345.678f) out[threadIdx.x] = acc;
}

double run(void (*k)(float*, float), int blocks_per_sm) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  float* out = nullptr;
  if (cudaMalloc(&out, 256 * sizeof(float)) != cudaSuccess) return -1.0;
  const int blocks = sms * blocks_per_sm;
  k<<<blocks, 256>>>(out, 0.75f);  // warm-up
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaEventRecord(e0);
  const int reps = 5;
  for (int r = 0; r < reps; ++r) k<<<blocks, 256>>>(out, 0.75f);
  cudaEventRecord(e1);
  cudaEventSynchronize(e1);
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaFree(out);
  if (cudaGetLastError() != cudaSuccess) return -1.0;
  const double ops = double(reps) * blocks * 256.0 * kIters * kChains;
  return ops / (ms * 1e-3);
}

}  // namespace

extern "C" {
// Results per second of lg2.approx.ftz.f32 (one MUFU op each) over the device.
double ecasq_peak_lg2_per_s() { return run(k_lg2, 8); }
// FP32 fused multiply-adds per second over the device.
double ecasq_peak_ffma_per_s() { return run(k_ffma, 8); }
}
