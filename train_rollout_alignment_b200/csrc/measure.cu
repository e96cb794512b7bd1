// measure.cu -- a measurement helper, not a step of the method: the issue
// rate of the 32 x 32 -> 64-bit integer multiply (mul.wide.u32), which bounds
// the Philox4x32-10 generator of the stochastic-rounding kernels (10 rounds
// of two such multiplies per random word).  The roofline of those kernels is
// derived from this measured rate instead of a constant.
//
// One CTA of kMeasureThreads threads per SM; every thread runs kChains
// independent multiply chains (x <- hi(x * K) ^ lo(x * K)), enough
// independent work that the multiplier, not latency, sets the pace.  Each CTA
// reads the SM clock before and after its loop; lanes per clock per SM =
// threads x iterations x chains / cycles.
#include "launch.h"

namespace nvfp4 {

constexpr int kMeasureThreads = 1024;
constexpr int kChains = 8;

__global__ void __launch_bounds__(kMeasureThreads, 1)
    k_measure_mul_wide(int iters, uint32_t seed, unsigned long long* __restrict__ cycles,
                       uint32_t* __restrict__ sink) {
  uint32_t x[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) x[c] = seed ^ (threadIdx.x * 0x9E3779B9u) ^ (uint32_t)c;
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
      const uint64_t p = (uint64_t)x[c] * (0xD2511F53u + 2u * (uint32_t)c);
      x[c] = (uint32_t)(p >> 32) ^ (uint32_t)p;
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  uint32_t acc = 0;
#pragma unroll
  for (int c = 0; c < kChains; ++c) acc ^= x[c];
  if (acc == 0x12345678u) sink[blockIdx.x] = acc;  // keeps the chains live
  if (threadIdx.x == 0) cycles[blockIdx.x] = (unsigned long long)(t1 - t0);
}

cudaError_t launch_measure_mul_wide(int ctas, int iters, unsigned long long* cycles, uint32_t* sink,
                                    cudaStream_t s) {
  k_measure_mul_wide<<<ctas, kMeasureThreads, 0, s>>>(iters, 0x2545F491u, cycles, sink);
  return cudaGetLastError();
}

}  // namespace nvfp4
