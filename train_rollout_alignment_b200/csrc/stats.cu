// stats.cu -- train/rollout mismatch counters between two NVFP4 tensors
// (TRACE explainer: the train/rollout distance is the quantity to shrink; the
// compaction paragraph observes that >99% of mismatches are one cell apart).
//
// One thread per 16-value block: 8 code bytes and 1 scale byte from each side.
// Positions are signed grid indices; decoded values are (G[m] * sb) * s_t in
// FP32 (the E2M1 decode instruction gives signed G[m] exactly).  Counters are
// per-thread u32, reduced per CTA and added to the u64 outputs with one atomic
// per counter per CTA.
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kStatsCtasPerSm = 4;
constexpr int kStatsUnroll = 4;

struct MismatchCounts {
  uint32_t mism, adj, far, sumd, scale, value;
};

__device__ __forceinline__ int signed_pos(uint32_t nib) {
  const int m = (int)(nib & 7u);
  return (nib & 8u) ? -m : m;
}

__device__ __forceinline__ void mismatch_block(uint2 a, uint2 b, uint32_t sba, uint32_t sbb,
                                               float tsa, float tsb, MismatchCounts& c) {
  const float sva = e4m3_value(sba), svb = e4m3_value(sbb);
  c.scale += (sba != sbb) ? 1u : 0u;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t wa = half ? a.y : a.x, wb = half ? b.y : b.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float ga[2], gb[2];
      e2m1x2_decode((wa >> (8 * j)) & 0xFFu, ga[0], ga[1]);
      e2m1x2_decode((wb >> (8 * j)) & 0xFFu, gb[0], gb[1]);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int sh = 4 * (2 * j + t);
        const int pa = signed_pos((wa >> sh) & 0xFu), pb = signed_pos((wb >> sh) & 0xFu);
        const uint32_t d = (uint32_t)abs(pa - pb);
        c.mism += d != 0u;
        c.adj += d == 1u;
        c.far += d >= 2u;
        c.sumd += d;
        const float ya = __fmul_rn(__fmul_rn(ga[t], sva), tsa);
        const float yb = __fmul_rn(__fmul_rn(gb[t], svb), tsb);
        c.value += (ya != yb) ? 1u : 0u;
      }
    }
  }
}

template <int U>
__global__ void __launch_bounds__(kThreads, kStatsCtasPerSm)
    k_mismatch_stats(const uint8_t* __restrict__ ca, const uint8_t* __restrict__ sa,
                     const float* __restrict__ ta, const uint8_t* __restrict__ cb,
                     const uint8_t* __restrict__ sb, const float* __restrict__ tb, int64_t nblk,
                     unsigned long long* __restrict__ stats8) {
  __shared__ unsigned long long red[6 * 8];
  const float tsa = *ta, tsb = *tb;
  MismatchCounts c{0u, 0u, 0u, 0u, 0u, 0u};
  const uint2* __restrict__ a2 = reinterpret_cast<const uint2*>(ca);
  const uint2* __restrict__ b2 = reinterpret_cast<const uint2*>(cb);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (; i + (U - 1) * stride < nblk; i += U * stride) {
    uint2 va[U], vb[U];
    uint32_t xa[U], xb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      va[u] = __ldg(a2 + i + u * stride);
      vb[u] = __ldg(b2 + i + u * stride);
      xa[u] = __ldg(sa + i + u * stride);
      xb[u] = __ldg(sb + i + u * stride);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) mismatch_block(va[u], vb[u], xa[u], xb[u], tsa, tsb, c);
  }
  for (; i < nblk; i += stride)
    mismatch_block(__ldg(a2 + i), __ldg(b2 + i), __ldg(sa + i), __ldg(sb + i), tsa, tsb, c);
  const unsigned long long vals[6] = {c.mism, c.adj, c.far, c.sumd, c.scale, c.value};
  block_add_u64<6>(vals, stats8 + 1, red);
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(stats8, (unsigned long long)nblk * 16ull);
}

cudaError_t launch_mismatch_stats(const uint8_t* ca, const uint8_t* sa, const float* ta,
                                  const uint8_t* cb, const uint8_t* sb, const float* tb,
                                  int64_t nblk, unsigned long long* stats8, cudaStream_t s) {
  if (nblk == 0) return cudaSuccess;
  k_mismatch_stats<kStatsUnroll><<<grid_for(nblk, kThreads, kStatsCtasPerSm), kThreads, 0, s>>>(
      ca, sa, ta, cb, sb, tb, nblk, stats8);
  return cudaGetLastError();
}

}  // namespace nvfp4
