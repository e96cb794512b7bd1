// stats.cu -- train/rollout mismatch counters between two NVFP4 tensors
// (TRACE explainer: the train/rollout distance is the quantity to shrink; the
// compaction paragraph observes that >99% of mismatches are one cell apart).
//
// One lane per 16-value block: 8 code bytes and 1 scale byte from each side,
// 1.125 bytes per element.  On sm_100a the logic pipe (LOP3/SHF/PRMT/ISETP)
// retires 64 lanes per clock per SM, so keeping pace with HBM leaves about 3
// logic instructions per element.  Two ideas keep the kernel under that:
//
//  * Position counters only need work where codes differ.  A block whose 16
//    codes are identical on both sides contributes nothing, so each warp
//    pushes its "dirty" blocks into a shared-memory queue (ballot + prefix
//    rank) and processes them 32 at a time, one per lane, with the packed
//    counting below.  The cost follows the mismatch rate, not the size.
//  * Decoded-value mismatches (value = (G[m] * sb) * s_t in FP32) are decided
//    per block with no per-element FP32 work:
//      - same scale byte and same tensor scale, all products normal floats:
//        values differ exactly where positions differ (taken from the queue);
//      - otherwise two nonzero values can only be equal if
//        (sb_a * s_t_a) / (sb_b * s_t_b) lies within ~2^-22 of a ratio of two
//        grid values, i.e. of 2^k, 3 * 2^k or 2^k / 3 (the grid is
//        {2^k, 3 * 2^k}).  The significand of that ratio depends only on the
//        two scale significands (16 x 16 cases) given the tensor scales, so a
//        per-CTA table says where only zero/zero pairs can be equal;
//      - any other block compares the 16 values in FP32 (rare).
//    When the two tensor scales differ and no pair of nonzero scale
//    significands gives a ratio near a grid ratio (checked once per CTA over
//    all 15 x 15 pairs, together with the normal-float condition for every
//    nonzero scale byte), every block with two nonzero scales takes the
//    zero/zero rule without table lookups.
#include "launch.h"
#include "stats_device.cuh"

namespace nvfp4 {

constexpr int kStatsCtasPerSm = 4;
constexpr int kStatsUnroll = 2;  // two pairs (four blocks) in flight per lane

template <int U>
__global__ void __launch_bounds__(kThreads, kStatsCtasPerSm)
    k_mismatch_stats(const uint8_t* __restrict__ ca, const uint8_t* __restrict__ sa,
                     const float* __restrict__ ta, const uint8_t* __restrict__ cb,
                     const uint8_t* __restrict__ sb, const float* __restrict__ tb, int64_t nblk,
                     unsigned long long* __restrict__ stats8) {
  __shared__ StatsShared sm;
  const float tsa = *ta, tsb = *tb;
  const bool same_ts = __float_as_uint(tsa) == __float_as_uint(tsb);
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const bool far_all = stats_tables_init(sm, tsa, tsb);

  MismatchCounts c{0u, 0u, 0u, 0u, 0u};
  const uint4* __restrict__ a4 = reinterpret_cast<const uint4*>(ca);
  const uint4* __restrict__ b4 = reinterpret_cast<const uint4*>(cb);
  const uint16_t* __restrict__ sa2 = reinterpret_cast<const uint16_t*>(sa);
  const uint16_t* __restrict__ sb2 = reinterpret_cast<const uint16_t*>(sb);
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int64_t npair = nblk >> 1;                       // two blocks per lane per load
  const int64_t wstride = (int64_t)gridDim.x * kThreads;
  int qn = 0;                                            // warp-uniform queue length
  for (int64_t wb = (int64_t)blockIdx.x * kThreads + warp * 32; wb < npair; wb += U * wstride) {
    uint4 va[U], vb[U];
    uint32_t xa[U], xb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t p = wb + u * wstride + lane;
      if (p < npair) {
        va[u] = __ldg(a4 + p);
        vb[u] = __ldg(b4 + p);
        xa[u] = __ldg(sa2 + p);
        xb[u] = __ldg(sb2 + p);
      } else {
        va[u] = vb[u] = make_uint4(0u, 0u, 0u, 0u);
        xa[u] = xb[u] = 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool valid = wb + u * wstride + lane < npair;
      count_block(sm, va[u].x, va[u].y, vb[u].x, vb[u].y, xa[u] & 0xFFu, xb[u] & 0xFFu, valid,
                  same_ts, far_all, tsa, tsb, warp, lane, lt_mask, qn, c);
      count_block(sm, va[u].z, va[u].w, vb[u].z, vb[u].w, xa[u] >> 8, xb[u] >> 8, valid, same_ts,
                  far_all, tsa, tsb, warp, lane, lt_mask, qn, c);
    }
  }
  if (nblk & 1) {  // a trailing odd block: warp 0 of CTA 0, lane 0
    if (blockIdx.x == 0 && warp == 0) {
      const int64_t i = nblk - 1;
      uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
      uint32_t x = 0u, y = 0u;
      if (lane == 0) {
        a = __ldg(reinterpret_cast<const uint2*>(ca) + i);
        b = __ldg(reinterpret_cast<const uint2*>(cb) + i);
        x = __ldg(sa + i);
        y = __ldg(sb + i);
      }
      count_block(sm, a.x, a.y, b.x, b.y, x, y, lane == 0, same_ts, far_all, tsa, tsb, warp, lane,
                  lt_mask, qn, c);
    }
  }
  stats_finish(sm, warp, lane, qn, c, stats8);
  if (blockIdx.x == 0 && t == 0) atomicAdd(stats8, (unsigned long long)nblk * 16ull);
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
