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
#include "umma.cuh"

namespace nvfp4 {

constexpr int kStatsCtasPerSm = 4;
[[maybe_unused]] constexpr int kStatsUnroll = 2;  // register form: two pairs (four blocks) in flight per lane

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

// The same counters with their inputs staged through shared memory: one
// producer warp streams chunks of kStatsChunk blocks (both sides' codes and
// scale bytes, four bulk copies per chunk) through a ring of stages, and
// each of the eight compute warps' threads takes one pair of adjacent blocks
// per chunk from shared memory, so no compute thread waits on a global load.
// The blocks after the last whole chunk are counted by CTA 0 with direct
// loads.  Every wait is bounded (2 s); a wait that gives up stops the CTA and
// sets bit 0 of stats8[7].
constexpr int kStatsChunk = 2 * kThreads;          // 512 blocks: one pair per compute thread
constexpr int kStatsStagedThreads = kThreads + 32;
#ifndef NVFP4_STATS_STAGES
#define NVFP4_STATS_STAGES 4
#endif
#ifndef NVFP4_STATS_CTAS
#define NVFP4_STATS_CTAS 4
#endif
constexpr int kStatsStages = NVFP4_STATS_STAGES;
constexpr int kStatsStagedCtas = NVFP4_STATS_CTAS;
constexpr uint32_t kSsCa = 0, kSsCb = kStatsChunk * 8, kSsSa = 2 * kStatsChunk * 8,
                   kSsSb = kSsSa + kStatsChunk, kSsPayload = kSsSb + kStatsChunk;
constexpr uint32_t kSsBytes = (kSsPayload + 127) / 128 * 128;
constexpr uint32_t kSsSmem = kStatsStages * kSsBytes + 128;

__global__ void __launch_bounds__(kStatsStagedThreads, kStatsStagedCtas)
    k_mismatch_stats_staged(const uint8_t* __restrict__ ca, const uint8_t* __restrict__ sa,
                            const float* __restrict__ ta, const uint8_t* __restrict__ cb,
                            const uint8_t* __restrict__ sb, const float* __restrict__ tb,
                            int64_t nblk, unsigned long long* __restrict__ stats8) {
  extern __shared__ __align__(128) uint8_t stage_smem[];
  __shared__ StatsShared sm;
  __shared__ int abort_flag;
  const uint32_t sbase = umma::smem_u32(stage_smem);
  const uint32_t full = sbase + kStatsStages * kSsBytes, empty = full + 8 * kStatsStages;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t nfull = nblk / kStatsChunk;
  const bool producer = warp == kWarps && lane == 0;
  auto load_chunk = [&](int64_t ch, int s) {
    const int64_t b0 = ch * kStatsChunk;
    const uint32_t bar = full + 8 * s, st = sbase + s * kSsBytes;
    umma::mbar_arrive_expect_tx(bar, kSsPayload);
    umma::bulk_load(st + kSsCa, ca + b0 * 8, kStatsChunk * 8, bar);
    umma::bulk_load(st + kSsCb, cb + b0 * 8, kStatsChunk * 8, bar);
    umma::bulk_load(st + kSsSa, sa + b0, kStatsChunk, bar);
    umma::bulk_load(st + kSsSb, sb + b0, kStatsChunk, bar);
  };
  // The producer sets up the ring and fills every stage before the CTA
  // builds its tables, so the first loads overlap that set-up.
  int64_t ch0 = blockIdx.x;
  int it0 = 0;
  if (producer) {
    for (int s = 0; s < kStatsStages; ++s) {
      umma::mbar_init(full + 8 * s, 1);
      umma::mbar_init(empty + 8 * s, kWarps);
    }
    abort_flag = 0;
    umma::fence_mbar_init();
    for (; it0 < kStatsStages && ch0 < nfull; ++it0, ch0 += gridDim.x) load_chunk(ch0, it0);
  }
  const float tsa = *ta, tsb = *tb;
  const bool same_ts = __float_as_uint(tsa) == __float_as_uint(tsb);
  const bool far_all = stats_tables_init(sm, tsa, tsb);  // ends in a barrier
  volatile int* abort = &abort_flag;
  MismatchCounts c{0u, 0u, 0u, 0u, 0u};
  int qn = 0;
  if (warp == kWarps) {
    if (producer) {
      int it = it0;
      for (int64_t ch = ch0; ch < nfull; ch += gridDim.x, ++it) {
        const int s = it % kStatsStages;
        const uint32_t ph = (uint32_t)(it / kStatsStages) & 1u;
        if (!umma::mbar_wait(empty + 8 * s, ph ^ 1u, abort)) break;
        load_chunk(ch, s);
      }
    }
    __syncwarp();
  } else {
    const uint32_t lt_mask = (1u << lane) - 1u;
    int it = 0;
    for (int64_t ch = blockIdx.x; ch < nfull; ch += gridDim.x, ++it) {
      const int s = it % kStatsStages;
      const uint32_t ph = (uint32_t)(it / kStatsStages) & 1u;
      const bool ok = umma::mbar_wait(full + 8 * s, ph, abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint8_t* st = stage_smem + s * kSsBytes;
      const uint4 va = *reinterpret_cast<const uint4*>(st + kSsCa + 16 * t);
      const uint4 vb = *reinterpret_cast<const uint4*>(st + kSsCb + 16 * t);
      const uint32_t xa = *reinterpret_cast<const uint16_t*>(st + kSsSa + 2 * t);
      const uint32_t xb = *reinterpret_cast<const uint16_t*>(st + kSsSb + 2 * t);
      count_block(sm, va.x, va.y, vb.x, vb.y, xa & 0xFFu, xb & 0xFFu, true, same_ts, far_all, tsa,
                  tsb, warp, lane, lt_mask, qn, c);
      count_block(sm, va.z, va.w, vb.z, vb.w, xa >> 8, xb >> 8, true, same_ts, far_all, tsa, tsb,
                  warp, lane, lt_mask, qn, c);
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(empty + 8 * s);
    }
    // blocks after the last whole chunk: CTA 0, direct loads, warps in step
    if (blockIdx.x == 0) {
      for (int64_t i0 = nfull * kStatsChunk + 32 * warp; i0 < nblk; i0 += kThreads) {
        const int64_t i = i0 + lane;
        const bool valid = i < nblk;
        uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
        uint32_t x = 0u, y = 0u;
        if (valid) {
          a = __ldg(reinterpret_cast<const uint2*>(ca) + i);
          b = __ldg(reinterpret_cast<const uint2*>(cb) + i);
          x = __ldg(sa + i);
          y = __ldg(sb + i);
        }
        count_block(sm, a.x, a.y, b.x, b.y, x, y, valid, same_ts, far_all, tsa, tsb, warp, lane,
                    lt_mask, qn, c);
      }
    }
  }
  stats_finish(sm, warp, lane, qn, c, stats8);
  if (blockIdx.x == 0 && t == 0) atomicAdd(stats8, (unsigned long long)nblk * 16ull);
  __syncthreads();
  if (*abort && t == 0) atomicOr(stats8 + 7, 1ull);
}

#ifndef NVFP4_STATS_STAGED
#define NVFP4_STATS_STAGED 1
#endif

cudaError_t launch_mismatch_stats(const uint8_t* ca, const uint8_t* sa, const float* ta,
                                  const uint8_t* cb, const uint8_t* sb, const float* tb,
                                  int64_t nblk, unsigned long long* stats8, cudaStream_t s) {
  if (nblk == 0) return cudaSuccess;
#if NVFP4_STATS_STAGED
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_mismatch_stats_staged, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSsSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int64_t chunks = nblk / kStatsChunk;
  const int64_t slots = (int64_t)sm_count() * kStatsStagedCtas;
  const int g = (int)(chunks < 1 ? 1 : (chunks < slots ? chunks : slots));
  k_mismatch_stats_staged<<<g, kStatsStagedThreads, kSsSmem, s>>>(ca, sa, ta, cb, sb, tb, nblk, stats8);
#else
  k_mismatch_stats<kStatsUnroll><<<grid_for(nblk, kThreads, kStatsCtasPerSm), kThreads, 0, s>>>(
      ca, sa, ta, cb, sb, tb, nblk, stats8);
#endif
  return cudaGetLastError();
}

}  // namespace nvfp4
