// stats.cu -- train/rollout mismatch counters between two NVFP4 tensors
// (TRACE explainer: the train/rollout distance is the quantity to shrink; the
// compaction paragraph observes that >99% of mismatches are one cell apart).
//
// One thread per 16-value block: 8 code bytes and 1 scale byte from each side.
// The kernel moves 1.125 bytes per element, so its integer work has to stay
// near 6 instructions per element to keep pace with HBM: positions are handled
// 8 nibbles at a time (SWAR) and |pos_a - pos_b| 4 bytes at a time.
//
// Decoded-value mismatches, exactly (decoded value = (G[m] * sb) * s_t in FP32):
//   * identical scales (same scale byte, same tensor scale) and all decoded
//     magnitudes normal: values differ exactly where positions differ;
//   * otherwise two nonzero values can only be equal if
//     (sb_a * s_t_a) / (sb_b * s_t_b) lies within ~2^-22 of a ratio of two
//     grid values, i.e. of 2^k, 3 * 2^k or 2^k / 3 (the grid is
//     {2^k, 3 * 2^k}).  When the ratio's significand is far from 1, 4/3 and
//     3/2, only zero/zero pairs are equal;
//   * any other block falls back to the element-by-element FP32 comparison.
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kStatsCtasPerSm = 4;
constexpr int kStatsUnroll = 4;

struct MismatchCounts {
  uint32_t mism, far, sumd, scale, value;
};

// 8 codes -> 8 offset positions 8 + pos in [1, 15] (+0 and -0 both give 8).
__device__ __forceinline__ uint32_t offset_pos(uint32_t w) {
  const uint32_t M = w & 0x77777777u;
  const uint32_t K = ((w >> 3) & 0x11111111u) * 7u;  // 7 in negative nibbles
  return ((M ^ K) + 0x88888888u) - K;                // s ? 8 - m : 8 + m
}

// bit 0 of each nibble: nibble nonzero.
__device__ __forceinline__ uint32_t nib_nonzero(uint32_t t) {
  t |= t >> 1;
  t |= t >> 2;
  return t & 0x11111111u;
}

// |a - b| for 4 byte lanes holding values in [1, 15].
__device__ __forceinline__ uint32_t absdiff_bytes(uint32_t a, uint32_t b) {
  const uint32_t t = (a | 0x10101010u) - b;          // 16 + a - b in [2, 30]
  const uint32_t ng = ((t >> 4) & 0x01010101u) ^ 0x01010101u;  // a < b
  return ((t ^ (ng * 0x0Fu)) & 0x0F0F0F0Fu) + ng;
}

// Counts for one word of 8 elements; returns the nibble mask of positions
// that differ (bit 0 per nibble).
__device__ __forceinline__ uint32_t mismatch_word(uint32_t wa, uint32_t wb, MismatchCounts& c) {
  const uint32_t pa = offset_pos(wa), pb = offset_pos(wb);
  const uint32_t diff = nib_nonzero(pa ^ pb);
  const uint32_t d_even = absdiff_bytes(pa & 0x0F0F0F0Fu, pb & 0x0F0F0F0Fu);
  const uint32_t d_odd = absdiff_bytes((pa >> 4) & 0x0F0F0F0Fu, (pb >> 4) & 0x0F0F0F0Fu);
  c.sumd = __dp4a(d_even + d_odd, 0x01010101u, c.sumd);  // each byte sum <= 28
  const uint32_t far_e = ((d_even & 0x0E0E0E0Eu) + 0x7F7F7F7Fu) & 0x80808080u;
  const uint32_t far_o = ((d_odd & 0x0E0E0E0Eu) + 0x7F7F7F7Fu) & 0x80808080u;
  c.far += __popc(far_e | (far_o >> 1));
  c.mism += __popc(diff);
  return diff;
}

__device__ __forceinline__ bool near_grid_ratio(float rho) {
  const int f = (int)(__float_as_uint(rho) & 0x7FFFFFu);  // significand bits
  const int tol = 64;                                      // 2^-17 relative
  return f < tol || f > 0x800000 - tol || abs(f - 0x2AAAAB) < tol || abs(f - 0x400000) < tol;
}

__device__ __forceinline__ uint32_t value_mismatch_slow(uint2 a, uint2 b, float sva, float svb,
                                                        float tsa, float tsb) {
  uint32_t n = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t wa = half ? a.y : a.x, wb = half ? b.y : b.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float ga[2], gb[2];
      e2m1x2_decode((wa >> (8 * j)) & 0xFFu, ga[0], ga[1]);
      e2m1x2_decode((wb >> (8 * j)) & 0xFFu, gb[0], gb[1]);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        n += (__fmul_rn(__fmul_rn(ga[t], sva), tsa) != __fmul_rn(__fmul_rn(gb[t], svb), tsb)) ? 1u : 0u;
    }
  }
  return n;
}

__device__ __forceinline__ void mismatch_block(uint2 a, uint2 b, uint32_t sba, uint32_t sbb,
                                               float tsa, float tsb, bool same_ts,
                                               MismatchCounts& c) {
  c.scale += (sba != sbb) ? 1u : 0u;
  const uint32_t d0 = mismatch_word(a.x, b.x, c);
  const uint32_t d1 = mismatch_word(a.y, b.y, c);
  const float sva = e4m3_value(sba), svb = e4m3_value(sbb);
  const float xa = __fmul_rn(sva, tsa), xb = __fmul_rn(svb, tsb);
  // every nonzero decoded value is a normal float (no underflow, no overflow)
  const bool normal = xa >= 0x1p-124f && xb >= 0x1p-124f && xa <= 0x1p120f && xb <= 0x1p120f;
  uint32_t value;
  if (normal && same_ts && sba == sbb) {
    value = __popc(d0) + __popc(d1);
  } else if (normal && !near_grid_ratio(__fdividef(xa, xb))) {
    // only zero/zero pairs can be equal
    const uint32_t nz0 = nib_nonzero((a.x | b.x) & 0x77777777u);
    const uint32_t nz1 = nib_nonzero((a.y | b.y) & 0x77777777u);
    value = __popc(nz0) + __popc(nz1);
  } else {
    value = value_mismatch_slow(a, b, sva, svb, tsa, tsb);
  }
  c.value += value;
}

template <int U>
__global__ void __launch_bounds__(kThreads, kStatsCtasPerSm)
    k_mismatch_stats(const uint8_t* __restrict__ ca, const uint8_t* __restrict__ sa,
                     const float* __restrict__ ta, const uint8_t* __restrict__ cb,
                     const uint8_t* __restrict__ sb, const float* __restrict__ tb, int64_t nblk,
                     unsigned long long* __restrict__ stats8) {
  __shared__ unsigned long long red[6 * 8];
  const float tsa = *ta, tsb = *tb;
  const bool same_ts = __float_as_uint(tsa) == __float_as_uint(tsb);
  MismatchCounts c{0u, 0u, 0u, 0u, 0u};
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
    for (int u = 0; u < U; ++u) mismatch_block(va[u], vb[u], xa[u], xb[u], tsa, tsb, same_ts, c);
  }
  for (; i < nblk; i += stride)
    mismatch_block(__ldg(a2 + i), __ldg(b2 + i), __ldg(sa + i), __ldg(sb + i), tsa, tsb, same_ts, c);
  const unsigned long long vals[6] = {c.mism, (unsigned long long)(c.mism - c.far), c.far, c.sumd,
                                      c.scale, c.value};
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
