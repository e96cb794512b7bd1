// stats_device.cuh -- the mismatch counters between two NVFP4 tensors, as
// device building blocks shared by the standalone counter kernel (stats.cu)
// and the guided re-quantization that counts while it quantizes
// (quantize.cu).  How the counting works is described in stats.cu.
#pragma once

#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kWarps = kThreads / 32;
constexpr int kQueue = 64;  // dirty-block slots per warp (at most 31 + 32 are ever held)

struct MismatchCounts {
  uint32_t mism, far, sumd, scale, value;
};

// Number of set bits of a mask that only uses bit 7 of each byte.
__device__ __forceinline__ uint32_t count_byte_msb(uint32_t m) { return ((m >> 7) * 0x01010101u) >> 24; }

// 8 codes -> 8 offset positions 8 + pos in [1, 15] (+0 and -0 both give 8).
__device__ __forceinline__ uint32_t offset_pos(uint32_t w) {
  const uint32_t M = w & 0x77777777u;
  const uint32_t K = ((w >> 3) & 0x11111111u) * 7u;  // 7 in negative nibbles
  return ((M ^ K) + 0x88888888u) - K;                // s ? 8 - m : 8 + m
}

// |a - b| for 4 byte lanes holding values in [1, 15].
__device__ __forceinline__ uint32_t absdiff_bytes(uint32_t a, uint32_t b) {
  const uint32_t t = (a | 0x10101010u) - b;                     // 16 + a - b in [2, 30]
  const uint32_t ng = ((t >> 4) & 0x01010101u) ^ 0x01010101u;  // a < b
  return ((t ^ (ng * 0x0Fu)) & 0x0F0F0F0Fu) + ng;
}

// Position counters of one word (8 elements); returns the number of
// positions that differ.
__device__ __forceinline__ uint32_t position_word(uint32_t wa, uint32_t wb, MismatchCounts& c) {
  const uint32_t pa = offset_pos(wa), pb = offset_pos(wb);
  const uint32_t n = count_nib(nib_nonzero(pa ^ pb));
  const uint32_t d_even = absdiff_bytes(pa & 0x0F0F0F0Fu, pb & 0x0F0F0F0Fu);
  const uint32_t d_odd = absdiff_bytes((pa >> 4) & 0x0F0F0F0Fu, (pb >> 4) & 0x0F0F0F0Fu);
  c.sumd = __dp4a(d_even + d_odd, 0x01010101u, c.sumd);  // each byte sum <= 28
  const uint32_t far_e = ((d_even & 0x0E0E0E0Eu) + 0x7F7F7F7Fu) & 0x80808080u;
  const uint32_t far_o = ((d_odd & 0x0E0E0E0Eu) + 0x7F7F7F7Fu) & 0x80808080u;
  c.far += count_byte_msb(far_e) + count_byte_msb(far_o);
  c.mism += n;
  return n;
}

__device__ __forceinline__ bool near_grid_ratio(float rho) {
  const int f = (int)(__float_as_uint(rho) & 0x7FFFFFu);  // significand bits
  const int tol = 64;                                      // 2^-17 relative
  return f < tol || f > 0x800000 - tol || abs(f - 0x2AAAAB) < tol || abs(f - 0x400000) < tol;
}

// Integer significand of an E4M3 byte: 8 + mantissa (normal) or mantissa.
__device__ __forceinline__ uint32_t e4m3_significand(uint32_t b) {
  return (b & 7u) | ((b & 0x78u) ? 8u : 0u);
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

struct StatsShared {
  uint4 queue[kWarps][kQueue];
  uint8_t queue_same[kWarps][kQueue];  // value counter follows positions
  // per scale byte: 16 * significand (side a) / significand (side b) when every
  // nonzero decoded value of such a block is a normal float, else 0x100
  uint16_t key_a[128], key_b[128];
  uint8_t ratio_far[256];  // [key_a + key_b]: only zero/zero pairs can be equal
  unsigned long long red[6 * 8];
};

// Lane `lane` takes queue slot `lane` (if < n) and counts it; the slots
// n..qn-1 then move to the front.  Returns the new queue length.
__device__ __forceinline__ int flush_queue(StatsShared& sm, int warp, int lane, int qn, int n,
                                           MismatchCounts& c) {
  __syncwarp();
  if (lane < n) {
    const uint4 e = sm.queue[warp][lane];
    const uint32_t mb = position_word(e.x, e.z, c) + position_word(e.y, e.w, c);
    if (sm.queue_same[warp][lane]) c.value += mb;
  }
  __syncwarp();
  const int rest = qn - n;
  if (lane < rest) {
    sm.queue[warp][lane] = sm.queue[warp][n + lane];
    sm.queue_same[warp][lane] = sm.queue_same[warp][n + lane];
  }
  __syncwarp();
  return rest;
}

// Elements of a block (words x, y of both sides) whose magnitudes are not
// both zero: bit 3 of each nibble of ((a | b) & 7) + 7 flags the first word's
// elements, the second word's flags move to bit 2, one popc counts both.
__device__ __forceinline__ uint32_t not_both_zero2(uint32_t ax, uint32_t ay, uint32_t bx, uint32_t by) {
  const uint32_t f0 = (((ax | bx) & 0x77777777u) + 0x77777777u) & 0x88888888u;
  const uint32_t f1 = ((((ay | by) & 0x77777777u) + 0x77777777u) >> 1) & 0x44444444u;
  return __popc(f0 | f1);
}

// One block of the stream: count its scale and (unless positions decide it)
// its decoded-value mismatches, and queue it if its codes differ.
// far_all: CTA-uniform, the tensor scales differ and every pair of nonzero
// scale bytes is regular and far from a grid ratio.  The common case -- both
// scales nonzero under far_all, and no block of the warp step differing --
// takes no table lookup and no queue work.
__device__ __forceinline__ void count_block(StatsShared& sm, uint32_t ax, uint32_t ay, uint32_t bx,
                                            uint32_t by, uint32_t sa, uint32_t sb, bool valid,
                                            bool same_ts, bool far_all, float tsa, float tsb,
                                            int warp, int lane, uint32_t lt_mask, int& qn,
                                            MismatchCounts& c) {
  sa &= 0x7Fu;
  sb &= 0x7Fu;
  const bool fast = far_all && sa != 0u && sb != 0u;
  bool same = false;
  if (fast) {
    if (valid) {
      c.scale += (sa != sb) ? 1u : 0u;
      c.value += not_both_zero2(ax, ay, bx, by);  // only zero pairs are equal
    }
  } else {
    const uint32_t ka = sm.key_a[sa], kb = sm.key_b[sb];
    same = same_ts && sa == sb && ka < 0x100u;
    if (valid) {
      c.scale += (sa != sb) ? 1u : 0u;
      if (!same) {
        const uint32_t k = ka + kb;
        if (k < 0x100u && sm.ratio_far[k]) {
          c.value += not_both_zero2(ax, ay, bx, by);
        } else {
          c.value += value_mismatch_slow(make_uint2(ax, ay), make_uint2(bx, by), e4m3_value(sa),
                                         e4m3_value(sb), tsa, tsb);
        }
      }
    }
  }
  const bool dirty = ((ax ^ bx) | (ay ^ by)) != 0u;
  const uint32_t m = __ballot_sync(0xFFFFFFFFu, dirty);
  if (m != 0u) {  // warp-uniform
    if (dirty) {
      const int slot = qn + __popc(m & lt_mask);
      sm.queue[warp][slot] = make_uint4(ax, ay, bx, by);
      sm.queue_same[warp][slot] = same;
    }
    qn += __popc(m);
    if (qn >= 32) qn = flush_queue(sm, warp, lane, qn, 32, c);
  }
}

// Per-CTA tables of the decoded-value counter for tensor scales tsa (side
// a) and tsb (side b); returns the CTA-uniform far_all flag (see count_block).
// Every thread of the CTA calls it (it ends in a barrier); threads 0..255
// cover the 256 significand pairs, any further threads only vote.
__device__ __forceinline__ bool stats_tables_init(StatsShared& sm, float tsa, float tsb) {
  const bool same_ts = __float_as_uint(tsa) == __float_as_uint(tsb);
  const int t = threadIdx.x < 256 ? (int)threadIdx.x : 0;
  if (threadIdx.x < 128) {
    const float sv = e4m3_value(t);
    const float xa = __fmul_rn(sv, tsa), xb = __fmul_rn(sv, tsb);
    // every nonzero decoded value of the block is a normal float
    const uint32_t sig = e4m3_significand(t);
    sm.key_a[t] = (xa >= 0x1p-124f && xa <= 0x1p120f) ? (uint16_t)(sig << 4) : (uint16_t)0x100;
    sm.key_b[t] = (xb >= 0x1p-124f && xb <= 0x1p120f) ? (uint16_t)sig : (uint16_t)0x100;
  }
  bool ok = true;
  {
    // significand of (sb_a * s_t_a) / (sb_b * s_t_b) for scale significands
    // ma, mb (powers of two do not change it); approximate to a few ulps,
    // far below the 2^-17 tolerance of near_grid_ratio
    const uint32_t ma = (uint32_t)t >> 4, mb = (uint32_t)t & 15u;
    const float tr = __fdiv_rn(tsa, tsb);
    bool far_ratio = false;
    if (ma != 0u && mb != 0u && tr >= 0x1p-120f && tr <= 0x1p120f)
      far_ratio = !near_grid_ratio(__fmul_rn(__fdiv_rn((float)ma, (float)mb), tr));
    if (threadIdx.x < 256) sm.ratio_far[t] = far_ratio;
    // the CTA-wide shortcut: every nonzero significand pair far, every
    // nonzero scale byte regular on both sides
    ok = (ma == 0u || mb == 0u || far_ratio);
  }
  if (threadIdx.x < 128 && t != 0) {
    const float sv = e4m3_value(t);
    const float xa = __fmul_rn(sv, tsa), xb = __fmul_rn(sv, tsb);
    ok = ok && xa >= 0x1p-124f && xa <= 0x1p120f && xb >= 0x1p-124f && xb <= 0x1p120f;
  }
  return __syncthreads_and(ok && !same_ts) != 0;
}

// Empties the warp's queue and adds the CTA's six counters to stats8[1..6]
// (every thread of the CTA calls it; warps from kWarps on only take part in
// the barrier).
__device__ __forceinline__ void stats_finish(StatsShared& sm, int warp, int lane, int qn,
                                             MismatchCounts& c, unsigned long long* stats8) {
  if (qn > 0) flush_queue(sm, warp, lane, qn, qn, c);
  const unsigned long long vals[6] = {c.mism, (unsigned long long)(c.mism - c.far), c.far, c.sumd,
                                      c.scale, c.value};
  block_add_u64<6, kWarps>(vals, stats8 + 1, sm.red);
}

}  // namespace nvfp4
