// quantize.cu -- streaming NVFP4 kernels over BF16 tensors (sm_100a):
//   * tensor amax                       (TRACE explainer: each side scales its own values)
//   * round-to-nearest quantize + fused hint emit   (rollout side)
//   * guided re-quantize + counters     (train side; TRACE explainer,
//                                        prescription and compaction paragraphs)
//   * standalone hint emit from codes
//
// Data layout: the tensor is a flat sequence of 16-value blocks (rows * cols / 16
// of them, cols % 16 == 0), so every kernel streams blocks: one thread owns one
// block, reads its 32 bytes with a single 256-bit load and writes 8 bytes of
// codes, 1 scale byte and 2/4/8 bytes of hints.  A warp therefore moves 1 KiB of
// input and 256 B of codes per step, fully coalesced.  Grids are persistent
// (a fixed number of CTAs per SM, grid-stride), each thread keeps U blocks in
// flight.  HBM-bound: no tensor cores.
#include "launch.h"
#include "nvfp4_device.cuh"
#include "stats_device.cuh"
#include "umma.cuh"

namespace nvfp4 {

#ifndef NVFP4_STREAM_CTAS
#define NVFP4_STREAM_CTAS 4
#endif
#ifndef NVFP4_STREAM_UNROLL
#define NVFP4_STREAM_UNROLL 2
#endif
#ifndef NVFP4_GUIDED_UNROLL
#define NVFP4_GUIDED_UNROLL 3   // guided alone: three blocks in flight per thread (measured best)
#endif
constexpr int kCtasPerSm = NVFP4_STREAM_CTAS;
constexpr int kUnroll = NVFP4_STREAM_UNROLL;
constexpr int kGuidedUnroll = NVFP4_GUIDED_UNROLL;
constexpr int kAmaxUnroll = 4;  // 128 bytes in flight per thread: the amax pass has no other work

// ----------------------------------------------------------------- amax
// Max of |x| over BF16 magnitudes: |x| is the 15 low bits, and for non-negative
// values the bit patterns order like the numbers, so an unsigned max on packed
// 16-bit halves is exact.  Result: FP32 bits of A in ws[0] and
// NVFP4_WARN_NONFINITE in ws[1] when an Inf/NaN pattern was seen, published by
// the last CTA to finish (grid_max_publish: no clearing pass before it).
template <int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_amax_bf16(const uint16_t* __restrict__ x, int64_t nblk, uint32_t* __restrict__ ws) {
  __shared__ uint32_t red[kThreads / 32];
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  uint32_t m2 = 0;  // two packed 16-bit maxima
  for (; i + (U - 1) * stride < nblk; i += U * stride) {
    Block16 b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) b[u] = ld_block(x + (i + u * stride) * 16);
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int k = 0; k < 8; ++k) m2 = __vmaxu2(m2, b[u].w[k] & 0x7FFF7FFFu);
  }
  for (; i < nblk; i += stride) {
    Block16 b = ld_block(x + i * 16);
#pragma unroll
    for (int k = 0; k < 8; ++k) m2 = __vmaxu2(m2, b.w[k] & 0x7FFF7FFFu);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16) << 16;  // FP32 bits of the max magnitude
  m = block_max_u32(m, red);
  if (threadIdx.x == 0) grid_max_publish(ws, m);
}

// Hint bits of one block (16 codes) from its 8 code bytes.
template <int HB>
__device__ __forceinline__ void hint_store(uint8_t* __restrict__ hints, int64_t blk, uint2 c) {
  if (HB == 1) reinterpret_cast<uint16_t*>(hints)[blk] = (uint16_t)hint_field1(c);
  if (HB == 2) reinterpret_cast<uint32_t*>(hints)[blk] = hint_field2(c);
  if (HB == 4) reinterpret_cast<uint2*>(hints)[blk] = c;
}

// ----------------------------------------------------------------- RTN quantize
template <int HB>
__device__ __forceinline__ void rtn_block_scaled(const Block16& b, BlockScale bs, int64_t blk,
                                                 uint8_t* __restrict__ codes,
                                                 uint8_t* __restrict__ scales,
                                                 uint8_t* __restrict__ hints) {
  uint2 c;
  if (inv_overflowed(bs.inv)) {
    c = overflow_codes_bf16(b);
  } else {
    float x[16];
    unpack_block(b, x);
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(x[k], bs.inv);
    c = pack_codes16(v);
  }
  reinterpret_cast<uint2*>(codes)[blk] = c;
  scales[blk] = (uint8_t)bs.sb;
  hint_store<HB>(hints, blk, c);
}

template <int HB>
__device__ __forceinline__ void rtn_block(const Block16& b, float s_t, const ScaleTables& tab,
                                          int64_t blk, uint8_t* __restrict__ codes,
                                          uint8_t* __restrict__ scales,
                                          uint8_t* __restrict__ hints) {
  rtn_block_scaled<HB>(b, block_scale_bf16(block_amax_bits(b), s_t, tab), blk, codes, scales, hints);
}

// Blocks are visited from the END of the tensor backwards: the amax pass that
// runs just before streams forwards, so the tail it read last is still in L2.
template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_quantize_rtn(const uint16_t* __restrict__ x, int64_t nblk, const uint32_t* __restrict__ ws,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   float* __restrict__ tensor_scale, uint8_t* __restrict__ hints) {
  __shared__ ScaleTables tab;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  // the first step's loads are issued before the tables are built
  Block16 b[U];
  bool step = i + (U - 1) * stride < nblk;
  if (step) {
#pragma unroll
    for (int u = 0; u < U; ++u) b[u] = ld_block(x + (nblk - 1 - (i + u * stride)) * 16);
  }
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  while (step) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      rtn_block<HB>(b[u], s_t, tab, nblk - 1 - (i + u * stride), codes, scales, hints);
    i += U * stride;
    step = i + (U - 1) * stride < nblk;
    if (step) {
#pragma unroll
      for (int u = 0; u < U; ++u) b[u] = ld_block(x + (nblk - 1 - (i + u * stride)) * 16);
    }
  }
  for (; i < nblk; i += stride)
    rtn_block<HB>(ld_block(x + (nblk - 1 - i) * 16), s_t, tab, nblk - 1 - i, codes, scales, hints);
}

// ----------------------------------------------------------------- guided
// Per element, with v = x * inv, a = |v| and m the round-to-nearest magnitude:
//   a off the grid and below 6 -> it lies in (G[lo], G[lo+1]) with lo the
//       floor index, and m is lo or lo + 1;  the other end of that bracket
//       replaces m when the hint names it;
//   a on the grid (zero included) or above 6 -> no decision, m stays.
// HB = 1, 2: magnitude bits modulo 2^HB.  HB = 4: signed grid positions.
// Everything runs on packed words of 8 nibbles:
//   R  = round-to-nearest codes of v (hardware conversion, sign of x);
//   Zs = codes of v rounded toward zero: the floor index lo with the sign;
//   P  = the same for v moved one ulp toward zero (its bit pattern minus 1).
//        Off the grid that cannot cross a grid point, so P == Zs; on a grid
//        point the magnitude drops one cell; v = +-0 turns into a NaN pattern,
//        which converts to magnitude 7.  So P != Zs (in magnitude) marks "no
//        decision" exactly where a is on the grid.
// Off the grid the other bracket end is O = 2 * lo + 1 - m; a > 6 gives
// lo = m = 7 and O = 8, which also means no decision.  Per-element flags live
// in bit 3 of each nibble: a nibble value in 0..8 is nonzero exactly when
// adding 7 sets its bit 3 (no carry leaves the nibble).
struct GuidedCounts {
  uint32_t consulted, changed, outside;  // per thread: at most 16 per block visited
};

// hword: for HB = 1, 2 the hint fields of these 8 elements in the low bits of
// each nibble (higher nibble bits are ignored); for HB = 4 their full codes.
template <int HB>
__device__ __forceinline__ uint32_t guided_select(uint32_t R, uint32_t Zm, uint32_t pz,
                                                  uint32_t hword, GuidedCounts& cnt) {
  constexpr uint32_t kB3 = 0x88888888u, kSeven = 0x77777777u;
  const uint32_t M = R & kSeven;  // round-to-nearest magnitudes
  const uint32_t O = (Zm << 1) + 0x11111111u - M;
  const uint32_t off = ~((pz + kSeven) | O) & kB3;  // a rounding decision exists
  uint32_t take, differs;  // differs: the hint does not name the round-to-nearest cell
  if (HB == 4) {
    // signed positions: equal codes, or both magnitudes zero
    const auto nz4 = [](uint32_t t) { return (((t & kSeven) + kSeven) | t) & kB3; };
    const uint32_t zh = ~((hword & kSeven) + kSeven);
    take = ~nz4(hword ^ (O | (R & kB3))) | (~(O + kSeven) & zh);
    differs = nz4(hword ^ R) & ((M + kSeven) | ~zh);
  } else {
    const uint32_t mask = HB == 1 ? 0x11111111u : 0x33333333u;
    take = ~(((hword ^ O) & mask) + kSeven);
    differs = ((hword ^ M) & mask) + kSeven;
  }
  take &= off;
  cnt.consulted += __popc(off);
  cnt.changed += __popc(take);
  cnt.outside += __popc(off & ~take & differs);
  // magnitude-bit select mask: 7 in every nibble whose bit 3 is set in take,
  // (take * 7) >> 3 taken from the high word of take * (7 << 29)
  const uint32_t T = __umulhi(take, 0xE0000000u);
  return (R & ~T) | (O & T);  // the sign bits of R stay
}

template <int HB>
__device__ __forceinline__ uint32_t hint_field(const uint8_t* __restrict__ hints, int64_t blk,
                                               uint2& h4) {
  if (HB == 1) return reinterpret_cast<const uint16_t*>(hints)[blk];
  if (HB == 2) return reinterpret_cast<const uint32_t*>(hints)[blk];
  h4 = reinterpret_cast<const uint2*>(hints)[blk];
  return 0;
}

// The guided codes of one block given its reciprocal scale inv (no stores).
template <int HB>
__device__ __forceinline__ uint2 guided_codes(const Block16& b, uint32_t hw, uint2 h4, float inv,
                                              GuidedCounts& cnt, uint32_t one) {
  if (inv_overflowed(inv)) return overflow_codes_bf16(b);  // every element saturated or zero: no decision
  float x[16];
  unpack_block(b, x);
  const uint32_t h1 = HB == 1 ? hint_spread1(hw) : 0u;
  uint32_t out[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[8], p[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      v[t] = __fmul_rn(x[8 * half + t], inv);
      // one ulp toward zero: bits * one - 1 with one == 1 known only at run
      // time, so it issues as a multiply-add on the FP pipe
      p[t] = __uint_as_float(__float_as_uint(v[t]) * one + 0xFFFFFFFFu);
    }
    const uint32_t R = pack_rn8(v);
    const uint32_t Zs = pack_rz8(v);
    const uint32_t pz = (pack_rz8(p) ^ Zs) & 0x77777777u;
    uint32_t hword;
    if (HB == 4) hword = half ? h4.y : h4.x;
    else if (HB == 2) hword = half ? (hw >> 2) : hw;
    else hword = half ? (h1 >> 1) : h1;
    out[half] = guided_select<HB>(R, Zs & 0x77777777u, pz, hword, cnt);
  }
  return make_uint2(out[0], out[1]);
}

// The round-to-nearest codes of one block given inv (no stores).
__device__ __forceinline__ uint2 rtn_codes(const Block16& b, float inv) {
  if (inv_overflowed(inv)) return overflow_codes_bf16(b);
  float x[16];
  unpack_block(b, x);
  float v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(x[k], inv);
  return pack_codes16(v);
}

template <int HB>
__device__ __forceinline__ void guided_block_scaled(const Block16& b, uint32_t hw, uint2 h4,
                                                    BlockScale bs, int64_t blk,
                                                    uint8_t* __restrict__ codes,
                                                    uint8_t* __restrict__ scales, GuidedCounts& cnt,
                                                    uint32_t one) {
  reinterpret_cast<uint2*>(codes)[blk] = guided_codes<HB>(b, hw, h4, bs.inv, cnt, one);
  scales[blk] = (uint8_t)bs.sb;
}

template <int HB>
__device__ __forceinline__ void guided_block(const Block16& b, uint32_t hw, uint2 h4, float s_t,
                                             const ScaleTables& tab, int64_t blk,
                                             uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales, GuidedCounts& cnt,
                                             uint32_t one) {
  guided_block_scaled<HB>(b, hw, h4, block_scale_bf16(block_amax_bits(b), s_t, tab), blk, codes,
                          scales, cnt, one);
}

template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_guided(const uint16_t* __restrict__ x, int64_t nblk, const uint8_t* __restrict__ hints,
             const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
             unsigned long long* __restrict__ stats4, uint32_t one) {
  __shared__ unsigned long long red[3 * 8];
  __shared__ ScaleTables tab;
  GuidedCounts cnt{0u, 0u, 0u};
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  Block16 b[U];
  uint32_t hw[U];
  uint2 h4[U];
  auto load_step = [&]() {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = nblk - 1 - (i + u * stride);
      b[u] = ld_block(x + blk * 16);
      hw[u] = hint_field<HB>(hints, blk, h4[u]);
    }
  };
  // the first step's loads are issued before the tables are built
  bool step = i + (U - 1) * stride < nblk;
  if (step) load_step();
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  while (step) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      guided_block<HB>(b[u], hw[u], h4[u], s_t, tab, nblk - 1 - (i + u * stride), codes, scales, cnt,
                       one);
    i += U * stride;
    step = i + (U - 1) * stride < nblk;
    if (step) load_step();
  }
  for (; i < nblk; i += stride) {
    const int64_t blk = nblk - 1 - i;
    uint2 h4;
    const uint32_t hw = hint_field<HB>(hints, blk, h4);
    guided_block<HB>(ld_block(x + blk * 16), hw, h4, s_t, tab, blk, codes, scales, cnt, one);
  }
  if (stats4 != nullptr) {
    const unsigned long long vals[3] = {cnt.consulted, cnt.changed, cnt.outside};
    block_add_u64<3>(vals, stats4, red);
  }
}

// ----------------------------------------------------------------- guided + counters
// The train side's guided re-quantization (round-to-nearest for HB = 0) that
// also counts the mismatches against the rollout's NVFP4 tensor while it has
// its own codes in registers: the counters of nvfp4_mismatch_stats (side a =
// rollout, side b = train) without writing the train codes and reading them
// back.  Per block it reads the rollout's 8 code bytes and scale byte beside
// its own inputs.  The loop runs warp-uniformly (the counters' dirty-block
// queue needs every lane of the warp); a lane past the end counts a block of
// zeros against zeros, which adds nothing.
#ifndef NVFP4_GS_CTAS
#define NVFP4_GS_CTAS 4
#endif
#ifndef NVFP4_GS_UNROLL
#define NVFP4_GS_UNROLL 2
#endif
constexpr int kGsCtasPerSm = NVFP4_GS_CTAS;
[[maybe_unused]] constexpr int kGsUnroll = NVFP4_GS_UNROLL;  // register form only

template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kGsCtasPerSm)
    k_guided_stats(const uint16_t* __restrict__ x, int64_t nblk, const uint8_t* __restrict__ hints,
                   const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
                   unsigned long long* __restrict__ stats4, const uint8_t* __restrict__ rcodes,
                   const uint8_t* __restrict__ rscales, const float* __restrict__ rts,
                   unsigned long long* __restrict__ stats8, uint32_t one) {
  __shared__ ScaleTables tab;
  __shared__ StatsShared sm;
  __shared__ unsigned long long red4[3 * 8];
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  const float ts_r = *rts;
  const bool same_ts = __float_as_uint(ts_r) == __float_as_uint(s_t);
  const bool far_all = stats_tables_init(sm, ts_r, s_t);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  GuidedCounts gcnt{0u, 0u, 0u};
  MismatchCounts mc{0u, 0u, 0u, 0u, 0u};
  int qn = 0;  // warp-uniform queue length
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t base = (int64_t)blockIdx.x * kThreads + warp * 32; base < nblk; base += U * stride) {
    Block16 b[U];
    uint32_t hw[U], rs[U];
    uint2 h4[U], rc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + u * stride + lane;
      const int64_t blk = nblk - 1 - i;  // backwards, as the other quantizers
      b[u] = Block16{};
      hw[u] = 0u;
      h4[u] = rc[u] = make_uint2(0u, 0u);
      rs[u] = 0u;
      if (i < nblk) {
        b[u] = ld_block(x + blk * 16);
        if constexpr (HB != 0) hw[u] = hint_field<HB>(hints, blk, h4[u]);
        rc[u] = __ldg(reinterpret_cast<const uint2*>(rcodes) + blk);
        rs[u] = __ldg(rscales + blk);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + u * stride + lane;
      const bool valid = i < nblk;
      const int64_t blk = nblk - 1 - i;
      uint2 c = make_uint2(0u, 0u);
      uint32_t sb = 0u;
      if (valid) {
        const BlockScale bs = block_scale_bf16(block_amax_bits(b[u]), s_t, tab);
        if constexpr (HB != 0) c = guided_codes<HB>(b[u], hw[u], h4[u], bs.inv, gcnt, one);
        else c = rtn_codes(b[u], bs.inv);
        sb = bs.sb;
        reinterpret_cast<uint2*>(codes)[blk] = c;
        scales[blk] = (uint8_t)sb;
      }
      count_block(sm, rc[u].x, rc[u].y, c.x, c.y, rs[u], sb, valid, same_ts, far_all, ts_r, s_t,
                  warp, lane, lt_mask, qn, mc);
    }
  }
  stats_finish(sm, warp, lane, qn, mc, stats8);
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(stats8, (unsigned long long)nblk * 16ull);
  if (HB != 0 && stats4 != nullptr) {
    const unsigned long long vals[3] = {gcnt.consulted, gcnt.changed, gcnt.outside};
    block_add_u64<3>(vals, stats4, red4);
  }
}

// ----------------------------------------------------------------- staged guided (+ counters)
// The guided pass with its inputs staged through shared memory by bulk
// copies: one producer warp streams chunks of kStageBlocks blocks (their BF16
// values, hint fields and, with counters, the rollout's codes and scale
// bytes) through a ring of shared-memory stages with cp.async.bulk (one copy
// per input stream and chunk, completion counted on an mbarrier), and eight
// compute warps take kGuidedBpt blocks per thread from shared memory.  Global-memory
// latency is hidden by the ring instead of by registers, so the compute
// threads never wait on a load and keep the logic pipe busy.  Chunk c holds
// blocks kStageBlocks * c .. + kStageBlocks - 1 (so every copy starts on a
// 16-byte boundary, whatever the tensor size); the chunks are visited from
// the end of the tensor backwards (the amax pass just read its tail), and
// the blocks after the last whole chunk (nblk % kStageBlocks of them) are
// done first, by CTA 0, with direct loads.  Every wait is bounded (2 s); a
// wait that gives up stops the CTA and sets NVFP4_WARN_TIMEOUT in ws[1].
// HB = 0 (with counters only): round-to-nearest codes.
#ifndef NVFP4_GUIDED_BPT
#define NVFP4_GUIDED_BPT 2
#endif
#ifndef NVFP4_GUIDED_STAGES
#define NVFP4_GUIDED_STAGES 2
#endif
#ifndef NVFP4_GUIDED_CTAS
#define NVFP4_GUIDED_CTAS 3
#endif
constexpr int kGuidedBpt = NVFP4_GUIDED_BPT;        // blocks per compute thread and chunk
constexpr int kStageBlocks = kThreads * kGuidedBpt; // blocks per chunk
constexpr int kComputeWarps = kThreads / 32;        // 8
constexpr int kStagedThreads = kThreads + 32;       // + the producer warp
constexpr int kGuidedStages = NVFP4_GUIDED_STAGES;
constexpr int kGuidedCtas = NVFP4_GUIDED_CTAS;

template <int HB, bool STATS>
struct GuidedStage {
  static constexpr uint32_t kHintBytes = HB == 0 ? 0u : (HB == 4 ? 8u : (uint32_t)HB * 2u);  // per block
  static constexpr uint32_t x = 0;
  static constexpr uint32_t hints = x + kStageBlocks * 32;
  static constexpr uint32_t rc = hints + kStageBlocks * kHintBytes;
  static constexpr uint32_t rs = rc + (STATS ? kStageBlocks * 8 : 0);
  static constexpr uint32_t payload = rs + (STATS ? kStageBlocks : 0);
  static constexpr uint32_t bytes = (payload + 127) / 128 * 128;
  static constexpr uint32_t smem = kGuidedStages * bytes + 128;  // + barriers
};

template <int HB>
__device__ __forceinline__ uint32_t hint_field_smem(const uint8_t* st, int t, uint2& h4) {
  if (HB == 1) return *reinterpret_cast<const uint16_t*>(st + 2 * t);
  if (HB == 2) return *reinterpret_cast<const uint32_t*>(st + 4 * t);
  if (HB == 4) h4 = *reinterpret_cast<const uint2*>(st + 8 * t);
  return 0u;
}

template <int HB, bool STATS>
__global__ void __launch_bounds__(kStagedThreads, kGuidedCtas)
    k_guided_staged(const uint16_t* __restrict__ x, int64_t nblk, const uint8_t* __restrict__ hints,
                    uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
                    unsigned long long* __restrict__ stats4, const uint8_t* __restrict__ rcodes,
                    const uint8_t* __restrict__ rscales, const float* __restrict__ rts,
                    unsigned long long* __restrict__ stats8, uint32_t one) {
  using L = GuidedStage<HB, STATS>;
  extern __shared__ __align__(128) uint8_t stage_smem[];
  __shared__ ScaleTables tab;
  __shared__ StatsShared sm;
  __shared__ unsigned long long red4[3 * 8];
  __shared__ int abort_flag;
  const uint32_t sbase = umma::smem_u32(stage_smem);
  const uint32_t full = sbase + kGuidedStages * L::bytes, empty = full + 8 * kGuidedStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nfull = nblk / kStageBlocks;  // whole chunks
  const int64_t tail0 = nfull * kStageBlocks;  // blocks tail0 .. nblk-1: direct loads, CTA 0
  const bool producer = warp == kComputeWarps && lane == 0;
  auto load_chunk = [&](int64_t c, int s) {  // chunks are visited from the end backwards
    const int64_t b0 = (nfull - 1 - c) * kStageBlocks;
    const uint32_t bar = full + 8 * s, st = sbase + s * L::bytes;
    umma::mbar_arrive_expect_tx(bar, L::payload);
    umma::bulk_load(st + L::x, x + b0 * 16, kStageBlocks * 32, bar);
    if (HB != 0) umma::bulk_load(st + L::hints, hints + b0 * L::kHintBytes, kStageBlocks * L::kHintBytes, bar);
    if (STATS) {
      umma::bulk_load(st + L::rc, rcodes + b0 * 8, kStageBlocks * 8, bar);
      umma::bulk_load(st + L::rs, rscales + b0, kStageBlocks, bar);
    }
  };
  // The producer sets up the ring and fills every stage before the CTA
  // builds its tables, so the first loads overlap that set-up.
  int64_t c0 = blockIdx.x;
  int it0 = 0;
  if (producer) {
    for (int s = 0; s < kGuidedStages; ++s) {
      umma::mbar_init(full + 8 * s, 1);
      umma::mbar_init(empty + 8 * s, kComputeWarps);
    }
    abort_flag = 0;
    umma::fence_mbar_init();
    for (; it0 < kGuidedStages && c0 < nfull; ++it0, c0 += gridDim.x) load_chunk(c0, it0);
  }
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);  // ends in a barrier: the mbarriers are ready too
  const float ts_r = STATS ? *rts : 0.0f;
  const bool same_ts = STATS && __float_as_uint(ts_r) == __float_as_uint(s_t);
  bool far_all = false;
  if constexpr (STATS) far_all = stats_tables_init(sm, ts_r, s_t);
  volatile int* abort = &abort_flag;
  GuidedCounts gcnt{0u, 0u, 0u};
  MismatchCounts mc{0u, 0u, 0u, 0u, 0u};
  int qn = 0;

  if (warp == kComputeWarps) {
    // ---------------- producer: one lane issues the bulk copies
    if (producer) {
      int it = it0;
      for (int64_t c = c0; c < nfull; c += gridDim.x, ++it) {
        const int s = it % kGuidedStages;
        const uint32_t ph = (uint32_t)(it / kGuidedStages) & 1u;
        if (!umma::mbar_wait(empty + 8 * s, ph ^ 1u, abort)) break;
        load_chunk(c, s);
      }
    }
    __syncwarp();
  } else {
    // ---------------- compute: one block per thread per chunk
    const int t = threadIdx.x;
    const uint32_t lt_mask = (1u << lane) - 1u;
    // the blocks after the last whole chunk: CTA 0, direct loads, every lane
    // of a warp in step (the counters' queue is warp-wide)
    if (tail0 < nblk && blockIdx.x == 0) {
      for (int64_t i0 = tail0 + 32 * warp; i0 < nblk; i0 += kThreads) {
        const int64_t i = i0 + lane;
        const bool valid = i < nblk;
        uint2 cw = make_uint2(0u, 0u), rc = make_uint2(0u, 0u);
        uint32_t sb = 0u, rs = 0u;
        if (valid) {
          const Block16 b = ld_block(x + i * 16);
          uint2 h4 = make_uint2(0u, 0u);
          uint32_t hw = 0u;
          if constexpr (HB != 0) hw = hint_field<HB>(hints, i, h4);
          const BlockScale bs = block_scale_bf16(block_amax_bits(b), s_t, tab);
          if constexpr (HB != 0) cw = guided_codes<HB>(b, hw, h4, bs.inv, gcnt, one);
          else cw = rtn_codes(b, bs.inv);
          sb = bs.sb;
          reinterpret_cast<uint2*>(codes)[i] = cw;
          scales[i] = (uint8_t)sb;
          if (STATS) {
            rc = __ldg(reinterpret_cast<const uint2*>(rcodes) + i);
            rs = __ldg(rscales + i);
          }
        }
        if constexpr (STATS)
          count_block(sm, rc.x, rc.y, cw.x, cw.y, rs, sb, valid, same_ts, far_all, ts_r, s_t, warp,
                      lane, lt_mask, qn, mc);
      }
    }
    int it = 0;
    for (int64_t c = blockIdx.x; c < nfull; c += gridDim.x, ++it) {
      const int s = it % kGuidedStages;
      const uint32_t ph = (uint32_t)(it / kGuidedStages) & 1u;
      const bool ok = umma::mbar_wait(full + 8 * s, ph, abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint8_t* st = stage_smem + s * L::bytes;
      const int64_t blk0 = (nfull - 1 - c) * kStageBlocks;
      // thread t takes blocks t, t + 256, ... of the chunk: a warp reads 1 KiB
      // of contiguous values per block slot
      Block16 b[kGuidedBpt];
      uint32_t hw[kGuidedBpt], rs[kGuidedBpt];
      uint2 h4[kGuidedBpt], rc[kGuidedBpt];
#pragma unroll
      for (int k = 0; k < kGuidedBpt; ++k) {
        const int j = k * kThreads + t;
        const uint4 lo = *reinterpret_cast<const uint4*>(st + L::x + 32 * j);
        const uint4 hi = *reinterpret_cast<const uint4*>(st + L::x + 32 * j + 16);
        b[k].w[0] = lo.x; b[k].w[1] = lo.y; b[k].w[2] = lo.z; b[k].w[3] = lo.w;
        b[k].w[4] = hi.x; b[k].w[5] = hi.y; b[k].w[6] = hi.z; b[k].w[7] = hi.w;
        h4[k] = make_uint2(0u, 0u);
        hw[k] = hint_field_smem<HB>(st + L::hints, j, h4[k]);
        rc[k] = make_uint2(0u, 0u);
        rs[k] = 0u;
        if (STATS) {
          rc[k] = *reinterpret_cast<const uint2*>(st + L::rc + 8 * j);
          rs[k] = st[L::rs + j];
        }
      }
#pragma unroll
      for (int k = 0; k < kGuidedBpt; ++k) {
        const int64_t blk = blk0 + k * kThreads + t;
        const BlockScale bs = block_scale_bf16(block_amax_bits(b[k]), s_t, tab);
        uint2 cw;
        if constexpr (HB != 0) cw = guided_codes<HB>(b[k], hw[k], h4[k], bs.inv, gcnt, one);
        else cw = rtn_codes(b[k], bs.inv);
        reinterpret_cast<uint2*>(codes)[blk] = cw;
        scales[blk] = (uint8_t)bs.sb;
        if constexpr (STATS)
          count_block(sm, rc[k].x, rc[k].y, cw.x, cw.y, rs[k], bs.sb, true, same_ts, far_all, ts_r,
                      s_t, warp, lane, lt_mask, qn, mc);
      }
      __syncwarp();
      if (lane == 0) umma::mbar_arrive(empty + 8 * s);
    }
  }
  if constexpr (STATS) {
    stats_finish(sm, warp, lane, qn, mc, stats8);
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(stats8, (unsigned long long)nblk * 16ull);
  }
  if (HB != 0 && stats4 != nullptr) {
    const unsigned long long vals[3] = {gcnt.consulted, gcnt.changed, gcnt.outside};
    block_add_u64<3, kComputeWarps>(vals, stats4, red4);
  }
  __syncthreads();
  if (*abort && threadIdx.x == 0) atomicOr(ws + 1, NVFP4_WARN_TIMEOUT);
}

// ----------------------------------------------------------------- KV-cache rows
// One FP32 scale per row of [rows, cols] (one token's vector for one head of a
// KV cache, cols = head_dim), as if every row were its own tensor.  LPR =
// cols / 16 lanes share a row (one 16-value block each), so a warp covers
// 32 / LPR rows = 1 KiB of contiguous input per step; the row amax is a
// shuffle reduction over those lanes.  The block scale takes RN(amax_b / 6)
// from the per-CTA table of BF16 mantissas; q / s_row and 1 / (sb s_row) are
// divisions (s_row changes from row to row).  The per-block work is the
// tensor kernels' own.
__device__ __forceinline__ BlockScale block_scale_row(uint32_t amax_bits, float s_row,
                                                      const ScaleTables& t) {
  const uint32_t e = amax_bits >> 23;
  float q;
  if (e >= 4u && e < 255u)
    q = __uint_as_float(t.div6[(amax_bits >> 16) & 0x7Fu] + ((e - 127u) << 23));
  else
    q = __fdiv_rn(__uint_as_float(amax_bits), kE2M1Max);
  BlockScale r;
  r.sb = e4m3_rn_satfinite(__fdiv_rn(q, s_row));
  const float sbv = e4m3_value(r.sb);
  // the correctly rounded reciprocal, which is the correctly rounded 1 / y
  r.inv = (sbv == 0.0f) ? 0.0f : __frcp_rn(__fmul_rn(sbv, s_row));
  return r;
}

// One row group in flight per warp and many warps per SM (measured on the
// 65536 x 16 x 128 cache: RTN + hints 65 us at 6 CTAs, guided 84 us at 5,
// against 74 / 96 us with two groups per warp at 3 CTAs).
#ifndef NVFP4_ROWS_CTAS_RTN
#define NVFP4_ROWS_CTAS_RTN 6
#endif
#ifndef NVFP4_ROWS_CTAS_GUIDED
#define NVFP4_ROWS_CTAS_GUIDED 5
#endif
#ifndef NVFP4_ROWS_UNROLL
#define NVFP4_ROWS_UNROLL 1
#endif
template <bool GUIDED>
constexpr int rows_ctas_per_sm() { return GUIDED ? NVFP4_ROWS_CTAS_GUIDED : NVFP4_ROWS_CTAS_RTN; }

template <int LPR, int HB, bool GUIDED>
__global__ void __launch_bounds__(kThreads, rows_ctas_per_sm<GUIDED>())
    k_rows(const uint16_t* __restrict__ x, int64_t rows, const uint8_t* __restrict__ hints_in,
           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
           float* __restrict__ row_scales, uint8_t* __restrict__ hints_out,
           unsigned long long* __restrict__ stats4, uint32_t one) {
  __shared__ ScaleTables tab;  // the RN(amax / 6) table; its inv part is not used
  __shared__ unsigned long long red[3 * 8];
  scale_tables_init(tab, 1.0f);
  constexpr int kRpw = 32 / LPR;  // rows per warp step
  constexpr int kRowsUnroll = NVFP4_ROWS_UNROLL;
  const int lane = threadIdx.x & 31, sub = lane / LPR, j = lane % LPR;
  const int64_t ngroups = (rows + kRpw - 1) / kRpw;
  const int64_t wstride = (int64_t)gridDim.x * (kThreads / 32);
  GuidedCounts cnt{0u, 0u, 0u};
  for (int64_t g0 = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); g0 < ngroups;
       g0 += kRowsUnroll * wstride) {
    Block16 b[kRowsUnroll];
    uint32_t hw[kRowsUnroll];
    uint2 h4[kRowsUnroll];
#pragma unroll
    for (int u = 0; u < kRowsUnroll; ++u) {
      const int64_t row = (g0 + u * wstride) * kRpw + sub;
      const int64_t blk = row * LPR + j;
      b[u] = Block16{};
      hw[u] = 0u;
      h4[u] = make_uint2(0u, 0u);
      if (g0 + u * wstride < ngroups && row < rows) {
        b[u] = ld_block(x + blk * 16);
        if constexpr (GUIDED) hw[u] = hint_field<HB>(hints_in, blk, h4[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kRowsUnroll; ++u) {
      const int64_t row = (g0 + u * wstride) * kRpw + sub;
      const int64_t blk = row * LPR + j;
      const uint32_t own = block_amax_bits(b[u]);
      uint32_t m = own;
#pragma unroll
      for (int o = 1; o < LPR; o <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (g0 + u * wstride >= ngroups || row >= rows) continue;
      const float s_row = tensor_scale_from_amax(__uint_as_float(m));
      if (j == 0) row_scales[row] = s_row;
      const BlockScale bs = block_scale_row(own, s_row, tab);
      if constexpr (GUIDED)
        guided_block_scaled<HB>(b[u], hw[u], h4[u], bs, blk, codes, scales, cnt, one);
      else
        rtn_block_scaled<HB>(b[u], bs, blk, codes, scales, hints_out);
    }
  }
  if constexpr (GUIDED) {
    if (stats4 != nullptr) {
      const unsigned long long vals[3] = {cnt.consulted, cnt.changed, cnt.outside};
      block_add_u64<3>(vals, stats4, red);
    }
  }
}

template <int LPR>
cudaError_t launch_rows_lpr(const uint16_t* x, int64_t rows, const uint8_t* hints_in, int hint_bits,
                            bool guided, uint8_t* codes, uint8_t* scales, float* row_scales,
                            uint8_t* hints_out, unsigned long long* stats4, cudaStream_t s) {
  const int64_t groups = (rows + 32 / LPR - 1) / (32 / LPR);
  const int g = grid_for(groups * 32, kThreads, rows_ctas_per_sm<false>());
  const int gg = grid_for(groups * 32, kThreads, rows_ctas_per_sm<true>());
  if (guided) {
    switch (hint_bits) {
      case 1: k_rows<LPR, 1, true><<<gg, kThreads, 0, s>>>(x, rows, hints_in, codes, scales, row_scales, nullptr, stats4, 1u); break;
      case 2: k_rows<LPR, 2, true><<<gg, kThreads, 0, s>>>(x, rows, hints_in, codes, scales, row_scales, nullptr, stats4, 1u); break;
      case 4: k_rows<LPR, 4, true><<<gg, kThreads, 0, s>>>(x, rows, hints_in, codes, scales, row_scales, nullptr, stats4, 1u); break;
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (hints_out ? hint_bits : 0) {
      case 0: k_rows<LPR, 0, false><<<g, kThreads, 0, s>>>(x, rows, nullptr, codes, scales, row_scales, nullptr, nullptr, 1u); break;
      case 1: k_rows<LPR, 1, false><<<g, kThreads, 0, s>>>(x, rows, nullptr, codes, scales, row_scales, hints_out, nullptr, 1u); break;
      case 2: k_rows<LPR, 2, false><<<g, kThreads, 0, s>>>(x, rows, nullptr, codes, scales, row_scales, hints_out, nullptr, 1u); break;
      case 4: k_rows<LPR, 4, false><<<g, kThreads, 0, s>>>(x, rows, nullptr, codes, scales, row_scales, hints_out, nullptr, 1u); break;
      default: return cudaErrorInvalidValue;
    }
  }
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* hints_in,
                                 int hint_bits, bool guided, uint8_t* codes, uint8_t* scales,
                                 float* row_scales, uint8_t* hints_out,
                                 unsigned long long* stats4, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  switch (cols) {
    case 16: return launch_rows_lpr<1>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    case 32: return launch_rows_lpr<2>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    case 64: return launch_rows_lpr<4>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    case 128: return launch_rows_lpr<8>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    case 256: return launch_rows_lpr<16>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    case 512: return launch_rows_lpr<32>(x, rows, hints_in, hint_bits, guided, codes, scales, row_scales, hints_out, stats4, s);
    default: return cudaErrorInvalidValue;
  }
}

// ----------------------------------------------------------------- emit hint
// Two blocks (16 bytes of codes) per load, U loads in flight per thread; a
// trailing odd block is done by thread 0.
template <int HB>
__device__ __forceinline__ void hint_store_pair(uint8_t* __restrict__ hints, int64_t pair, uint4 c) {
  if (HB == 1)
    reinterpret_cast<uint32_t*>(hints)[pair] =
        hint_field1(make_uint2(c.x, c.y)) | (hint_field1(make_uint2(c.z, c.w)) << 16);
  if (HB == 2)
    reinterpret_cast<uint2*>(hints)[pair] =
        make_uint2(hint_field2(make_uint2(c.x, c.y)), hint_field2(make_uint2(c.z, c.w)));
  if (HB == 4) reinterpret_cast<uint4*>(hints)[pair] = c;
}

template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_emit_hint(const uint8_t* __restrict__ codes, int64_t nblk, uint8_t* __restrict__ hints) {
  const int64_t npair = nblk >> 1;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  const uint4* __restrict__ c4 = reinterpret_cast<const uint4*>(codes);
  for (; i + (U - 1) * stride < npair; i += U * stride) {
    uint4 c[U];
#pragma unroll
    for (int u = 0; u < U; ++u) c[u] = __ldg(c4 + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) hint_store_pair<HB>(hints, i + u * stride, c[u]);
  }
  for (; i < npair; i += stride) hint_store_pair<HB>(hints, i, __ldg(c4 + i));
  if ((nblk & 1) && blockIdx.x == 0 && threadIdx.x == 0)
    hint_store<HB>(hints, nblk - 1, __ldg(reinterpret_cast<const uint2*>(codes) + nblk - 1));
}

__global__ void k_set_f32(float* dst, float value) { *dst = value; }

// ----------------------------------------------------------------- launchers
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 1;
  }
  return cached[dev];
}

int grid_for(int64_t work_items, int items_per_cta, int ctas_per_sm) {
  const int64_t need = (work_items + items_per_cta - 1) / items_per_cta;
  const int64_t full = (int64_t)sm_count() * ctas_per_sm;
  return (int)(need < full ? (need > 0 ? need : 1) : full);
}

cudaError_t launch_amax_bf16(const uint16_t* x, int64_t nblk, uint32_t* ws, cudaStream_t s) {
  // nblk == 0 still launches one CTA: it publishes A = 0
  k_amax_bf16<kAmaxUnroll><<<grid_for(nblk, kThreads, kCtasPerSm), kThreads, 0, s>>>(x, nblk, ws);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rtn(const uint16_t* x, int64_t nblk, const uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                uint8_t* hints, int hint_bits, cudaStream_t s) {
  const int g = grid_for(nblk, kThreads, kCtasPerSm);
  const int hb = hints ? hint_bits : 0;
  switch (hb) {
    case 0: k_quantize_rtn<0, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, ws, codes, scales, tensor_scale, hints); break;
    case 1: k_quantize_rtn<1, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, ws, codes, scales, tensor_scale, hints); break;
    case 2: k_quantize_rtn<2, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, ws, codes, scales, tensor_scale, hints); break;
    case 4: k_quantize_rtn<4, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, ws, codes, scales, tensor_scale, hints); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

#ifndef NVFP4_GUIDED_STAGED
#define NVFP4_GUIDED_STAGED 0   // guided alone: staged (1) or two blocks per thread from registers (0)
#endif
#ifndef NVFP4_GS_STAGED
#define NVFP4_GS_STAGED 1       // guided + counters: staged (1) or from registers (0)
#endif

template <int HB, bool STATS>
cudaError_t launch_staged(const uint16_t* x, int64_t nblk, const uint8_t* hints, const uint32_t* ws,
                          uint8_t* codes, uint8_t* scales, float* tensor_scale,
                          unsigned long long* stats4, const uint8_t* rcodes, const uint8_t* rscales,
                          const float* rts, unsigned long long* stats8, cudaStream_t s) {
  using L = GuidedStage<HB, STATS>;
  // the dynamic shared-memory opt-in is a property of the function on each device
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_guided_staged<HB, STATS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)L::smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int64_t chunks = nblk / kStageBlocks;
  const int64_t slots = (int64_t)sm_count() * kGuidedCtas;
  const int g = (int)(chunks < 1 ? 1 : (chunks < slots ? chunks : slots));
  k_guided_staged<HB, STATS><<<g, kStagedThreads, L::smem, s>>>(
      x, nblk, hints, const_cast<uint32_t*>(ws), codes, scales, tensor_scale, stats4, rcodes, rscales,
      rts, stats8, 1u);
  return cudaGetLastError();
}

cudaError_t launch_guided(const uint16_t* x, int64_t nblk, const uint8_t* hints, int hint_bits,
                          const uint32_t* ws, uint8_t* codes, uint8_t* scales,
                          float* tensor_scale, unsigned long long* stats4, cudaStream_t s) {
  if (hints == nullptr)
    return launch_quantize_rtn(x, nblk, ws, codes, scales, tensor_scale, nullptr, 0, s);
#if NVFP4_GUIDED_STAGED
  switch (hint_bits) {
    case 1: return launch_staged<1, false>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, nullptr, nullptr, nullptr, nullptr, s);
    case 2: return launch_staged<2, false>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, nullptr, nullptr, nullptr, nullptr, s);
    case 4: return launch_staged<4, false>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, nullptr, nullptr, nullptr, nullptr, s);
    default: return cudaErrorInvalidValue;
  }
#else
  const int g = grid_for(nblk, kThreads, kCtasPerSm);
  switch (hint_bits) {
    case 1: k_guided<1, kGuidedUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    case 2: k_guided<2, kGuidedUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    case 4: k_guided<4, kGuidedUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
#endif
}

cudaError_t launch_guided_stats(const uint16_t* x, int64_t nblk, const uint8_t* hints,
                                int hint_bits, const uint32_t* ws, uint8_t* codes, uint8_t* scales,
                                float* tensor_scale, unsigned long long* stats4,
                                const uint8_t* rcodes, const uint8_t* rscales, const float* rts,
                                unsigned long long* stats8, cudaStream_t s) {
#if NVFP4_GS_STAGED
  switch (hints ? hint_bits : 0) {
    case 0: return launch_staged<0, true>(x, nblk, nullptr, ws, codes, scales, tensor_scale, nullptr, rcodes, rscales, rts, stats8, s);
    case 1: return launch_staged<1, true>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, s);
    case 2: return launch_staged<2, true>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, s);
    case 4: return launch_staged<4, true>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, s);
    default: return cudaErrorInvalidValue;
  }
#else
  const int g = grid_for(nblk, kThreads, kGsCtasPerSm);
  switch (hints ? hint_bits : 0) {
    case 0: k_guided_stats<0, kGsUnroll><<<g, kThreads, 0, s>>>(x, nblk, nullptr, ws, codes, scales, tensor_scale, nullptr, rcodes, rscales, rts, stats8, 1u); break;
    case 1: k_guided_stats<1, kGsUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, 1u); break;
    case 2: k_guided_stats<2, kGsUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, 1u); break;
    case 4: k_guided_stats<4, kGsUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, rcodes, rscales, rts, stats8, 1u); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
#endif
}

cudaError_t launch_emit_hint(const uint8_t* codes, int64_t nblk, int hint_bits, uint8_t* hints,
                             cudaStream_t s) {
  if (nblk == 0) return cudaSuccess;
  const int g = grid_for(nblk, kThreads, kCtasPerSm);
  switch (hint_bits) {
    case 1: k_emit_hint<1, 4><<<g, kThreads, 0, s>>>(codes, nblk, hints); break;
    case 2: k_emit_hint<2, 4><<<g, kThreads, 0, s>>>(codes, nblk, hints); break;
    case 4: k_emit_hint<4, 4><<<g, kThreads, 0, s>>>(codes, nblk, hints); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_set_f32(float* dst, float value, cudaStream_t s) {
  k_set_f32<<<1, 1, 0, s>>>(dst, value);
  return cudaGetLastError();
}

}  // namespace nvfp4
