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

namespace nvfp4 {

constexpr int kCtasPerSm = 4;
constexpr int kUnroll = 2;
constexpr int kAmaxUnroll = 4;  // 128 bytes in flight per thread: the amax pass has no other work

// ----------------------------------------------------------------- amax
// Max of |x| over BF16 magnitudes: |x| is the 15 low bits, and for non-negative
// values the bit patterns order like the numbers, so an unsigned max on packed
// 16-bit halves is exact.  Result: FP32 bits of A in ws[0] (atomicMax), and
// NVFP4_WARN_NONFINITE in ws[1] when an Inf/NaN pattern was seen.
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
  if (threadIdx.x == 0) {
    if (m) atomicMax(ws, m);
    if (m >= 0x7F800000u) atomicOr(ws + 1, 1u);
  }
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
__device__ __forceinline__ void rtn_block(const Block16& b, float s_t, const ScaleTables& tab,
                                          int64_t blk, uint8_t* __restrict__ codes,
                                          uint8_t* __restrict__ scales,
                                          uint8_t* __restrict__ hints) {
  float x[16];
  unpack_block(b, x);
  const BlockScale bs = block_scale_bf16(block_amax_bits(b), s_t, tab);
  float v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(x[k], bs.inv);
  const uint2 c = pack_codes16(v);
  reinterpret_cast<uint2*>(codes)[blk] = c;
  scales[blk] = (uint8_t)bs.sb;
  hint_store<HB>(hints, blk, c);
}

// Blocks are visited from the END of the tensor backwards: the amax pass that
// runs just before streams forwards, so the tail it read last is still in L2.
template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_quantize_rtn(const uint16_t* __restrict__ x, int64_t nblk, const uint32_t* __restrict__ ws,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   float* __restrict__ tensor_scale, uint8_t* __restrict__ hints) {
  __shared__ ScaleTables tab;
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (; i + (U - 1) * stride < nblk; i += U * stride) {
    Block16 b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) b[u] = ld_block(x + (nblk - 1 - (i + u * stride)) * 16);
#pragma unroll
    for (int u = 0; u < U; ++u)
      rtn_block<HB>(b[u], s_t, tab, nblk - 1 - (i + u * stride), codes, scales, hints);
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

template <int HB>
__device__ __forceinline__ void guided_block(const Block16& b, uint32_t hw, uint2 h4, float s_t,
                                             const ScaleTables& tab, int64_t blk,
                                             uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales, GuidedCounts& cnt,
                                             uint32_t one) {
  float x[16];
  unpack_block(b, x);
  const BlockScale bs = block_scale_bf16(block_amax_bits(b), s_t, tab);
  const uint32_t h1 = HB == 1 ? hint_spread1(hw) : 0u;
  uint32_t out[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[8], p[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      v[t] = __fmul_rn(x[8 * half + t], bs.inv);
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
  reinterpret_cast<uint2*>(codes)[blk] = make_uint2(out[0], out[1]);
  scales[blk] = (uint8_t)bs.sb;
}

template <int HB, int U>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    k_guided(const uint16_t* __restrict__ x, int64_t nblk, const uint8_t* __restrict__ hints,
             const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
             unsigned long long* __restrict__ stats4, uint32_t one) {
  __shared__ unsigned long long red[3 * 8];
  __shared__ ScaleTables tab;
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  GuidedCounts cnt{0u, 0u, 0u};
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (; i + (U - 1) * stride < nblk; i += U * stride) {
    Block16 b[U];
    uint32_t hw[U];
    uint2 h4[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = nblk - 1 - (i + u * stride);
      b[u] = ld_block(x + blk * 16);
      hw[u] = hint_field<HB>(hints, blk, h4[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      guided_block<HB>(b[u], hw[u], h4[u], s_t, tab, nblk - 1 - (i + u * stride), codes, scales, cnt,
                       one);
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
  if (nblk == 0) return cudaSuccess;
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

cudaError_t launch_guided(const uint16_t* x, int64_t nblk, const uint8_t* hints, int hint_bits,
                          const uint32_t* ws, uint8_t* codes, uint8_t* scales,
                          float* tensor_scale, unsigned long long* stats4, cudaStream_t s) {
  if (hints == nullptr)
    return launch_quantize_rtn(x, nblk, ws, codes, scales, tensor_scale, nullptr, 0, s);
  const int g = grid_for(nblk, kThreads, kCtasPerSm);
  switch (hint_bits) {
    case 1: k_guided<1, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    case 2: k_guided<2, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    case 4: k_guided<4, kUnroll><<<g, kThreads, 0, s>>>(x, nblk, hints, ws, codes, scales, tensor_scale, stats4, 1u); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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
