// nvfp4_device.cuh -- device-side building blocks for the NVFP4 kernels
// (sm_100a).  Everything here is bit-exact IEEE binary32: no FMA contraction
// (built with -fmad=false), no flush-to-zero, divisions via __fdiv_rn.
//
// Format (E2M1 codes, E4M3 block scale per 16 values, FP32 tensor scale) and
// scale recipe: see include/nvfp4_trace.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr float kTensorScaleDiv = 2688.0f;   // 6 (E2M1 max) * 448 (E4M3 max)
constexpr float kE2M1Max = 6.0f;
constexpr int kThreads = 256;                 // threads per CTA for the streaming kernels

// ----------------------------------------------------------------- loads/stores
// One 16-value BF16 block is 32 contiguous bytes: a single 256-bit load.
struct alignas(32) Block16 {
  uint32_t w[8];
};

__device__ __forceinline__ Block16 ld_block(const uint16_t* p) {
  Block16 b;
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(b.w[0]), "=r"(b.w[1]), "=r"(b.w[2]), "=r"(b.w[3]),
                 "=r"(b.w[4]), "=r"(b.w[5]), "=r"(b.w[6]), "=r"(b.w[7])
               : "l"(p));
  return b;
}

__device__ __forceinline__ void st_v8f(float* p, const float* v) {
  asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v[0]),
               "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}


// BF16 -> FP32 with the mixed-precision add of sm_100 (x + -0 == x for every
// x, signed zeros included), which runs on the FP pipes instead of the
// integer/logic pipe.
__device__ __forceinline__ void unpack_block(const Block16& b, float* x) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "add.rn.f32.bf16 %0, l, 0f80000000;\n\tadd.rn.f32.bf16 %1, h, 0f80000000;\n\t}"
        : "=f"(x[2 * k]), "=f"(x[2 * k + 1])
        : "r"(b.w[k]));
}

// Max |x| of a 16-value block as FP32 bits (low 16 bits zero), from packed
// BF16 maxima of magnitudes (max.xorsign.abs: the magnitude is the larger
// |x|, exact; the sign bit is dropped at the end).  A NaN element is passed
// over; the tensor amax pass flags non-finite inputs.
__device__ __forceinline__ uint32_t block_amax_bits(const Block16& b) {
  uint32_t m[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[k]) : "r"(b.w[2 * k]), "r"(b.w[2 * k + 1]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[0]) : "r"(m[0]), "r"(m[1]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[2]) : "r"(m[2]), "r"(m[3]));
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m[0]) : "r"(m[0]), "r"(m[2]));
  uint32_t r;
  asm("{\n\t.reg .b16 l, h, q;\n\tmov.b32 {l, h}, %1;\n\t"
      "max.xorsign.abs.bf16 q, l, h;\n\tmov.b32 %0, {0, q};\n\t}"
      : "=r"(r)
      : "r"(m[0]));
  return r & 0x7FFF0000u;
}

// ----------------------------------------------------------------- conversions
// Two FP32 values -> one byte holding two E2M1 codes, `lo` in bits 0..3 and
// `hi` in bits 4..7.  Hardware round-to-nearest-even with saturation to +-6;
// the sign of the input is kept (also for results that round to zero).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Four FP32 values -> four E2M1 codes (16 bits, a0 in bits 0..3) rounded
// toward zero: the hardware stochastic-rounding conversion with all random bits
// zero truncates, i.e. the magnitude index is floor onto the grid (saturating
// at 6, sign kept).
__device__ __forceinline__ uint32_t e2m1x4_rz(float a0, float a1, float a2, float a3) {
  unsigned short r;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=h"(r)
      : "f"(a3), "f"(a2), "f"(a1), "f"(a0), "r"(0u));
  return r;
}

// Byte of two E2M1 codes -> the two decoded values (sign included) as FP32.
__device__ __forceinline__ void e2m1x2_decode(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h2)
      : "r"(byte));
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((unsigned short)(h2 & 0xFFFFu)));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((unsigned short)(h2 >> 16)));
}

// FP32 >= 0 -> E4M3 byte, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_rn_satfinite(float f) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(f));
  return r & 0xFFu;
}

// E4M3 byte (sign bit ignored) -> exact FP32: e = 0 is m * 2^-9, otherwise
// (8 + m) * 2^(e - 10), i.e. the FP32 pattern with exponent e + 120.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  b &= 0x7Fu;
  float sub = __int2float_rn((int)(b & 7u)) * 0x1p-9f;
  float nrm = __uint_as_float((b << 20) + (120u << 23));
  return (b >> 3) ? nrm : sub;
}

// ----------------------------------------------------------------- scale recipe
// Tensor decode multiplier s_t = A / 2688 (A == 0 -> 1).
__device__ __forceinline__ float tensor_scale_from_amax(float A) {
  return (A == 0.0f) ? 1.0f : __fdiv_rn(A, kTensorScaleDiv);
}

struct BlockScale {
  uint32_t sb;   // E4M3 byte
  float inv;     // 1 / (sb * s_t); 0 when sb decodes to 0 (all codes become +-0)
};

// Per-CTA tables for tensors whose block maxima are BF16 values (at most 8
// significant bits), filled once per CTA from s_t:
//   inv[b]  = 1 / (E4M3(b) * s_t)        (0 when E4M3(b) == 0), all 128 bytes;
//   div6[m] = FP32 bits of RN((1 + m/128) / 6), one per BF16 mantissa.
// RN(amax / 6) for amax = (1 + m/128) * 2^E is div6[m] with E added to its
// exponent field whenever the result stays a normal float (scaling by a power
// of two commutes with round-to-nearest there), so only sbf = q / s_t keeps a
// division.
struct ScaleTables {
  float inv[128];
  uint32_t div6[128];
};

__device__ __forceinline__ void scale_tables_init(ScaleTables& t, float s_t) {
  const int i = threadIdx.x;
  if (i < 128) {
    const float sbv = e4m3_value((uint32_t)i);
    t.inv[i] = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, s_t));
    t.div6[i] = __float_as_uint(__fdiv_rn(__uint_as_float(0x3F800000u | ((uint32_t)i << 16)), kE2M1Max));
  }
  __syncthreads();
}

// The part of the tables that FP32 block maxima need (inv only).
__device__ __forceinline__ void scale_tables_init_f32(ScaleTables& t, float s_t) {
  const int i = threadIdx.x;
  if (i < 128) {
    const float sbv = e4m3_value((uint32_t)i);
    t.inv[i] = (sbv == 0.0f) ? 0.0f : __fdiv_rn(1.0f, __fmul_rn(sbv, s_t));
  }
  __syncthreads();
}

// Block scale sb = E4M3((amax_b / 6) / s_t) -- two correctly rounded FP32
// divisions in that order -- and inv = 1 / (sb * s_t) from the tables, for a
// BF16-valued amax (bits of the FP32 value, low 16 zero).
__device__ __forceinline__ BlockScale block_scale_bf16(uint32_t amax_bits, float s_t,
                                                       const ScaleTables& t) {
  const uint32_t e = amax_bits >> 23;  // biased exponent (amax >= 0)
  float q;
  if (e >= 4u && e < 255u)
    q = __uint_as_float(t.div6[(amax_bits >> 16) & 0x7Fu] + ((e - 127u) << 23));
  else
    q = __fdiv_rn(__uint_as_float(amax_bits), kE2M1Max);
  BlockScale r;
  r.sb = e4m3_rn_satfinite(__fdiv_rn(q, s_t));
  r.inv = t.inv[r.sb & 0x7Fu];
  return r;
}

// The same block scale for any FP32 amax (two divisions; inv from the table).
__device__ __forceinline__ BlockScale block_scale_f32(float amax_b, float s_t,
                                                      const ScaleTables& t) {
  BlockScale r;
  const float q = __fdiv_rn(amax_b, kE2M1Max);
  r.sb = e4m3_rn_satfinite(__fdiv_rn(q, s_t));
  r.inv = t.inv[r.sb & 0x7Fu];
  return r;
}

// 8 FP32 values -> 8 round-to-nearest codes, v[0] in bits 0..3.  The four
// conversion bytes are joined by one vector move (no shifts or masks).
__device__ __forceinline__ uint32_t pack_rn8(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// 8 FP32 values -> 8 codes rounded toward zero (sign kept), v[0] in bits
// 0..3; see e2m1x4_rz.  NaN inputs give code 7 (magnitude 6).
__device__ __forceinline__ uint32_t pack_rz8(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\t"
      "cvt.rs.satfinite.e2m1x4.f32 l, {%4, %3, %2, %1}, %9;\n\t"
      "cvt.rs.satfinite.e2m1x4.f32 h, {%8, %7, %6, %5}, %9;\n\t"
      "mov.b32 %0, {l, h};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
        "r"(0u));
  return r;
}

// A block whose inv = 1 / (sb * s_t) overflowed to +inf (a tensor or row
// scale deep in the subnormal range): every nonzero x scales to +-inf and
// saturates (code 7); a zero stays zero (0 * inf would be a NaN, and zero
// sits on the grid).  Sign from x.  Rare; not on the fast path.
__device__ __forceinline__ bool inv_overflowed(float inv) { return inv > 3.40282347e38f; }

__device__ __forceinline__ uint32_t overflow_code(uint32_t mag_nonzero, uint32_t sign) {
  return (sign << 3) | (mag_nonzero ? 7u : 0u);
}
__device__ __forceinline__ uint2 overflow_codes_bf16(const Block16& b) {
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t w = b.w[k];
    const uint32_t lo = overflow_code(w & 0x7FFFu, (w >> 15) & 1u);
    const uint32_t hi = overflow_code(w & 0x7FFF0000u, w >> 31);
    out[k >> 2] |= (lo | (hi << 4)) << (8 * (k & 3));
  }
  return make_uint2(out[0], out[1]);
}
__device__ __forceinline__ uint2 overflow_codes_f32(const float* y) {
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t u = __float_as_uint(y[k]);
    out[k >> 3] |= overflow_code(u & 0x7FFFFFFFu, u >> 31) << (4 * (k & 7));
  }
  return make_uint2(out[0], out[1]);
}

// 16 FP32 values (already multiplied by inv) -> 8 bytes of packed codes.
__device__ __forceinline__ uint2 pack_codes16(const float* v) {
  return make_uint2(pack_rn8(v), pack_rn8(v + 8));
}

// ----------------------------------------------------------------- hints
// Hint field of one block from its codes (c.x: elements 0..7, c.y: 8..15).
// 1 and 2 bits keep the low magnitude bits, and the fields of elements k and
// k + 8 are adjacent: field 2*(k%8) + k/8 of the block.
//   2 bits: nibble k of the 32-bit result = (m_{k+8} & 3) << 2 | (m_k & 3)
//   1 bit:  bits 2k, 2k+1 of the 16-bit result = m_k & 1, m_{k+8} & 1
__device__ __forceinline__ uint32_t hint_field2(uint2 c) {
  return (c.x & 0x33333333u) | ((c.y << 2) & 0xCCCCCCCCu);
}
__device__ __forceinline__ uint32_t hint_field1(uint2 c) {
  uint32_t y = (c.x & 0x11111111u) | ((c.y << 1) & 0x22222222u);  // 2 bits per nibble
  y = (y | (y >> 2)) & 0x0F0F0F0Fu;
  y = (y | (y >> 4)) & 0x00FF00FFu;
  return (y | (y >> 8)) & 0x0000FFFFu;
}
// Inverse spreading for 1-bit hints: the 16-bit field -> bits 0 (element k)
// and 1 (element k + 8) of nibble k.
__device__ __forceinline__ uint32_t hint_spread1(uint32_t h16) {
  uint32_t y = h16 & 0xFFFFu;
  y = (y | (y << 8)) & 0x00FF00FFu;
  y = (y | (y << 4)) & 0x0F0F0F0Fu;
  return (y | (y << 2)) & 0x33333333u;
}

// ----------------------------------------------------------------- nibble masks
// Masks below use bit 0 of each nibble as the per-element flag.
__device__ __forceinline__ uint32_t nib_nonzero(uint32_t t) {  // nibble != 0
  t |= t >> 1;
  t |= t >> 2;
  return t & 0x11111111u;
}
// Number of flags set (multiply-add instead of popc, which is a slow pipe).
__device__ __forceinline__ uint32_t count_nib(uint32_t m) { return (m * 0x11111111u) >> 28; }

// ----------------------------------------------------------------- reductions
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  return __reduce_max_sync(0xFFFFFFFFu, v);
}

// Block-wide max of a u32, result valid in every thread (blockDim.x == kThreads).
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* smem32) {
  v = warp_max_u32(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) smem32[warp] = v;
  __syncthreads();
  v = (lane < (kThreads / 32)) ? smem32[lane] : 0u;
  v = warp_max_u32(v);
  __syncthreads();
  return v;
}

// Scratch words of the amax passes (NVFP4_WS_WORDS in all): ws[0] A, ws[1]
// warnings, ws[2..3] results of other calls, ws[4] arrival counter and ws[5]
// running maximum of the pass in flight (zero between calls), ws[6..7] unused.
constexpr int kWsArrivals = 4;
constexpr int kWsRunningMax = 5;

// Tensor-wide maximum of the CTAs' values (non-negative FP32 bit patterns,
// NaN patterns above every number), published without clearing ws first:
// each CTA folds its value into the running maximum ws[5] and then takes a
// ticket from the arrival counter ws[4]; the CTA that arrives last reads and
// zeroes the running maximum, writes ws[0] = A, ws[1] = NVFP4_WARN_NONFINITE
// iff A is an Inf/NaN pattern (the largest patterns, so the maximum shows
// whether any was seen), ws[2] = ws[3] = 0, and zeroes the counter.  No CTA
// waits for another.  Needs ws[4] == ws[5] == 0 on entry, which every call
// leaves behind.  Called once per CTA by one thread.
__device__ __forceinline__ void grid_max_publish(uint32_t* ws, uint32_t m) {
  if (m) atomicMax(ws + kWsRunningMax, m);
  __threadfence();
  const uint32_t ticket = atomicAdd(ws + kWsArrivals, 1u);
  if (ticket == gridDim.x - 1) {
    __threadfence();
    const uint32_t A = atomicExch(ws + kWsRunningMax, 0u);
    ws[0] = A;
    ws[1] = (A >= 0x7F800000u) ? 1u : 0u;
    ws[2] = 0u;
    ws[3] = 0u;
    atomicExch(ws + kWsArrivals, 0u);
  }
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Adds the block-wide sums of `vals[0..N)` to the global counters `dst`.
// Warps 0 .. WARPS-1 contribute (a CTA may carry further warps, e.g. a copy
// producer, which only take part in the barrier); smem holds N x WARPS words.
template <int N, int WARPS = kThreads / 32>
__device__ __forceinline__ void block_add_u64(const unsigned long long* vals,
                                              unsigned long long* dst,
                                              unsigned long long* smem /*[N][WARPS]*/) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < N; ++k) {
    unsigned long long s = warp_sum_u64(vals[k]);
    if (lane == 0 && warp < WARPS) smem[k * WARPS + warp] = s;
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < N; ++k) {
      unsigned long long s = (lane < WARPS) ? smem[k * WARPS + lane] : 0ull;
      s = warp_sum_u64(s);
      if (lane == 0 && s != 0ull) atomicAdd(dst + k, s);
    }
  }
}

// ----------------------------------------------------------------- Philox4x32-10
// Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC'11.  Returns output word x0 only.  Each 32x32 -> 64-bit product is one
// wide multiply; with the key schedule and the shared counter words hoisted by
// the compiler, consecutive counters share the first round's second product.
__device__ __forceinline__ uint32_t philox4x32_10_x0(uint32_t c0, uint32_t c1, uint32_t c2,
                                                     uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    c1 = (uint32_t)p1;
    c3 = (uint32_t)p0;
    c0 = n0;
    c2 = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c0;
}

}  // namespace nvfp4
