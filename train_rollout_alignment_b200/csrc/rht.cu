// rht.cu -- 32-point random Hadamard transform followed by NVFP4
// round-to-nearest quantization ("Thinking Machines Lab releases 4-bit
// training", communication paragraph: a 32-dimensional random Hadamard
// transform precedes the low-bit combine payload).
//
// y = (H32 * (sigma (.) x)) * fl32(1/sqrt(32)) per contiguous 32-group.  One
// thread owns one group (two 16-value blocks, two 256-bit loads) and runs all
// five butterfly stages in registers.  The signs are applied to the BF16 words
// before unpacking (XOR of the sign bits, from a per-CTA table of 16 masks),
// which is exact.  Pass 1 needs only max |z| of the unnormalised sums:
// max_k fl(|z_k| * c) = fl(max_k |z_k| * c) because rounding is monotone.
// Pass 2 recomputes z (same code, same bits), y = fl(z * c), and quantizes.
// HBM-bound: 2 + 2 + 0.5625 bytes per element (+4 with y).
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kRhtCtasPerSm = 4;
constexpr float kInvSqrt32 = 0.17677669529663688f;  // nearest FP32 to 1/sqrt(32)

// Per-CTA sign masks: word k flips element 2k (bit 15) and 2k+1 (bit 31).
__device__ __forceinline__ void load_sign_masks(uint32_t* masks, uint32_t seed_lo,
                                                uint32_t seed_hi) {
  if (threadIdx.x < 32) {
    const uint32_t r = philox4x32_10_x0(threadIdx.x, 0u, 0u, 0u, seed_lo, seed_hi);
    const uint32_t neg = __ballot_sync(0xFFFFFFFFu, (r & 1u) != 0u);  // bit j: sigma_j = -1
    if (threadIdx.x < 16)
      masks[threadIdx.x] = (((neg >> (2 * threadIdx.x)) & 1u) << 15) |
                           (((neg >> (2 * threadIdx.x + 1)) & 1u) << 31);
  }
  __syncthreads();
}

// Packed FP32 pairs (sm_100 f32x2 arithmetic: both lanes rounded to nearest,
// exactly as two scalar operations).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f32x2 p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// First butterfly stage on one BF16 word (elements 2k, 2k+1 = lo, hi):
// (lo + hi, lo - hi) in FP32, the BF16 operand converted exactly inside the
// mixed-precision add and subtract.
__device__ __forceinline__ f32x2 stage1(uint32_t w) {
  const float hi = __uint_as_float(w & 0xFFFF0000u);
  float s, d;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.bf16 %0, l, %3;\n\tsub.rn.f32.bf16 %1, l, %3;\n\t}"
      : "=f"(s), "=f"(d)
      : "r"(w), "f"(hi));
  return pack2(s, d);
}

// z = H32 * (sigma (.) x) for the group at x (32 BF16 values), unnormalised,
// as 16 pairs P[m] = (z[2m], z[2m+1]).  Stage h = 1 pairs the two halves of a
// BF16 word; stages h = 2, 4, 8, 16 pair element j with j + h, i.e. pair m
// with pair m + h/2, half for half, so they run on packed pairs.  The
// operations and their order are those of the scalar butterfly.
// masks: the per-CTA sign masks in shared memory (broadcast reads).
__device__ __forceinline__ void hadamard32(const uint16_t* __restrict__ x, const uint32_t* masks,
                                           f32x2* P) {
  const Block16 b0 = ld_block(x), b1 = ld_block(x + 16);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    P[k] = stage1(b0.w[k] ^ masks[k]);
    P[8 + k] = stage1(b1.w[k] ^ masks[8 + k]);
  }
#pragma unroll
  for (int h2 = 1; h2 < 16; h2 <<= 1) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      if (m & h2) continue;
      const f32x2 a = P[m], c = P[m + h2];
      P[m] = add2(a, c);
      P[m + h2] = sub2(a, c);
    }
  }
}

__global__ void __launch_bounds__(kThreads, kRhtCtasPerSm)
    k_rht_amax(const uint16_t* __restrict__ x, int64_t ngroups, uint32_t seed_lo,
               uint32_t seed_hi, uint32_t* __restrict__ ws) {
  __shared__ uint32_t masks[16];
  __shared__ uint32_t red[kThreads / 32];
  load_sign_masks(masks, seed_lo, seed_hi);
  float zmax = 0.0f;  // max |z|; a NaN propagates (max.NaN), so it is not dropped
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t g = (int64_t)blockIdx.x * kThreads + threadIdx.x; g < ngroups; g += stride) {
    f32x2 P[16];
    hadamard32(x + g * 32, masks, P);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      float a, b;
      unpack2(P[m], a, b);
      asm("max.NaN.f32 %0, %0, %1;" : "+f"(zmax) : "f"(fabsf(a)));
      asm("max.NaN.f32 %0, %0, %1;" : "+f"(zmax) : "f"(fabsf(b)));
    }
  }
  const uint32_t zb = __float_as_uint(zmax);
  uint32_t best = zb >= 0x7F800000u ? zb : __float_as_uint(__fmul_rn(zmax, kInvSqrt32));
  best = block_max_u32(best, red);
  if (threadIdx.x == 0) grid_max_publish(ws, best);
}

__device__ __forceinline__ void quantize_block_f32(const float* y, float s_t, const ScaleTables& tab,
                                                   int64_t blk, uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales) {
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(y[k]));
  const BlockScale bs = block_scale_f32(amax, s_t, tab);
  if (inv_overflowed(bs.inv)) {
    reinterpret_cast<uint2*>(codes)[blk] = overflow_codes_f32(y);
  } else {
    const f32x2 inv2 = pack2(bs.inv, bs.inv);
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) unpack2(mul2(pack2(y[2 * k], y[2 * k + 1]), inv2), v[2 * k], v[2 * k + 1]);
    reinterpret_cast<uint2*>(codes)[blk] = pack_codes16(v);
  }
  scales[blk] = (uint8_t)bs.sb;
}

__global__ void __launch_bounds__(kThreads, kRhtCtasPerSm)
    k_rht_quantize(const uint16_t* __restrict__ x, int64_t ngroups, uint32_t seed_lo,
                   uint32_t seed_hi, const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
                   float* __restrict__ y_out) {
  __shared__ uint32_t masks[16];
  __shared__ ScaleTables tab;
  load_sign_masks(masks, seed_lo, seed_hi);
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init_f32(tab, s_t);
  const f32x2 c2 = pack2(kInvSqrt32, kInvSqrt32);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  // Groups are visited from the END of the tensor backwards: the amax pass
  // just before streamed forwards, so the tail it read last is still in L2.
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < ngroups; i += stride) {
    const int64_t g = ngroups - 1 - i;
    f32x2 P[16];
    hadamard32(x + g * 32, masks, P);
    float z[32];
#pragma unroll
    for (int m = 0; m < 16; ++m) unpack2(mul2(P[m], c2), z[2 * m], z[2 * m + 1]);
    if (y_out != nullptr) {
#pragma unroll
      for (int q = 0; q < 4; ++q) st_v8f(y_out + g * 32 + 8 * q, z + 8 * q);
    }
    quantize_block_f32(z, s_t, tab, 2 * g, codes, scales);
    quantize_block_f32(z + 16, s_t, tab, 2 * g + 1, codes, scales);
  }
}

cudaError_t launch_rht_quantize(const uint16_t* x, int64_t nblk, uint64_t seed, uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                float* y_out, cudaStream_t s) {
  if (nblk == 0) return launch_set_f32(tensor_scale, 1.0f, s);
  const uint32_t lo = (uint32_t)seed, hi = (uint32_t)(seed >> 32);
  const int64_t ngroups = nblk / 2;  // cols % 32 == 0
  const int g = grid_for(ngroups, kThreads, kRhtCtasPerSm);
  k_rht_amax<<<g, kThreads, 0, s>>>(x, ngroups, lo, hi, ws);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  k_rht_quantize<<<g, kThreads, 0, s>>>(x, ngroups, lo, hi, ws, codes, scales, tensor_scale, y_out);
  return cudaGetLastError();
}

}  // namespace nvfp4
