// sr_transpose.cu -- dequantize -> transpose -> stochastic-rounding
// re-quantize of a stack of NVFP4 matrices ("Thinking Machines Lab releases
// 4-bit training", forward/backward mismatch paragraph: the transpose changes
// which 16 values share a scale, so go back to high precision, transpose and
// re-quantize with stochastic rounding).
//
// Two kernels:
//   1. k_sr_amax: per matrix, max over blocks of G[max m] * sb (exact in FP32);
//      A' = that max times s_t (one rounding, which commutes with the max).
//   2. k_sr_transpose: one CTA per 64x64 tile of a matrix.  Each thread
//      dequantizes one source block (16 values, one scale decode) into a
//      padded FP32 tile in shared memory; then warp w takes 16 rows of 32
//      consecutive columns (conflict-free column reads), derives the new block
//      scale, draws one Philox4x32-10 word per element (counter = output
//      element index, draw) and writes 8 code bytes and one scale byte.
//      The lower grid point comes from the truncating E2M1 conversion; the
//      round-up test is one exact product comparison.  Integer-ALU bound
//      (10 Philox rounds per element).
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kTile = 64;
constexpr int kYStride = kTile + 1;  // padded FP32 row of the staged tile

__device__ __forceinline__ float grid_value(uint32_t m) {
  float lo, hi;
  e2m1x2_decode(m & 7u, lo, hi);
  return lo;
}

__global__ void __launch_bounds__(kThreads)
    k_sr_amax(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
              int64_t nb_per, uint32_t* __restrict__ ws) {
  __shared__ uint32_t red[kThreads / 32];
  const int64_t e = blockIdx.y;
  const uint2* __restrict__ c2 = reinterpret_cast<const uint2*>(codes) + e * nb_per;
  const uint8_t* __restrict__ se = scales + e * nb_per;
  uint32_t best = 0u;
  for (int64_t j = (int64_t)blockIdx.x * kThreads + threadIdx.x; j < nb_per;
       j += (int64_t)gridDim.x * kThreads) {
    const uint2 c = __ldg(c2 + j);
    const uint32_t m4 = __vmaxu4(__vmaxu4(c.x & 0x07070707u, (c.x >> 4) & 0x07070707u),
                                 __vmaxu4(c.y & 0x07070707u, (c.y >> 4) & 0x07070707u));
    const uint32_t m2 = __vmaxu4(m4, m4 >> 16);
    const uint32_t mm = max(m2 & 0xFFu, (m2 >> 8) & 0xFFu);
    const float P = __fmul_rn(grid_value(mm), e4m3_value(__ldg(se + j)));  // exact
    best = max(best, __float_as_uint(P));
  }
  best = block_max_u32(best, red);
  if (threadIdx.x == 0 && best) atomicMax(ws + e, best);
}

// Stochastic rounding of 8 values: a = |v| clamped to 6.  Z: their codes
// truncated toward zero (the lower grid point lo; 7 for a = 6).  With
// glo = G[lo], w = G[lo + 1] - G[lo] and d = a - glo (all exact), round up
// iff (r >> 8) < (d / w) * 2^24, evaluated as (r >> 8) * w < d * 2^24 (both
// products exact).  On the grid d = 0 and nothing moves; at 6, w is taken as
// |G[8 as a code] - 6| = 6 > 0 so nothing moves either.  Returns the 8 codes
// (magnitudes) with the round-up applied.
__device__ __forceinline__ uint32_t sr_word(const float* a, const uint32_t* r, uint32_t Z) {
  const uint32_t Zh = Z + 0x11111111u;  // codes of the upper grid points
  uint32_t up = 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float glo[2], ghi[2];
    e2m1x2_decode((Z >> (8 * j)) & 0xFFu, glo[0], glo[1]);
    e2m1x2_decode((Zh >> (8 * j)) & 0xFFu, ghi[0], ghi[1]);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int k = 2 * j + t;
      const float w = fabsf(__fsub_rn(ghi[t], glo[t]));
      const float d = __fsub_rn(a[k], glo[t]);
      const bool rnd = __fmul_rn(__uint2float_rn(r[k] >> 8), w) < __fmul_rn(d, 16777216.0f);
      up |= (rnd ? 1u : 0u) << (4 * k);
    }
  }
  return Z + up;
}

__global__ void __launch_bounds__(kThreads)
    k_sr_transpose(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                   const float* __restrict__ ts, int64_t rows, int64_t cols, uint32_t seed_lo,
                   uint32_t seed_hi, uint32_t draw, const uint32_t* __restrict__ ws,
                   uint8_t* __restrict__ codes_t, uint8_t* __restrict__ scales_t,
                   float* __restrict__ ts_t) {
  __shared__ float ys[kTile][kYStride];
  __shared__ ScaleTables tab;
  const int64_t e = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * kTile, c0 = (int64_t)blockIdx.x * kTile;
  const int t = threadIdx.x;
  const float s_in = __ldg(ts + e);
  const float A = __fmul_rn(__uint_as_float(ws[e]), s_in);
  const float s_t = tensor_scale_from_amax(A);
  scale_tables_init_f32(tab, s_t);
  {
    // dequantize: thread t takes 16 values (one source block) of tile row t / 4
    const int row = t >> 2, chunk = t & 3;
    const int64_t r = r0 + row, c = c0 + chunk * 16;
    float y[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) y[k] = 0.0f;
    if (r < rows && c < cols) {
      const int64_t base = e * rows + r;
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(codes + base * (cols / 2) + c / 2));
      const float sbv = e4m3_value(__ldg(scales + base * (cols / 16) + c / 16));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float g0, g1;
        e2m1x2_decode(((j < 4 ? v.x : v.y) >> (8 * (j & 3))) & 0xFFu, g0, g1);
        y[2 * j] = __fmul_rn(__fmul_rn(g0, sbv), s_in);  // (G[m] * sb) exact, then * s_t
        y[2 * j + 1] = __fmul_rn(__fmul_rn(g1, sbv), s_in);
      }
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) ys[row][chunk * 16 + k] = y[k];
  }
  __syncthreads();

  if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) ts_t[e] = s_t;

  // warp w: 16 rows (16 * (w % 4)) of 32 consecutive columns (32 * (w / 4))
  const int warp = t >> 5, lane = t & 31;
  const int rb = warp & 3, cl = (warp >> 2) * 32 + lane;
  const int64_t c = c0 + cl, rbase = r0 + rb * 16;
  if (c >= cols || rbase >= rows) return;
  float y[16];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    y[k] = ys[rb * 16 + k][cl];
    amax = fmaxf(amax, fabsf(y[k]));
  }
  const BlockScale bs = block_scale_f32(amax, s_t, tab);
  const uint64_t obase = ((uint64_t)e * (uint64_t)cols + (uint64_t)c) * (uint64_t)rows + (uint64_t)rbase;
  const uint32_t ctr_hi = (uint32_t)(obase >> 32);  // obase % 16 == 0: the 16 counters share it
  float a[16];
  uint32_t r[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    a[k] = fminf(fabsf(__fmul_rn(y[k], bs.inv)), kE2M1Max);
    r[k] = philox4x32_10_x0((uint32_t)obase + (uint32_t)k, ctr_hi, draw, 0u, seed_lo, seed_hi);
  }
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float* ah = a + 8 * h;
    const uint32_t Z = pack_rz8(ah);
    uint32_t S = 0u;  // signs of y
#pragma unroll
    for (int k = 0; k < 8; ++k) S |= (__float_as_uint(y[8 * h + k]) >> 31) << (4 * k + 3);
    out[h] = sr_word(ah, r + 8 * h, Z) | S;
  }
  if (bs.inv == 0.0f) {  // zero block scale: every code is +-0
    out[0] &= 0x88888888u;
    out[1] &= 0x88888888u;
  } else if (inv_overflowed(bs.inv)) {  // every nonzero y saturates, zeros stay
    const uint2 o = overflow_codes_f32(y);
    out[0] = o.x;
    out[1] = o.y;
  }
  *reinterpret_cast<uint2*>(codes_t + obase / 2) = make_uint2(out[0], out[1]);
  scales_t[obase / 16] = (uint8_t)bs.sb;
}

cudaError_t launch_sr_transpose(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                int64_t batch, int64_t rows, int64_t cols, uint64_t seed,
                                uint32_t draw, uint32_t* ws, uint8_t* codes_t,
                                uint8_t* scales_t, float* ts_t, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  cudaError_t err = cudaMemsetAsync(ws, 0, (size_t)batch * sizeof(uint32_t), s);
  if (err != cudaSuccess) return err;
  if (rows == 0 || cols == 0) {
    for (int64_t e = 0; e < batch; ++e) {
      err = launch_set_f32(ts_t + e, 1.0f, s);
      if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
  }
  const int64_t nb_per = rows * cols / 16;
  int64_t gx = ((int64_t)sm_count() * 8 + batch - 1) / batch;
  const int64_t need = (nb_per + kThreads - 1) / kThreads;
  if (gx > need) gx = need;
  if (gx < 1) gx = 1;
  k_sr_amax<<<dim3((unsigned)gx, (unsigned)batch), kThreads, 0, s>>>(codes, scales, nb_per, ws);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const dim3 grid((unsigned)((cols + kTile - 1) / kTile), (unsigned)((rows + kTile - 1) / kTile),
                  (unsigned)batch);
  k_sr_transpose<<<grid, kThreads, 0, s>>>(codes, scales, ts, rows, cols, (uint32_t)seed,
                                           (uint32_t)(seed >> 32), draw, ws, codes_t, scales_t,
                                           ts_t);
  return cudaGetLastError();
}

}  // namespace nvfp4
