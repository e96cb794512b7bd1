// sr_transpose.cu -- dequantize -> transpose -> stochastic-rounding
// re-quantize of a stack of NVFP4 matrices ("Thinking Machines Lab releases
// 4-bit training", forward/backward mismatch paragraph: the transpose changes
// which 16 values share a scale, so go back to high precision, transpose and
// re-quantize with stochastic rounding).
//
// Two kernels:
//   1. k_sr_amax: per matrix, max over blocks of G[max m] * sb (exact in FP32);
//      A' = that max times s_t (one rounding, which commutes with the max).
//   2. k_sr_transpose: one CTA per 64x64 tile of a matrix.  The tile's codes
//      (2 KiB) and scales (256 B) are staged in shared memory; thread t owns
//      output block (column c = t/4, rows 16*(t%4)..+15), dequantizes its 16
//      values, derives the new block scale, draws one Philox4x32-10 word per
//      element (counter = output element index, draw) and writes 8 code bytes
//      and one scale byte; the four threads of a column write 32 contiguous
//      bytes.  Integer-ALU bound (10 Philox rounds per element).
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kTile = 64;

__device__ __forceinline__ float grid_value(uint32_t m) {
  float lo, hi;
  e2m1x2_decode(m & 7u, lo, hi);
  return lo;
}

// Stochastic rounding of a = |v| with the 32-bit word r: on-grid values stay,
// a >= 6 gives 6, otherwise round up iff (r >> 8) < p * 2^24 with
// p = (a - G[lo]) / (G[hi] - G[lo]); both products are exact in FP32.
__device__ __forceinline__ uint32_t sr_magnitude(float a, uint32_t r) {
  if (a >= 6.0f) return 7u;
  if (a != a) return 0u;
  const uint32_t m = e2m1x2(a, 0.0f) & 7u;          // nearest grid index
  const uint32_t lo = (grid_value(m) > a) ? m - 1u : m;
  float glo, ghi;
  e2m1x2_decode(lo | ((lo + 1u) << 4), glo, ghi);
  if (glo == a) return lo;
  const float w = __fsub_rn(ghi, glo);               // 0.5, 1 or 2
  const float inv_w = (w == 0.5f) ? 2.0f : ((w == 1.0f) ? 1.0f : 0.5f);
  const float p = __fmul_rn(__fsub_rn(a, glo), inv_w);
  const float thr = __fmul_rn(p, 16777216.0f);
  return (__uint2float_rn(r >> 8) < thr) ? lo + 1u : lo;
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

__global__ void __launch_bounds__(kThreads)
    k_sr_transpose(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                   const float* __restrict__ ts, int64_t rows, int64_t cols, uint32_t seed_lo,
                   uint32_t seed_hi, uint32_t draw, const uint32_t* __restrict__ ws,
                   uint8_t* __restrict__ codes_t, uint8_t* __restrict__ scales_t,
                   float* __restrict__ ts_t) {
  __shared__ __align__(16) uint8_t cs[kTile][kTile / 2];
  __shared__ uint8_t ss[kTile][kTile / 16];
  const int64_t e = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * kTile, c0 = (int64_t)blockIdx.x * kTile;
  const int t = threadIdx.x;
  {
    const int row = t >> 2, chunk = t & 3;
    const int64_t r = r0 + row, c = c0 + chunk * 16;
    uint2 v = make_uint2(0u, 0u);
    uint8_t sv = 0;
    if (r < rows && c < cols) {
      const int64_t base = e * rows + r;
      v = __ldg(reinterpret_cast<const uint2*>(codes + base * (cols / 2) + c / 2));
      sv = __ldg(scales + base * (cols / 16) + c / 16);
    }
    *reinterpret_cast<uint2*>(&cs[row][chunk * 8]) = v;
    ss[row][chunk] = sv;
  }
  __syncthreads();

  const float s_in = __ldg(ts + e);
  const float A = __fmul_rn(__uint_as_float(ws[e]), s_in);
  const float s_t = tensor_scale_from_amax(A);
  if (blockIdx.x == 0 && blockIdx.y == 0 && t == 0) ts_t[e] = s_t;

  const int cl = t >> 2, rb = t & 3;
  const int64_t c = c0 + cl, rbase = r0 + rb * 16;
  if (c >= cols || rbase >= rows) return;
  float y[16];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int rl = rb * 16 + k;
    const uint32_t nib = (cs[rl][cl >> 1] >> (4 * (cl & 1))) & 0xFu;
    float g, unused;
    e2m1x2_decode(nib, g, unused);
    y[k] = __fmul_rn(__fmul_rn(g, e4m3_value(ss[rl][cl >> 4])), s_in);
    amax = fmaxf(amax, fabsf(y[k]));
  }
  const BlockScale bs = block_scale(amax, s_t);
  const uint64_t obase = ((uint64_t)e * (uint64_t)cols + (uint64_t)c) * (uint64_t)rows + (uint64_t)rbase;
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float v = __fmul_rn(y[k], bs.inv);
    uint32_t m = 0u;
    if (bs.inv != 0.0f) {
      const uint64_t i = obase + (uint64_t)k;
      const uint32_t r = philox4x32_10_x0((uint32_t)i, (uint32_t)(i >> 32), draw, 0u, seed_lo, seed_hi);
      m = sr_magnitude(fabsf(v), r);
    }
    const uint32_t sgn = __float_as_uint(y[k]) >> 31;
    out[k >> 3] |= ((sgn << 3) | m) << (4 * (k & 7));
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
