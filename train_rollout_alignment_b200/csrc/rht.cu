// rht.cu -- 32-point random Hadamard transform followed by NVFP4
// round-to-nearest quantization ("Thinking Machines Lab releases 4-bit
// training", communication paragraph: a 32-dimensional random Hadamard
// transform precedes the low-bit combine payload).
//
// y = (H32 * (sigma (.) x)) * fl32(1/sqrt(32)) per contiguous 32-group.  A
// group is two 16-value blocks held by a lane pair (2j, 2j+1): each lane runs
// the four in-register butterfly stages over its 16 values and the fifth stage
// with one shuffle (xor 1).  Loops are warp-uniform so the shuffle always has
// all 32 lanes.  Pass 1 computes y and its amax; pass 2 recomputes y (same
// code, same bits) and quantizes it, optionally storing y.  HBM-bound:
// 2 + 2.5625 bytes per element (+4 with y).
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kRhtCtasPerSm = 4;
constexpr int kRhtUnroll = 2;
constexpr float kInvSqrt32 = 0.17677669529663688f;  // nearest FP32 to 1/sqrt(32)

__device__ __forceinline__ void load_signs(float* sig_s, uint32_t seed_lo, uint32_t seed_hi) {
  if (threadIdx.x < 32) {
    const uint32_t r = philox4x32_10_x0(threadIdx.x, 0u, 0u, 0u, seed_lo, seed_hi);
    sig_s[threadIdx.x] = (r & 1u) ? -1.0f : 1.0f;
  }
  __syncthreads();
}

// The 16 transformed values of block `b` held by this lane (second half of
// the group when lane is odd).
__device__ __forceinline__ void rht16(const Block16& b, const float* sig, int odd, float* y) {
  float x[16];
  unpack_block(b, x);
#pragma unroll
  for (int k = 0; k < 16; ++k) x[k] = __fmul_rn(x[k], sig[16 * odd + k]);
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j & h) continue;
      const float a = x[j], c = x[j + h];
      x[j] = __fadd_rn(a, c);
      x[j + h] = __fsub_rn(a, c);
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float p = __shfl_xor_sync(0xFFFFFFFFu, x[k], 1);
    x[k] = odd ? __fsub_rn(p, x[k]) : __fadd_rn(x[k], p);
    y[k] = __fmul_rn(x[k], kInvSqrt32);
  }
}

template <int U>
__global__ void __launch_bounds__(kThreads, kRhtCtasPerSm)
    k_rht_amax(const uint16_t* __restrict__ x, int64_t nblk, uint32_t seed_lo, uint32_t seed_hi,
               uint32_t* __restrict__ ws) {
  __shared__ float sig[32];
  __shared__ uint32_t red[kThreads / 32];
  load_signs(sig, seed_lo, seed_hi);
  const int lane = threadIdx.x & 31, odd = lane & 1;
  const int64_t wstride = (int64_t)gridDim.x * kThreads;
  uint32_t best = 0u;
  for (int64_t wb = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); wb < nblk; wb += U * wstride) {
    Block16 b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = wb + u * wstride + lane;
      if (blk < nblk) b[u] = ld_block(x + blk * 16);
      else b[u] = Block16{{0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}};
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (wb + u * wstride >= nblk) break;  // warp-uniform
      float y[16];
      rht16(b[u], sig, odd, y);
#pragma unroll
      for (int k = 0; k < 16; ++k) best = max(best, __float_as_uint(y[k]) & 0x7FFFFFFFu);
    }
  }
  best = block_max_u32(best, red);
  if (threadIdx.x == 0) {
    if (best) atomicMax(ws, best);
    if (best >= 0x7F800000u) atomicOr(ws + 1, 1u);
  }
}

template <int U>
__global__ void __launch_bounds__(kThreads, kRhtCtasPerSm)
    k_rht_quantize(const uint16_t* __restrict__ x, int64_t nblk, uint32_t seed_lo,
                   uint32_t seed_hi, const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
                   uint8_t* __restrict__ scales, float* __restrict__ tensor_scale,
                   float* __restrict__ y_out) {
  __shared__ float sig[32];
  load_signs(sig, seed_lo, seed_hi);
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  const int lane = threadIdx.x & 31, odd = lane & 1;
  const int64_t wstride = (int64_t)gridDim.x * kThreads;
  for (int64_t wb = (int64_t)blockIdx.x * kThreads + (threadIdx.x & ~31); wb < nblk; wb += U * wstride) {
    Block16 b[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t blk = wb + u * wstride + lane;
      if (blk < nblk) b[u] = ld_block(x + blk * 16);
      else b[u] = Block16{{0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u}};
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (wb + u * wstride >= nblk) break;  // warp-uniform
      const int64_t blk = wb + u * wstride + lane;
      float y[16];
      rht16(b[u], sig, odd, y);
      if (blk >= nblk) continue;
      float amax = 0.0f;
#pragma unroll
      for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(y[k]));
      const BlockScale bs = block_scale(amax, s_t);
      float v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(y[k], bs.inv);
      reinterpret_cast<uint2*>(codes)[blk] = pack_codes16(v);
      scales[blk] = (uint8_t)bs.sb;
      if (y_out != nullptr) {
        st_v8f(y_out + blk * 16, y);
        st_v8f(y_out + blk * 16 + 8, y + 8);
      }
    }
  }
}

cudaError_t launch_rht_quantize(const uint16_t* x, int64_t nblk, uint64_t seed, uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                float* y_out, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(ws, 0, 4 * sizeof(uint32_t), s);
  if (err != cudaSuccess) return err;
  if (nblk == 0) return launch_set_f32(tensor_scale, 1.0f, s);
  const uint32_t lo = (uint32_t)seed, hi = (uint32_t)(seed >> 32);
  const int g = grid_for(nblk, kThreads, kRhtCtasPerSm);
  k_rht_amax<kRhtUnroll><<<g, kThreads, 0, s>>>(x, nblk, lo, hi, ws);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  k_rht_quantize<kRhtUnroll><<<g, kThreads, 0, s>>>(x, nblk, lo, hi, ws, codes, scales,
                                                   tensor_scale, y_out);
  return cudaGetLastError();
}

}  // namespace nvfp4
