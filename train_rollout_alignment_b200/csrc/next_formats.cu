// next_formats.cu -- the two alternatives to the dequantize -> transpose -> SR
// step that "Thinking Machines Lab releases 4-bit training" weighs
// (forward/backward mismatch paragraph, format table):
//   * 16x16-tile NVFP4: one E4M3 scale per 256-value tile (NVIDIA's proposal on
//     that page), which a transpose maps onto itself: quantize once, transpose
//     the codes and the tile scales without re-rounding;
//   * MXFP8 for the backward with stochastic rounding: E4M3 elements with one
//     E8M0 (power-of-two) scale per 32 values along the new rows;
// and dequantization of both formats (and of 16-value NVFP4 blocks).
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

// ----------------------------------------------------------------- tile-16 quantize
// A warp owns 32 horizontally adjacent tiles of one 16-row band (lane j: tile
// column 32 s + j, i.e. block 32 s + j of each of the 16 rows).  Each lane
// loads its 16 blocks (16 x 256-bit loads; every row is read as 1 KiB
// contiguous across the warp) and keeps them in registers: the tile maximum
// comes from all 16, then the same registers are quantized -- the band is
// read from memory once.  128 registers of data per thread, so CTAs are
// small (128 threads, 3 per SM: 12 warps with 16 KiB each in flight).
// Bands are visited from the end of the tensor backwards (the amax pass that
// runs just before streams forwards, so its tail is still in L2).
constexpr int kTileThreads = 128;
constexpr int kTileCtasPerSm = 3;

__global__ void __launch_bounds__(kTileThreads, kTileCtasPerSm)
    k_quantize_tile16(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                      const uint32_t* __restrict__ ws, uint8_t* __restrict__ codes,
                      uint8_t* __restrict__ tscales, float* __restrict__ tensor_scale) {
  __shared__ ScaleTables tab;
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = s_t;
  scale_tables_init(tab, s_t);
  const int lane = threadIdx.x & 31;
  const int64_t tc = cols / 16, segs = (tc + 31) / 32, nitems = (rows / 16) * segs;
  const int64_t wstride = (int64_t)gridDim.x * (kTileThreads / 32);
  for (int64_t w = (int64_t)blockIdx.x * (kTileThreads / 32) + (threadIdx.x >> 5); w < nitems;
       w += wstride) {
    const int64_t item = nitems - 1 - w;
    const int64_t ti = item / segs, tj = (item % segs) * 32 + lane;
    if (tj >= tc) continue;  // only in the last segment of a band
    const uint16_t* band = x + 16 * ti * cols + 16 * tj;
    Block16 b[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) b[r] = ld_block(band + r * cols);
    uint32_t m = 0u;
#pragma unroll
    for (int r = 0; r < 16; ++r) m = max(m, block_amax_bits(b[r]));
    const BlockScale bs = block_scale_bf16(m, s_t, tab);
    uint2* out = reinterpret_cast<uint2*>(codes + 16 * ti * (cols / 2)) + tj;
    if (inv_overflowed(bs.inv)) {
#pragma unroll
      for (int r = 0; r < 16; ++r) out[r * (cols / 16)] = overflow_codes_bf16(b[r]);
    } else {
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float xf[16], v[16];
        unpack_block(b[r], xf);
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = __fmul_rn(xf[k], bs.inv);
        out[r * (cols / 16)] = pack_codes16(v);
      }
    }
    tscales[ti * tc + tj] = (uint8_t)bs.sb;
  }
}

// ----------------------------------------------------------------- tile-16 transpose
// One CTA per 128 x 128 element square of one matrix.  The square's codes
// (128 rows of 64 bytes) are staged in shared memory as 32-bit words of 8
// nibbles; each thread then owns an 8 x 8 nibble block (8 rows x one word
// column), transposes it in registers with three rounds of masked swaps
// (4x4, 2x2 and single-nibble blocks) and writes 8 words, one per output
// row.  The row stride of 17 words and the lane -> block mapping (8 word
// columns x 4 row groups per warp) make the column reads conflict-free.  The
// square's 8 x 8 tile scales move to their transposed places.  Nothing is
// re-rounded.
constexpr int kSq = 128;
constexpr int kSqWords = kSq / 8;      // 32-bit words of codes per row of a square
constexpr int kSqStride = kSqWords + 1;

__device__ __forceinline__ void nib_swap(uint32_t& a, uint32_t& b, int shift, uint32_t mask) {
  const uint32_t t = ((a >> shift) ^ b) & mask;
  b ^= t;
  a ^= t << shift;
}

__global__ void __launch_bounds__(kThreads)
    k_transpose_tile16(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ tscales,
                       int64_t rows, int64_t cols, uint8_t* __restrict__ codes_t,
                       uint8_t* __restrict__ tscales_t) {
  __shared__ uint32_t sq[kSq][kSqStride];
  const int64_t e = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * kSq, c0 = (int64_t)blockIdx.x * kSq;
  const int64_t n = rows * cols, tr = rows / 16, tc = cols / 16;
  const int t = threadIdx.x;
  const uint8_t* src = codes + e * (n / 2);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    // 32 elements (16 bytes) per thread, as two 8-byte loads: a row of codes is
    // cols / 2 bytes, a multiple of 8 but not always of 16
    const int row = (t >> 2) + 64 * h, q = t & 3;
    const int64_t r = r0 + row, c = c0 + 32 * q;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows && c < cols) {
      if ((cols & 31) == 0) {  // 16-byte row segments: one load (codes are 16-byte aligned)
        v = __ldg(reinterpret_cast<const uint4*>(src + r * (cols / 2) + c / 2));
      } else {
        const uint2* p = reinterpret_cast<const uint2*>(src + r * (cols / 2) + c / 2);
        const uint2 lo = __ldg(p);
        v.x = lo.x;
        v.y = lo.y;
        if (c + 32 <= cols) {  // else the row ends after 16 elements
          const uint2 hi = __ldg(p + 1);
          v.z = hi.x;
          v.w = hi.y;
        }
      }
    }
    sq[row][4 * q] = v.x;
    sq[row][4 * q + 1] = v.y;
    sq[row][4 * q + 2] = v.z;
    sq[row][4 * q + 3] = v.w;
  }
  if (t < 64) {
    const int64_t ti = r0 / 16 + (t >> 3), tj = c0 / 16 + (t & 7);
    if (ti < tr && tj < tc)
      tscales_t[e * tr * tc + tj * tr + ti] = tscales[e * tr * tc + ti * tc + tj];
  }
  __syncthreads();
  const int warp = t >> 5, lane = t & 31;
  const int bc = (lane & 7) + 8 * (warp & 1);   // word column: input columns 8 bc ..
  const int br = (lane >> 3) + 4 * (warp >> 1);  // row group: input rows 8 br ..
  uint32_t m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = sq[8 * br + i][bc];
  // 4x4 and 2x2 nibble blocks move as whole half-words and bytes (one byte
  // permute per output word); single nibbles by masked swaps
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a = m[i], b = m[i + 4];
    m[i] = __byte_perm(a, b, 0x5410);      // low halves of a, b
    m[i + 4] = __byte_perm(a, b, 0x7632);  // high halves
  }
#pragma unroll
  for (int i = 0; i < 8; i += 4) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t a = m[i + k], b = m[i + k + 2];
      m[i + k] = __byte_perm(a, b, 0x6240);      // bytes a0 b0 a2 b2
      m[i + k + 2] = __byte_perm(a, b, 0x7351);  // bytes a1 b1 a3 b3
    }
  }
#pragma unroll
  for (int i = 0; i < 8; i += 2) nib_swap(m[i], m[i + 1], 4, 0x0F0F0F0Fu);
  // stage the square transposed (row 8 bc + j = output row, word br), then
  // write whole output rows with 8-byte stores (a row of codes_t is rows / 2
  // bytes: a multiple of 8)
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 8; ++j) sq[8 * bc + j][br] = m[j];
  __syncthreads();
  uint8_t* dst = codes_t + e * (n / 2);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const int idx = t + kThreads * h, orow = idx >> 3, q = idx & 7;  // 8 bytes = 16 elements
    const int64_t c = c0 + orow, r = r0 + 16 * q;
    if (c < cols && r < rows)
      *reinterpret_cast<uint2*>(dst + c * (rows / 2) + r / 2) = make_uint2(sq[orow][2 * q], sq[orow][2 * q + 1]);
  }
}

// ----------------------------------------------------------------- MXFP8 SR transpose
// E8M0 exponent of a 32-value block: floor(log2(amax)) - 8, clamped to
// [-127, 127]; -127 for an all-zero block.
__device__ __forceinline__ int e8m0_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u) return -127;
  const int biased = (int)(bits >> 23);
  const int fl = biased != 0 ? biased - 127 : (31 - __clz((int)(bits & 0x7FFFFFu))) - 149;
  return min(max(fl - 8, -127), 127);
}

// 2^k as an FP32 value for k in [-127, 127] (2^-127 is the one subnormal).
__device__ __forceinline__ float pow2f(int k) {
  return __uint_as_float(k >= -126 ? (uint32_t)(k + 127) << 23 : 0x00400000u);
}

// Stochastic rounding of a >= 0 onto the E4M3 values: lo = a with its FP32
// significand truncated to E4M3 precision (3 fraction bits; multiples of 2^-9
// below 2^-6), w = the E4M3 step there (a power of two), d = a - lo (exact);
// round up iff (r >> 8) * w < d * 2^24 (both products exact); a >= 448 -> 448.
// Returns the E4M3 byte of the magnitude.
__device__ __forceinline__ uint32_t e4m3_sr_byte(float a, uint32_t r) {
  if (a >= 448.0f) return 0x7Eu;
  float lo, w;
  if (a >= 0x1p-6f) {
    const uint32_t bits = __float_as_uint(a);
    lo = __uint_as_float(bits & 0xFFF00000u);
    w = __uint_as_float((bits & 0x7F800000u) - (3u << 23));
  } else {
    lo = __fmul_rn(floorf(__fmul_rn(a, 512.0f)), 0x1p-9f);
    w = 0x1p-9f;
  }
  const float d = __fsub_rn(a, lo);
  const bool up = __fmul_rn(__uint2float_rn(r >> 8), w) < __fmul_rn(d, 16777216.0f);
  return e4m3_rn_satfinite(up ? __fadd_rn(lo, w) : lo);
}

constexpr int kMxRows = 128;  // input rows (= output elements) per CTA
constexpr int kMxCols = 64;   // input columns (= output rows) per CTA
constexpr int kMxStride = kMxCols + 1;

__global__ void __launch_bounds__(kThreads)
    k_mxfp8_sr_transpose(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                         const float* __restrict__ ts, int64_t rows, int64_t cols,
                         uint32_t seed_lo, uint32_t seed_hi, uint32_t draw,
                         uint8_t* __restrict__ q_t, uint8_t* __restrict__ e8_t) {
  __shared__ float ys[kMxRows][kMxStride];
  const int64_t e = blockIdx.z;
  const int64_t r0 = (int64_t)blockIdx.y * kMxRows, c0 = (int64_t)blockIdx.x * kMxCols;
  const int t = threadIdx.x;
  const float s_in = __ldg(ts + e);
  // dequantize: 512 source blocks of 16 values, two per thread
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int blk = t + kThreads * j, row = blk >> 2, chunk = blk & 3;
    const int64_t r = r0 + row, c = c0 + 16 * chunk;
    if (r < rows && c < cols) {
      const int64_t base = e * rows + r;
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(codes + base * (cols / 2) + c / 2));
      const float sbv = e4m3_value(__ldg(scales + base * (cols / 16) + c / 16));
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float g0, g1;
        e2m1x2_decode(((k < 4 ? v.x : v.y) >> (8 * (k & 3))) & 0xFFu, g0, g1);
        ys[row][16 * chunk + 2 * k] = __fmul_rn(__fmul_rn(g0, sbv), s_in);
        ys[row][16 * chunk + 2 * k + 1] = __fmul_rn(__fmul_rn(g1, sbv), s_in);
      }
    }
  }
  __syncthreads();
  // warp w: 32 consecutive columns, one 32-row output block each
  const int warp = t >> 5, lane = t & 31;
  const int cl = (warp & 1) * 32 + lane, bq = warp >> 1;
  const int64_t c = c0 + cl, rb = r0 + 32 * bq;
  if (c >= cols || rb >= rows) return;
  float y[32];
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    y[k] = ys[32 * bq + k][cl];
    amax = fmaxf(amax, fabsf(y[k]));
  }
  const int ex = e8m0_exponent(amax);
  const float down = pow2f(-ex);
  const uint64_t obase = ((uint64_t)e * (uint64_t)cols + (uint64_t)c) * (uint64_t)rows + (uint64_t)rb;
  const uint32_t ctr_hi = (uint32_t)(obase >> 32);  // obase % 32 == 0: the 32 counters share it
  uint32_t out[8];
#pragma unroll
  for (int w4 = 0; w4 < 8; ++w4) {
    uint32_t word = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 4 * w4 + k;
      const uint32_t r = philox4x32_10_x0((uint32_t)obase + (uint32_t)i, ctr_hi, draw, 0u, seed_lo, seed_hi);
      const float v = __fmul_rn(y[i], down);
      const uint32_t byte = e4m3_sr_byte(fabsf(v), r) | ((__float_as_uint(y[i]) >> 31) << 7);
      word |= byte << (8 * k);
    }
    out[w4] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(q_t + obase);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
  e8_t[obase / 32] = (uint8_t)(ex + 127);
}

// ----------------------------------------------------------------- dequantize
// NVFP4 -> FP32: one thread per 16-value block; value = (G[m] * sb) * s_t in
// FP32 (the first product is exact), sign from the code.  tile16: the scale
// of block (row, b) is tile (row / 16, b) of a [rows/16, cols/16] grid.
__global__ void __launch_bounds__(kThreads)
    k_dequant_nvfp4(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                    const float* __restrict__ ts, int64_t nblk, int64_t bpr, int tile16,
                    float* __restrict__ out) {
  const float s_t = __ldg(ts);
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t si = tile16 ? ((i / bpr) / 16) * bpr + (i % bpr) : i;
    const float sbv = e4m3_value(__ldg(scales + si));
    const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes) + i);
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float g0, g1;
      e2m1x2_decode(((k < 4 ? c.x : c.y) >> (8 * (k & 3))) & 0xFFu, g0, g1);
      v[2 * k] = __fmul_rn(__fmul_rn(g0, sbv), s_t);
      v[2 * k + 1] = __fmul_rn(__fmul_rn(g1, sbv), s_t);
    }
    st_v8f(out + 16 * i, v);
    st_v8f(out + 16 * i + 8, v + 8);
  }
}

// E4M3 byte pair -> two FP32 values (hardware decode via f16; every E4M3 value
// is an f16 value).
__device__ __forceinline__ void e4m3x2_decode(uint32_t pair, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
      : "=r"(h2)
      : "r"(pair));
  asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"((unsigned short)(h2 & 0xFFFFu)));
  asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"((unsigned short)(h2 >> 16)));
}

// MXFP8 -> FP32: one thread per 32-value block; E4M3 value * 2^(byte - 127).
__global__ void __launch_bounds__(kThreads)
    k_dequant_mxfp8(const uint8_t* __restrict__ q, const uint8_t* __restrict__ e8, int64_t nblk,
                    float* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nblk;
       i += (int64_t)gridDim.x * kThreads) {
    const float unit = __uint_as_float(e8[i] != 0 ? (uint32_t)e8[i] << 23 : 0x00400000u);
    const uint4* src = reinterpret_cast<const uint4*>(q + 32 * i);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 w = __ldg(src + h);
      const uint32_t words[4] = {w.x, w.y, w.z, w.w};
      float v[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float a, b;
        e4m3x2_decode((words[k >> 1] >> (16 * (k & 1))) & 0xFFFFu, a, b);
        v[2 * k] = __fmul_rn(a, unit);
        v[2 * k + 1] = __fmul_rn(b, unit);
      }
      st_v8f(out + 32 * i + 16 * h, v);
      st_v8f(out + 32 * i + 16 * h + 8, v + 8);
    }
  }
}

// ----------------------------------------------------------------- launchers
cudaError_t launch_quantize_tile16(const uint16_t* x, int64_t rows, int64_t cols, const uint32_t* ws,
                                   uint8_t* codes, uint8_t* tscales, float* tensor_scale,
                                   cudaStream_t s) {
  const int64_t items = (rows / 16) * ((cols / 16 + 31) / 32);  // one warp each
  const int g = grid_for(items * 32, kTileThreads, kTileCtasPerSm);
  k_quantize_tile16<<<g, kTileThreads, 0, s>>>(x, rows, cols, ws, codes, tscales, tensor_scale);
  return cudaGetLastError();
}

cudaError_t launch_transpose_tile16(const uint8_t* codes, const uint8_t* tscales, int64_t batch,
                                    int64_t rows, int64_t cols, uint8_t* codes_t,
                                    uint8_t* tscales_t, cudaStream_t s) {
  const dim3 grid((unsigned)((cols + kSq - 1) / kSq), (unsigned)((rows + kSq - 1) / kSq),
                  (unsigned)batch);
  k_transpose_tile16<<<grid, kThreads, 0, s>>>(codes, tscales, rows, cols, codes_t, tscales_t);
  return cudaGetLastError();
}

cudaError_t launch_mxfp8_sr_transpose(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                      int64_t batch, int64_t rows, int64_t cols, uint64_t seed,
                                      uint32_t draw, uint8_t* q_t, uint8_t* e8_t, cudaStream_t s) {
  const dim3 grid((unsigned)((cols + kMxCols - 1) / kMxCols),
                  (unsigned)((rows + kMxRows - 1) / kMxRows), (unsigned)batch);
  k_mxfp8_sr_transpose<<<grid, kThreads, 0, s>>>(codes, scales, ts, rows, cols, (uint32_t)seed,
                                                 (uint32_t)(seed >> 32), draw, q_t, e8_t);
  return cudaGetLastError();
}

cudaError_t launch_dequant_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                 int64_t rows, int64_t cols, int tile16, float* out,
                                 cudaStream_t s) {
  const int64_t nblk = rows * cols / 16;
  k_dequant_nvfp4<<<grid_for(nblk, kThreads, 4), kThreads, 0, s>>>(codes, scales, ts, nblk,
                                                                   cols / 16, tile16, out);
  return cudaGetLastError();
}

cudaError_t launch_dequant_mxfp8(const uint8_t* q, const uint8_t* e8, int64_t n, float* out,
                                 cudaStream_t s) {
  const int64_t nblk = n / 32;
  k_dequant_mxfp8<<<grid_for(nblk, kThreads, 4), kThreads, 0, s>>>(q, e8, nblk, out);
  return cudaGetLastError();
}

}  // namespace nvfp4
