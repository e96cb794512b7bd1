// producer.cu -- the fused rollout producer: an NVFP4 x NVFP4 GEMM on the
// 5th-generation tensor cores whose epilogue quantizes its own output to
// NVFP4 (and emits the rollout hints), so the next layer's NVFP4 GEMM reads it
// directly ("Thinking Machines Lab releases 4-bit training": the MoE forward
// GEMMs of pre-training and rollout sampling run in NVFP4, and tokens are sent
// to the experts in NVFP4).
//
//   D = s_a s_b * (A B^T)      A [m, k], B [n, k], E2M1 codes with one E4M3
//                              scale per 16 elements along k
//   out = NVFP4(D)             codes, row-layout scales, MMA-layout scales,
//                              hints; tensor scale from a given amax A_out
//
// Persistent and warp-specialized: two CTAs per SM, each walking 128 x 128
// output tiles.  In a CTA, warp 0 (one lane) streams K-blocks of 256 -- A and
// B tiles by 128-byte-swizzled TMA, their scale tiles by bulk copy -- through
// a 3-stage shared-memory ring that runs on across tile boundaries.  Warp 1
// (one lane) copies each stage's scales into TMEM (tcgen05.cp) and issues four
// 128x128x64 block-scaled MMAs into a 128-column FP32 accumulator.  Warps
// 2..9 drain it: warp w owns TMEM lanes 32 (w % 4) .. + 31 (tile rows) and
// one 64-column half of the tile, one 16-column NVFP4 block per tcgen05.ld,
// multiply by s_a s_b, quantize in registers and store, handing the
// accumulator back as soon as its last block is read.  While one CTA's epilogue runs, its producer keeps loading
// the next tile and the SM's other CTA keeps the tensor core busy.
//
// The tensor scale of the output cannot wait for the output's own amax in a
// single pass; it comes from ws[0] (an amax known beforehand -- the previous
// step's, or a calibration), and the call records the observed max |D| in
// ws[2] for the next step.  Blocks above 6 * 448 * s_t saturate.
#include <cstdint>
#include <cudaTypedefs.h>

#include "../../include/nvfp4_trace.h"
#include "launch.h"
#include "nvfp4_device.cuh"
#include "umma.cuh"

namespace nvfp4 {
namespace {

using namespace umma;

// Pipeline shape (compile-time).  Measured on B200 at 8192 x 4096 x 4096:
// 2 CTAs per SM with 3 stages and one accumulator each (108 us) beat one CTA
// with 6 stages and two accumulators (148 us) -- two independent
// producer/MMA pipelines per SM keep more loads in flight than one deeper
// ring -- and 8 epilogue warps (100 us) beat 4, because the accumulator is
// handed back twice as soon.
//   STAGES  shared-memory ring depth (K-blocks of 256 in flight per CTA)
//   ACC     accumulator buffers per CTA (2: a CTA's epilogue overlaps its own
//           next tile's MMAs; needs TMEM for 2 x 128 columns)
//   CTAS    resident CTAs per SM
//   EPI_WARPS  epilogue warps (4: one per TMEM lane quadrant, all 128
//           columns; 8: two per quadrant, 64 columns each)
#ifndef NVFP4_GEMM_STAGES
#define NVFP4_GEMM_STAGES 3
#endif
#ifndef NVFP4_GEMM_ACC
#define NVFP4_GEMM_ACC 1
#endif
#ifndef NVFP4_GEMM_CTAS
#define NVFP4_GEMM_CTAS 2
#endif
#ifndef NVFP4_GEMM_EPI_WARPS
#define NVFP4_GEMM_EPI_WARPS 8
#endif
#ifndef NVFP4_GEMM_PAIR
#define NVFP4_GEMM_PAIR 1   // 256 x 256 tiles over CTA pairs where the shape allows
#endif

constexpr int kBM = 128, kBN = 128;
constexpr int kBK = 256;                             // elements per K-block (128 bytes)
constexpr int kStages = NVFP4_GEMM_STAGES;
constexpr int kAccBufs = NVFP4_GEMM_ACC;
constexpr int kCtasPerSm = NVFP4_GEMM_CTAS;
constexpr int kEpiWarps = NVFP4_GEMM_EPI_WARPS;
constexpr int kEpiColGroups = kEpiWarps / 4;         // column slices per lane quadrant
constexpr int kEpiBlocks = kBN / 16 / kEpiColGroups; // 16-column blocks per epilogue thread
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "epilogue warps");
constexpr int kSfWarp = 2 + kEpiWarps;               // the warp that copies scale factors
constexpr int kProducerThreads = 32 * (3 + kEpiWarps);
constexpr uint32_t kTileBytes = kBM * kBK / 2;       // 16 KB for A, same for B (kBN == kBM)
constexpr uint32_t kScaleTile = 512;                 // 128 rows x 4 scales
constexpr uint32_t kScaleBytes = (kBK / 64) * kScaleTile;  // 2 KB per operand per stage
constexpr uint32_t kStageTx = 2 * kTileBytes + 2 * kScaleBytes;
// TMEM: accumulator buffer b at column 128 b; then stage s scales at
// kTmemSfBase + 32 s (SFA +0..15, SFB +16..31)
constexpr uint32_t kTmemSfBase = kAccBufs * kBN;
constexpr uint32_t kTmemNeed = kTmemSfBase + 32 * kStages;
constexpr uint32_t kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                               : kTmemNeed <= 256 ? 256 : 512;
static_assert(kTmemNeed <= 512 && kCtasPerSm * kTmemCols <= 512, "TMEM budget");

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kTileBytes;
constexpr uint32_t kOffSfa = kOffB + kStages * kTileBytes;
constexpr uint32_t kOffSfb = kOffSfa + kStages * kScaleBytes;
// barriers: full[STAGES], empty[STAGES], acc_full[ACC], acc_empty[ACC], sf_ready[STAGES]
constexpr uint32_t kOffBar = kOffSfb + kStages * kScaleBytes;
constexpr uint32_t kOffTmemSlot = kOffBar + 8 * (3 * kStages + 2 * kAccBufs);
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kOffTables = (kOffAbort + 4 + 15) / 16 * 16;
constexpr uint32_t kSmemUsed = kOffTables + sizeof(ScaleTables);
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;    // slack to align the base to 1024
static_assert(kOffB % 1024 == 0 && kOffSfa % 1024 == 0, "swizzled tiles need 1024-byte bases");
static_assert(kSmemBytes <= 227 * 1024 && kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024,
              "shared memory per SM");

// Byte offset of scale (row r, scale column c) in the 128x4-tiled MMA layout of
// a matrix with col_tiles = ceil(sf_cols / 4) scale tiles per 128 rows.
__device__ __forceinline__ size_t mma_scale_offset(int64_t r, int64_t c, int64_t col_tiles) {
  const int64_t rr = r & 127;
  return (size_t)(((r >> 7) * col_tiles + (c >> 2)) * kScaleTile) + (size_t)((rr & 31) * 16) +
         (size_t)((rr >> 5) * 4) + (size_t)(c & 3);
}

// ----------------------------------------------------------------- scale layout
// One thread per 4-byte word (row r, scale tile kt) of the padded MMA layout.
__global__ void __launch_bounds__(kThreads) k_scales_to_mma(const uint8_t* __restrict__ scales,
                                                            int64_t rows, int64_t sf_cols,
                                                            int64_t padded_rows, int64_t col_tiles,
                                                            uint8_t* __restrict__ out) {
  const int64_t words = padded_rows * col_tiles;
  for (int64_t w = (int64_t)blockIdx.x * kThreads + threadIdx.x; w < words;
       w += (int64_t)gridDim.x * kThreads) {
    const int64_t r = w / col_tiles, kt = w - r * col_tiles;
    uint32_t v = 0;
    if (r < rows) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t c = kt * 4 + j;
        if (c < sf_cols) v |= (uint32_t)scales[r * sf_cols + c] << (8 * j);
      }
    }
    *reinterpret_cast<uint32_t*>(out + mma_scale_offset(r, kt * 4, col_tiles)) = v;
  }
}

// ----------------------------------------------------------------- GEMM + quantize
struct ProducerOut {
  uint8_t* codes;       // [m, n/2]
  uint8_t* scales;      // [m, n/16]
  uint8_t* scales_mma;  // MMA layout of the same scales, or null
  float* tensor_scale;
  uint8_t* hints;       // null when HB == 0
  float* d_out;         // FP32 D [m, n], or null
};

// Group (expert) of the A rows starting at `row`: the last g with
// group_rows[g] <= row (group_rows non-decreasing, group_rows[0] = 0).  The
// result is in [0, groups - 1] whatever the array holds, so B reads stay
// inside the stacked weights.  groups == 1 reads nothing.
__device__ __forceinline__ int group_of(const int32_t* __restrict__ group_rows, int groups,
                                        int64_t row) {
  int lo = 0, hi = groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)__ldg(group_rows + mid) <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Whole-sector stores of one thread's row segment (its blocks are adjacent
// in the row): 32 bytes of codes for 4 blocks in one 256-bit store.
template <int NB>
__device__ __forceinline__ void store_row_segment(uint8_t* __restrict__ p, const uint2* c) {
  static_assert(NB == 4 || NB == 8, "blocks per thread");
#pragma unroll
  for (int q = 0; q < NB / 4; ++q)
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p + 32 * q),
                 "r"(c[4 * q].x), "r"(c[4 * q].y), "r"(c[4 * q + 1].x), "r"(c[4 * q + 1].y),
                 "r"(c[4 * q + 2].x), "r"(c[4 * q + 2].y), "r"(c[4 * q + 3].x),
                 "r"(c[4 * q + 3].y)
                 : "memory");
}
template <int HB, int NB>
__device__ __forceinline__ void store_hints_segment(uint8_t* __restrict__ hints, int64_t blk0,
                                                    const uint2* c) {
  if (HB == 4) {
    store_row_segment<NB>(hints + blk0 * 8, c);
  } else if (HB == 2) {  // 4 bytes per block: 16-byte stores
#pragma unroll
    for (int q = 0; q < NB / 4; ++q)
      reinterpret_cast<uint4*>(hints + blk0 * 4)[q] =
          make_uint4(hint_field2(c[4 * q]), hint_field2(c[4 * q + 1]), hint_field2(c[4 * q + 2]),
                     hint_field2(c[4 * q + 3]));
  } else if (HB == 1) {  // 2 bytes per block: 8-byte stores
#pragma unroll
    for (int q = 0; q < NB / 4; ++q)
      reinterpret_cast<uint2*>(hints + blk0 * 2)[q] =
          make_uint2(hint_field1(c[4 * q]) | (hint_field1(c[4 * q + 1]) << 16),
                     hint_field1(c[4 * q + 2]) | (hint_field1(c[4 * q + 3]) << 16));
  }
}

template <int HB>
__global__ void __launch_bounds__(kProducerThreads, kCtasPerSm)
    k_gemm_nvfp4_quantize(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b,
                          const uint8_t* __restrict__ a_sf, const uint8_t* __restrict__ b_sf,
                          const float* __restrict__ a_ts, const float* __restrict__ b_ts,
                          const int32_t* __restrict__ group_rows, int groups, int n,
                          int n_tiles_n, int tiles, int kblocks, uint32_t* __restrict__ ws,
                          ProducerOut out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t full = base + kOffBar, empty = full + 8 * kStages;
  const uint32_t acc_full = empty + 8 * kStages, acc_empty = acc_full + 8 * kAccBufs;
  const uint32_t sf_ready = acc_empty + 8 * kAccBufs;  // [STAGES]: a stage's scales are in TMEM
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffAbort);
  ScaleTables& tab = *reinterpret_cast<ScaleTables*>(smem + kOffTables);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
      mbar_init(sf_ready + 8 * s, 1);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(acc_full + 8 * b, 1);
      mbar_init(acc_empty + 8 * b, kEpiWarps);
    }
    *abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(base + kOffTmemSlot, kTmemCols);
    tc_fence_before();
  }
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  // MoE form: the rows past group_rows[groups] (within m) are not computed;
  // every role reads the same value, so their tile loops agree
  if (group_rows != nullptr) {
    const int64_t m_rows = (int64_t)(tiles / n_tiles_n) * kBM;
    int64_t used = (int64_t)__ldg(group_rows + groups);
    used = used < 0 ? 0 : (used > m_rows ? m_rows : used);
    tiles = (int)((used / kBM) * n_tiles_n);
  }
  scale_tables_init_f32(tab, s_t);  // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmemSlot);
  const int64_t col_tiles_k = (int64_t)kblocks * (kBK / 64);

  if (warp == 0) {
    // ---------------- producer: TMA for the tiles, bulk copies for the scales
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
        const int mt = tile / n_tiles_n, nt = tile - mt * n_tiles_n;
        // B is the groups' weights stacked [groups * n, k]: this tile's rows
        const int bt = group_of(group_rows, groups, (int64_t)mt * kBM) * n_tiles_n + nt;
        const uint8_t* sfa = a_sf + (size_t)mt * col_tiles_k * kScaleTile;
        const uint8_t* sfb = b_sf + (size_t)bt * col_tiles_k * kScaleTile;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(empty + 8 * s, ph ^ 1u, abort)) break;
          const uint32_t bar = full + 8 * s;
          mbar_arrive_expect_tx(bar, kStageTx);
          tma_load_2d(base + kOffA + s * kTileBytes, &tm_a, bar, kb * (kBK / 2), mt * kBM);
          tma_load_2d(base + kOffB + s * kTileBytes, &tm_b, bar, kb * (kBK / 2), bt * kBN);
          bulk_load(base + kOffSfa + s * kScaleBytes, sfa + (size_t)kb * kScaleBytes, kScaleBytes,
                    bar);
          bulk_load(base + kOffSfb + s * kScaleBytes, sfb + (size_t)kb * kScaleBytes, kScaleBytes,
                    bar);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvf4(kBM, kBN);
      int it = 0, tc = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x, ++tc) {
        const int buf = tc % kAccBufs;
        const uint32_t aph = (uint32_t)(tc / kAccBufs) & 1u;
        if (!mbar_wait(acc_empty + 8 * buf, aph ^ 1u, abort)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * kBN);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(sf_ready + 8 * s, ph, abort)) break;  // implies the stage has landed
          tc_fence_after();
          const uint32_t sf = tmem + kTmemSfBase + 32u * (uint32_t)s;  // SFA +0, SFB +16
          const uint64_t da = desc_kmajor_sw128(base + kOffA + s * kTileBytes);
          const uint64_t db = desc_kmajor_sw128(base + kOffB + s * kTileBytes);
#pragma unroll
          for (int j = 0; j < kBK / 64; ++j)  // K = 64 = 32 bytes per MMA: start address + 2
            mma_nvf4(d, da + 2 * j, db + 2 * j, idesc, sf + 4 * j, sf + 16 + 4 * j,
                     (kb | j) != 0);
          mma_commit(empty + 8 * s);
        }
        mma_commit(acc_full + 8 * buf);
      }
    }
    __syncwarp();
  } else if (warp == kSfWarp) {
    // ---------------- scale-factor copies into TMEM as soon as a stage has
    // landed, running ahead of the MMA warp (copies issued by the MMA warp
    // itself stall the tensor pipe between stages).  A stage's TMEM slot is
    // free then: the stage was reloaded only after the MMAs that last read
    // the slot had completed.
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(full + 8 * s, (uint32_t)(it / kStages) & 1u, abort)) break;
          tc_fence_after();
          const uint32_t sf = tmem + kTmemSfBase + 32u * (uint32_t)s;  // SFA +0, SFB +16
#pragma unroll
          for (int j = 0; j < kBK / 64; ++j) {
            cp_32x128b_warpx4(sf + 4 * j,
                              desc_scale_chunk(base + kOffSfa + s * kScaleBytes + j * kScaleTile));
            cp_32x128b_warpx4(sf + 16 + 4 * j,
                              desc_scale_chunk(base + kOffSfb + s * kScaleBytes + j * kScaleTile));
          }
          mma_commit(sf_ready + 8 * s);
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: TMEM -> D -> NVFP4
    const int q = warp & 3;  // TMEM lane quadrant this warp may read
    const int cg = (warp - 2) >> 2;  // column slice: blocks cg * kEpiBlocks ..
    const float a_scale = *a_ts;
    const int64_t sf_cols_out = n / 16;
    const int64_t col_tiles_n = n / 64;
    if (blockIdx.x == 0 && warp == 2 && lane == 0) *out.tensor_scale = s_t;
    float dmax = 0.0f;
    int tc = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
      const int mt = tile / n_tiles_n, nt = tile - mt * n_tiles_n;
      const int buf = tc % kAccBufs;
      const uint32_t aph = (uint32_t)(tc / kAccBufs) & 1u;
      const bool ok = mbar_wait(acc_full + 8 * buf, aph, abort);
      __syncwarp();  // tcgen05.ld is warp-collective
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const float alpha = __fmul_rn(a_scale, b_ts[group_of(group_rows, groups, (int64_t)mt * kBM)]);
      const int64_t row = (int64_t)mt * kBM + q * 32 + lane;
      const int b0 = cg * kEpiBlocks;  // first 16-column block of this warp
      const uint32_t t_row = tmem + (uint32_t)(buf * kBN + 16 * b0) + ((uint32_t)(q * 32) << 16);
      const int64_t blk0 = row * sf_cols_out + (int64_t)nt * (kBN / 16) + b0;
      uint64_t sc = 0;     // this thread's scale bytes, block c16 in byte c16
      uint2 cc[kEpiBlocks];  // its codes: kEpiBlocks x 8 bytes of one row, stored at once
#pragma unroll
      for (int c16 = 0; c16 < kEpiBlocks; ++c16) {
        float y[16];
        tmem_ld16(t_row + 16 * c16, y);
        if (c16 == kEpiBlocks - 1) {  // slice fully read: release it to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + 8 * buf);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          y[i] = __fmul_rn(y[i], alpha);
          amax = fmaxf(amax, fabsf(y[i]));
        }
        dmax = fmaxf(dmax, amax);
        if (out.d_out != nullptr) {
          float* dp = out.d_out + row * n + (int64_t)nt * kBN + 16 * (b0 + c16);
#pragma unroll
          for (int h = 0; h < 2; ++h) st_v8f(dp + 8 * h, y + 8 * h);
        }
        const BlockScale bs = block_scale_f32(amax, s_t, tab);
        if (inv_overflowed(bs.inv)) {
          cc[c16] = overflow_codes_f32(y);
        } else {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(y[i], bs.inv);
          cc[c16] = pack_codes16(v);
        }
        sc |= (uint64_t)bs.sb << (8 * c16);
      }
      // one row segment per thread: codes kEpiBlocks x 8 bytes (32-byte aligned:
      // n % 128 == 0), hints kEpiBlocks x (2 / 4 / 8) bytes
      store_row_segment<kEpiBlocks>(out.codes + blk0 * 8, cc);
      if (HB != 0) store_hints_segment<HB, kEpiBlocks>(out.hints, blk0, cc);
      if (kEpiBlocks == 8)
        *reinterpret_cast<uint64_t*>(out.scales + blk0) = sc;
      else
        *reinterpret_cast<uint32_t*>(out.scales + blk0) = (uint32_t)sc;
      if (out.scales_mma != nullptr) {
#pragma unroll
        for (int h = 0; h < kEpiBlocks / 4; ++h) {
          const int64_t c = (int64_t)nt * (kBN / 16) + b0 + 4 * h;
          *reinterpret_cast<uint32_t*>(out.scales_mma + mma_scale_offset(row, c, col_tiles_n)) =
              (uint32_t)(sc >> (32 * h));
        }
      }
    }
    const uint32_t wmax = warp_max_u32(__float_as_uint(dmax));
    if (lane == 0) atomicMax(ws + 2, wmax);
  }

  tc_fence_before();
  __syncthreads();
  if (*abort && threadIdx.x == 0) atomicOr(ws + 1, NVFP4_WARN_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ----------------------------------------------------------------- the CTA-pair form
// The same GEMM + quantizing epilogue on 256 x 256 output tiles shared by a
// cluster of two CTAs on two SMs (tcgen05 cta_group::2): each CTA holds
// 128 rows of A and 128 of the 256 rows of B per K-block, the pair's MMA
// (issued by the even CTA) computes the 256 x 256 tile, and each CTA's TMEM
// receives its 128 rows.  Per SM and K-block of 256 this streams 38 KB for
// 16.8 MFLOP where the 128 x 128 form streams 36 KB for 8.4: half the L2
// traffic per FLOP, the resource the single-CTA form runs out of.  Each CTA
// also needs the scales of all 256 rows of B (its TMEM reads the scale of
// every output column).  TMEM: the 256-column accumulator and the scale
// factors of every stage (48 columns each); there is no room for a second
// accumulator, so 16 epilogue warps load their 64 columns each into
// registers at once and hand the accumulator back before quantizing.  All
// loads are TMA loads (no multicast) whose completion is counted on the even
// CTA's barrier (in the tcgen05.st form below, the scale tiles on each CTA's
// own); the MMA's completion is signalled to both CTAs.
#ifndef NVFP4_PAIR_STAGES
#define NVFP4_PAIR_STAGES 5
#endif
// Scale factors into TMEM: 0 = one thread of a dedicated warp issues
// tcgen05.cp copies (the default); 1 = four warps (one per lane quadrant)
// load them from shared memory and write them with tcgen05.st.  Both give the
// same results; the stores measured slower (123 against 85 us at 8192 x 4096
// x 4096, 422 against 270 us at K = 16384), and with four more warps the
// block's register budget leaves 80 per thread (the epilogue then reads the
// accumulator in two 32-column loads).
#ifndef NVFP4_PAIR_SF_ST
#define NVFP4_PAIR_SF_ST 0
#endif
constexpr int kPairStages = NVFP4_PAIR_STAGES;
constexpr int kPairBN = 256;                                 // output columns per tile
constexpr int kPairEpiWarps = 16;
constexpr int kPairSfWarp = 2 + kPairEpiWarps;                // the first scale-factor warp
constexpr int kPairSfWarps = NVFP4_PAIR_SF_ST ? 4 : 1;
constexpr int kPairThreads = 32 * (2 + kPairEpiWarps + kPairSfWarps);
constexpr uint32_t kPairA = 128 * (kBK / 2);                  // 16 KB
constexpr uint32_t kPairB = 128 * (kBK / 2);                  // 16 KB: this CTA's half of B
constexpr uint32_t kPairSfa = (kBK / 64) * kScaleTile;        // 2 KB
constexpr uint32_t kPairSfb = 2 * (kBK / 64) * kScaleTile;    // 4 KB: both 128-row tiles of B
constexpr uint32_t kPairStageTx = kPairA + kPairB + kPairSfa + kPairSfb;
constexpr uint32_t kPOffA = 0;
constexpr uint32_t kPOffB = kPOffA + kPairStages * kPairA;
constexpr uint32_t kPOffSfa = kPOffB + kPairStages * kPairB;
constexpr uint32_t kPOffSfb = kPOffSfa + kPairStages * kPairSfa;
// barriers: full[S], empty[S], acc_full, acc_empty, sf_ready[S], sf_landed[S]
constexpr uint32_t kPOffBar = kPOffSfb + kPairStages * kPairSfb;
constexpr uint32_t kPOffSlot = kPOffBar + 8 * (4 * kPairStages + 2);
constexpr uint32_t kPOffAbort = kPOffSlot + 4;
constexpr uint32_t kPOffTables = (kPOffAbort + 4 + 15) / 16 * 16;
constexpr uint32_t kPairSmem = kPOffTables + sizeof(ScaleTables) + 1024;
constexpr uint32_t kPairTmemCols = 512;
constexpr uint32_t kPairTmemSf = 256;                          // stage s scales at 256 + 48 s
static_assert(kPairTmemSf + 48 * kPairStages <= kPairTmemCols, "TMEM budget");  // at most 5 stages
static_assert(kPairSmem <= 227 * 1024, "shared memory");
static_assert(kPOffB % 1024 == 0 && kPOffSfa % 1024 == 0, "swizzled tiles need 1024-byte bases");

template <int HB>
__global__ void __launch_bounds__(kPairThreads, 1)
    k_gemm_nvfp4_quantize_pair(const __grid_constant__ CUtensorMap tm_a,
                               const __grid_constant__ CUtensorMap tm_b,
                               const __grid_constant__ CUtensorMap tm_sa,
                               const __grid_constant__ CUtensorMap tm_sb,
                               const float* __restrict__ a_ts, const float* __restrict__ b_ts,
                               int n, int n_tiles_n, int tiles, int kblocks,
                               uint32_t* __restrict__ ws, ProducerOut out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
  const uint32_t base = smem_u32(smem);
  const uint32_t full = base + kPOffBar, empty = full + 8 * kPairStages;
  const uint32_t acc_full = empty + 8 * kPairStages, acc_empty = acc_full + 8;
  const uint32_t sf_ready = acc_empty + 8;  // [S]: the stage's scale factors are in TMEM
  // [S], per CTA: this CTA's scale tiles of the stage have landed (SF_ST form)
  const uint32_t sf_landed = sf_ready + 8 * kPairStages;
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kPOffAbort);
  ScaleTables& tab = *reinterpret_cast<ScaleTables*>(smem + kPOffTables);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * kPairEpiWarps);
    for (int st = 0; st < kPairStages; ++st) {
      mbar_init(sf_ready + 8 * st, NVFP4_PAIR_SF_ST ? 2 * kPairSfWarps : 1);
      mbar_init(sf_landed + 8 * st, 1);
    }
    *abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_sa);
    prefetch_tensormap(&tm_sb);
  }
  cluster_sync();  // both CTAs' barriers exist before either signals the other's
  if (warp == 1) {
    tmem_alloc_pair(base + kPOffSlot, kPairTmemCols);
    tc_fence_before();
  }
  const float s_t = tensor_scale_from_amax(__uint_as_float(ws[0]));
  scale_tables_init_f32(tab, s_t);  // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + kPOffSlot);
  const int64_t col_tiles_k = (int64_t)kblocks * (kBK / 64);

  if (warp == 0) {
    // ---------------- producer (both CTAs): this CTA's halves of A and B, the
    // scales of its A rows and of all 256 B rows; completion on CTA 0's barrier
    if (lane == 0) {
      int it = 0;
      for (int tile = cluster; tile < tiles && !*abort; tile += clusters) {
        const int mt = tile / n_tiles_n, nt = tile - mt * n_tiles_n;
        const int a_row = mt * 256 + (int)rank * 128, b_row = nt * kPairBN + (int)rank * 128;
        // scale rows of 256 bytes: tile (rt, kt) starts at row (rt * col_tiles_k + kt) * 2
        const int sfa_row = (int)(((int64_t)(2 * mt + (int)rank) * col_tiles_k) * 2);
        const int sfb_row0 = (int)(((int64_t)(2 * nt) * col_tiles_k) * 2);
        const int sfb_row1 = (int)(((int64_t)(2 * nt + 1) * col_tiles_k) * 2);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kPairStages;
          const uint32_t ph = (uint32_t)(it / kPairStages) & 1u;
          if (!mbar_wait(empty + 8 * s, ph ^ 1u, abort)) break;
          const uint32_t bar = mapa_shared(full + 8 * s, 0);
#if NVFP4_PAIR_SF_ST
          // A and B of both CTAs on CTA 0's barrier; this CTA's scale tiles on
          // its own barrier, for its scale-factor warps
          if (rank == 0) mbar_arrive_expect_tx(full + 8 * s, 2 * (kPairA + kPairB));
          tma_load_2d_pair(base + kPOffA + s * kPairA, &tm_a, bar, kb * (kBK / 2), a_row);
          tma_load_2d_pair(base + kPOffB + s * kPairB, &tm_b, bar, kb * (kBK / 2), b_row);
          const uint32_t lb = sf_landed + 8 * s;
          mbar_arrive_expect_tx(lb, kPairSfa + kPairSfb);
          tma_load_2d(base + kPOffSfa + s * kPairSfa, &tm_sa, lb, 0, sfa_row + kb * 8);
          tma_load_2d(base + kPOffSfb + s * kPairSfb, &tm_sb, lb, 0, sfb_row0 + kb * 8);
          tma_load_2d(base + kPOffSfb + s * kPairSfb + kPairSfb / 2, &tm_sb, lb, 0, sfb_row1 + kb * 8);
#else
          if (rank == 0) mbar_arrive_expect_tx(full + 8 * s, 2 * kPairStageTx);
          tma_load_2d_pair(base + kPOffA + s * kPairA, &tm_a, bar, kb * (kBK / 2), a_row);
          tma_load_2d_pair(base + kPOffB + s * kPairB, &tm_b, bar, kb * (kBK / 2), b_row);
          tma_load_2d_pair(base + kPOffSfa + s * kPairSfa, &tm_sa, bar, 0, sfa_row + kb * 8);
          tma_load_2d_pair(base + kPOffSfb + s * kPairSfb, &tm_sb, bar, 0, sfb_row0 + kb * 8);
          tma_load_2d_pair(base + kPOffSfb + s * kPairSfb + kPairSfb / 2, &tm_sb, bar, 0,
                           sfb_row1 + kb * 8);
#endif
        }
      }
      // drain: the MMA's completion signal for every stage has reached this
      // CTA before it can leave the cluster
      for (int i = 0; i < kPairStages; ++i, ++it) {
        const int s = it % kPairStages;
        if (!mbar_wait(empty + 8 * s, ((uint32_t)(it / kPairStages) & 1u) ^ 1u, abort)) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: CTA 0 only.  It waits for a stage's scale
    // factors to be in TMEM (copied by the scale-factor warp, which runs ahead)
    // and issues the stage's four MMAs.
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_nvf4(256, kPairBN);
      int it = 0, tc = 0;
      for (int tile = cluster; tile < tiles && !*abort; tile += clusters, ++tc) {
        if (!mbar_wait(acc_empty, ((uint32_t)tc & 1u) ^ 1u, abort)) break;
        tc_fence_after();
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kPairStages;
          const uint32_t ph = (uint32_t)(it / kPairStages) & 1u;
#if NVFP4_PAIR_SF_ST
          if (!mbar_wait(full + 8 * s, ph, abort)) break;
          if (!mbar_wait_cluster(sf_ready + 8 * s, ph, abort)) break;  // both CTAs' scale factors
#else
          if (!mbar_wait(sf_ready + 8 * s, ph, abort)) break;  // implies the stage's data is in
#endif
          tc_fence_after();
          const uint32_t sf = tmem + kPairTmemSf + 48u * (uint32_t)s;  // SFA +4j, SFB +16+8j
          const uint64_t da = desc_kmajor_sw128(base + kPOffA + s * kPairA);
          const uint64_t db = desc_kmajor_sw128(base + kPOffB + s * kPairB);
#pragma unroll
          for (int j = 0; j < kBK / 64; ++j)
            mma_nvf4_pair(tmem, da + 2 * j, db + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j,
                          (kb | j) != 0);
          mma_commit_pair(empty + 8 * s, 0x3);
        }
        mma_commit_pair(acc_full, 0x3);
      }
    }
    __syncwarp();
  } else if (warp >= kPairSfWarp) {
#if NVFP4_PAIR_SF_ST
    // ---------------- scale factors (both CTAs): the warp of lane quadrant q
    // writes the stage's scale factors into its 32 TMEM lanes as soon as this
    // CTA's scale tiles have landed: lane l takes the 16-byte row l of each
    // 512-byte scale tile (the scales of rows l, l + 32, l + 64, l + 96) into
    // 4 columns, the layout the MMA reads (every quadrant holds the same).
    // The slot is free then: the tiles were reloaded only after the MMAs that
    // read the slot last had completed.  Each warp then arrives on CTA 0's
    // sf_ready.
    const int q = warp & 3;
    const uint32_t ready0 = mapa_shared(sf_ready, 0);
    int it = 0;
    bool go = true;
    for (int tile = cluster; go && tile < tiles && !*abort; tile += clusters) {
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % kPairStages;
        const bool ok = mbar_wait(sf_landed + 8 * s, (uint32_t)(it / kPairStages) & 1u, abort);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          go = false;
          break;
        }
        const uint8_t* sa = smem + kPOffSfa + s * kPairSfa + 16 * lane;
        const uint8_t* sb = smem + kPOffSfb + s * kPairSfb + 16 * lane;
        uint32_t va[16], vb[32];
#pragma unroll
        for (int j = 0; j < kBK / 64; ++j) {
          const uint4 a = *reinterpret_cast<const uint4*>(sa + j * kScaleTile);
          const uint4 b0 = *reinterpret_cast<const uint4*>(sb + j * kScaleTile);
          const uint4 b1 = *reinterpret_cast<const uint4*>(sb + kPairSfb / 2 + j * kScaleTile);
          va[4 * j] = a.x; va[4 * j + 1] = a.y; va[4 * j + 2] = a.z; va[4 * j + 3] = a.w;
          vb[8 * j] = b0.x; vb[8 * j + 1] = b0.y; vb[8 * j + 2] = b0.z; vb[8 * j + 3] = b0.w;
          vb[8 * j + 4] = b1.x; vb[8 * j + 5] = b1.y; vb[8 * j + 6] = b1.z; vb[8 * j + 7] = b1.w;
        }
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + kPairTmemSf + 48u * (uint32_t)s;
        tmem_st16(taddr, va);        // SFA: columns 4j .. 4j + 3
        tmem_st32(taddr + 16, vb);   // SFB: columns 16 + 8j (rows 0-127), 20 + 8j (rows 128-255)
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready0 + 8 * s);
      }
    }
    __syncwarp();
#else
    // ---------------- scale-factor copies: CTA 0 only, as soon as a stage has
    // landed.  Its TMEM slot is free then: the stage was reloaded only after
    // the MMAs that read the slot last had completed.
    if (rank == 0 && lane == 0) {
      int it = 0;
      for (int tile = cluster; tile < tiles && !*abort; tile += clusters) {
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = it % kPairStages;
          if (!mbar_wait(full + 8 * s, (uint32_t)(it / kPairStages) & 1u, abort)) break;
          tc_fence_after();
          const uint32_t sf = tmem + kPairTmemSf + 48u * (uint32_t)s;
          const uint32_t sfa_s = base + kPOffSfa + s * kPairSfa;
          const uint32_t sfb_s = base + kPOffSfb + s * kPairSfb;
#pragma unroll
          for (int j = 0; j < kBK / 64; ++j) {
            cp_32x128b_warpx4_pair(sf + 4 * j, desc_scale_chunk(sfa_s + j * kScaleTile));
            cp_32x128b_warpx4_pair(sf + 16 + 8 * j, desc_scale_chunk(sfb_s + j * kScaleTile));
            cp_32x128b_warpx4_pair(sf + 20 + 8 * j,
                                   desc_scale_chunk(sfb_s + kPairSfb / 2 + j * kScaleTile));
          }
          mma_commit_pair(sf_ready + 8 * s, 0x1);
        }
      }
    }
    __syncwarp();
#endif
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of the tile
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int cg = (warp - 2) >> 2;    // 64-column group
    const float alpha = __fmul_rn(*a_ts, *b_ts);
    const int64_t sf_cols_out = n / 16;
    const int64_t col_tiles_n = n / 64;
    const uint32_t acc_empty0 = mapa_shared(acc_empty, 0);
    if (blockIdx.x == 0 && warp == 2 && lane == 0) *out.tensor_scale = s_t;
    float dmax = 0.0f;
    int tc = 0;
    for (int tile = cluster; tile < tiles; tile += clusters, ++tc) {
      const int mt = tile / n_tiles_n, nt = tile - mt * n_tiles_n;
      const bool ok = mbar_wait(acc_full, (uint32_t)tc & 1u, abort);
      __syncwarp();  // tcgen05.ld is warp-collective
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      float y[64];
#if NVFP4_PAIR_SF_ST
      // two loads of 32 columns: with four scale-factor warps the block's
      // register budget leaves too few for one 64-column load
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cg * 64), y);
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cg * 64 + 32), y + 32);
#else
      tmem_ld64(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cg * 64), y);
#endif
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);  // the accumulator may be overwritten
      const int64_t row = (int64_t)mt * 256 + rank * 128 + q * 32 + lane;
      const int64_t col0 = (int64_t)nt * kPairBN + cg * 64;
      const int64_t blk0 = row * sf_cols_out + col0 / 16;
      uint32_t sc = 0;
      uint2 cc[4];
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        float* yb = y + 16 * c16;
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          yb[i] = __fmul_rn(yb[i], alpha);
          amax = fmaxf(amax, fabsf(yb[i]));
        }
        dmax = fmaxf(dmax, amax);
        if (out.d_out != nullptr) {
          float* dp = out.d_out + row * n + col0 + 16 * c16;
#pragma unroll
          for (int h = 0; h < 2; ++h) st_v8f(dp + 8 * h, yb + 8 * h);
        }
        const BlockScale bs = block_scale_f32(amax, s_t, tab);
        if (inv_overflowed(bs.inv)) {
          cc[c16] = overflow_codes_f32(yb);
        } else {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(yb[i], bs.inv);
          cc[c16] = pack_codes16(v);
        }
        sc |= bs.sb << (8 * c16);
      }
      store_row_segment<4>(out.codes + blk0 * 8, cc);
      if (HB != 0) store_hints_segment<HB, 4>(out.hints, blk0, cc);
      *reinterpret_cast<uint32_t*>(out.scales + blk0) = sc;
      if (out.scales_mma != nullptr)
        *reinterpret_cast<uint32_t*>(out.scales_mma + mma_scale_offset(row, col0 / 16, col_tiles_n)) = sc;
    }
    const uint32_t wmax = warp_max_u32(__float_as_uint(dmax));
    if (lane == 0) atomicMax(ws + 2, wmax);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // every MMA of the pair has completed and been read
  if (*abort && threadIdx.x == 0) atomicOr(ws + 1, NVFP4_WARN_TIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPairTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows, k/2] bytes of packed codes, boxes of 128 rows x 128 bytes, 128-byte swizzle.
bool codes_tensor_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t k) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
  cuuint32_t box[2] = {kBK / 2, kBM};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core scale layout viewed as [bytes / 256, 256]: boxes of 8 rows
// of 256 bytes, i.e. the 2 KiB of one 128-row tile group for one K-block of
// 256 (every span starts on a 512-byte tile boundary), fetched as eight
// 256-byte requests.
constexpr int kSfRow = 256;
bool scales_tensor_map(CUtensorMap* map, const uint8_t* sf, int64_t rows, int64_t k) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const int64_t bytes = ((rows + 127) / 128) * (k / 64) * kScaleTile;
  cuuint64_t dims[2] = {kSfRow, (cuuint64_t)(bytes / kSfRow)};
  cuuint64_t strides[1] = {kSfRow};
  cuuint32_t box[2] = {kSfRow, (cuuint32_t)((kBK / 64) * kScaleTile / kSfRow)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(sf), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HB>
cudaError_t launch_gemm_pair_hb(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                                const CUtensorMap& tsb, const float* a_ts, const float* b_ts,
                                int64_t m, int64_t n, int64_t k, uint32_t* ws,
                                const ProducerOut& out, cudaStream_t s) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_gemm_nvfp4_quantize_pair<HB>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int64_t tiles = (m / 256) * (n / kPairBN);
  const int64_t pairs = sm_count() / 2;
  const int clusters = (int)(tiles < pairs ? tiles : pairs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = kPairSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm_nvfp4_quantize_pair<HB>, ta, tb, tsa, tsb, a_ts, b_ts, (int)n,
                            (int)(n / kPairBN), (int)tiles, (int)(k / kBK), ws, out);
}

template <int HB>
cudaError_t launch_gemm_hb(const CUtensorMap& ta, const CUtensorMap& tb, const uint8_t* a_sf,
                           const uint8_t* b_sf, const float* a_ts, const float* b_ts,
                           const int32_t* group_rows, int groups, int64_t m, int64_t n, int64_t k,
                           uint32_t* ws, const ProducerOut& out, cudaStream_t s) {
  // The shared-memory opt-in is a property of the function on each device.
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_gemm_nvfp4_quantize<HB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int64_t tiles = (m / kBM) * (n / kBN);
  const int64_t slots = (int64_t)kCtasPerSm * sm_count();
  const int grid = (int)(tiles < slots ? tiles : slots);
  k_gemm_nvfp4_quantize<HB><<<grid, kProducerThreads, kSmemBytes, s>>>(
      ta, tb, a_sf, b_sf, a_ts, b_ts, group_rows, groups, (int)n, (int)(n / kBN), (int)tiles,
      (int)(k / kBK), ws, out);
  return cudaGetLastError();
}

// The bounded wait of the GEMM pipeline on a barrier that nothing completes
// (initialised for one arrival that never comes): it must give up after
// kWaitLimitNs and report NVFP4_WARN_TIMEOUT, leaving the context usable.
__global__ void k_wait_selftest(uint32_t* ws) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(smem_u32(&bar), 0, &abort)) atomicOr(ws + 1, NVFP4_WARN_TIMEOUT);
}

__global__ void k_tensor_scale_from_ws(const uint32_t* ws, float* tensor_scale) {
  *tensor_scale = tensor_scale_from_amax(__uint_as_float(ws[0]));
}

}  // namespace

cudaError_t launch_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t sf_cols,
                                 uint8_t* out, cudaStream_t s) {
  const int64_t padded_rows = (rows + 127) / 128 * 128, col_tiles = (sf_cols + 3) / 4;
  const int64_t words = padded_rows * col_tiles;
  if (words == 0) return cudaSuccess;
  k_scales_to_mma<<<grid_for(words, kThreads, 4), kThreads, 0, s>>>(scales, rows, sf_cols,
                                                                   padded_rows, col_tiles, out);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(uint32_t* ws, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(ws + 1, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  k_wait_selftest<<<1, 32, 0, s>>>(ws);
  return cudaGetLastError();
}

cudaError_t launch_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_ts,
                                 const uint8_t* b_codes, const uint8_t* b_sf, const float* b_ts,
                                 const int32_t* group_rows, int64_t groups, int64_t m, int64_t n,
                                 int64_t k, uint32_t* ws, uint8_t* codes, uint8_t* scales,
                                 uint8_t* scales_mma, float* tensor_scale, uint8_t* hints,
                                 int hint_bits, float* d_out, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(ws + 1, 0, 3 * sizeof(uint32_t), s);
  if (e != cudaSuccess) return e;
  if (m == 0 || n == 0) {
    k_tensor_scale_from_ws<<<1, 1, 0, s>>>(ws, tensor_scale);
    return cudaGetLastError();
  }
  CUtensorMap ta, tb;
  if (!codes_tensor_map(&ta, a_codes, m, k) || !codes_tensor_map(&tb, b_codes, groups * n, k))
    return cudaErrorInvalidValue;
  const ProducerOut out{codes, scales, scales_mma, tensor_scale, hints, d_out};
  const int g = (int)groups;
#if NVFP4_GEMM_PAIR
  // the CTA-pair form: plain GEMMs whose tiles of 256 x 256 cover the output
  if (groups == 1 && m % 256 == 0 && n % kPairBN == 0 && sm_count() >= 2) {
    CUtensorMap tsa, tsb;
    if (!scales_tensor_map(&tsa, a_sf, m, k) || !scales_tensor_map(&tsb, b_sf, n, k))
      return cudaErrorInvalidValue;
    switch (hints == nullptr ? 0 : hint_bits) {
      case 1: return launch_gemm_pair_hb<1>(ta, tb, tsa, tsb, a_ts, b_ts, m, n, k, ws, out, s);
      case 2: return launch_gemm_pair_hb<2>(ta, tb, tsa, tsb, a_ts, b_ts, m, n, k, ws, out, s);
      case 4: return launch_gemm_pair_hb<4>(ta, tb, tsa, tsb, a_ts, b_ts, m, n, k, ws, out, s);
      default: return launch_gemm_pair_hb<0>(ta, tb, tsa, tsb, a_ts, b_ts, m, n, k, ws, out, s);
    }
  }
#endif
  switch (hints == nullptr ? 0 : hint_bits) {
    case 1: return launch_gemm_hb<1>(ta, tb, a_sf, b_sf, a_ts, b_ts, group_rows, g, m, n, k, ws, out, s);
    case 2: return launch_gemm_hb<2>(ta, tb, a_sf, b_sf, a_ts, b_ts, group_rows, g, m, n, k, ws, out, s);
    case 4: return launch_gemm_hb<4>(ta, tb, a_sf, b_sf, a_ts, b_ts, group_rows, g, m, n, k, ws, out, s);
    default: return launch_gemm_hb<0>(ta, tb, a_sf, b_sf, a_ts, b_ts, group_rows, g, m, n, k, ws, out, s);
  }
}

}  // namespace nvfp4
