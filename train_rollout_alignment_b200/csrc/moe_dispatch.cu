// moe_dispatch.cu -- the dispatch half of the rollout producer on one GPU
// ("Thinking Machines Lab releases 4-bit training": the MoE forward runs in
// NVFP4, and the tokens reach their experts in NVFP4).  The routed tokens'
// NVFP4 rows are grouped by expert, each group padded to a multiple of 128
// rows, in the layout nvfp4_moe_gemm_quantize reads (codes row-major, scales
// in the tensor-core layout), without ever leaving NVFP4.
//
// Grouping (nvfp4_moe_route): a stable counting sort of the assignments
// a = token * top_k + slot by expert id.  The assignments are cut into chunks
// of kChunk; pass 1 counts each chunk's assignments per expert (shared-memory
// histogram); pass 2 turns those counts into each chunk's first row inside
// every expert's group (one warp per expert scans the chunks) and the groups'
// padded offsets; pass 3 places the assignments of every chunk in order:
// within a warp, lanes routed to the same expert find each other with
// match.any and take ranks by lane, and the warps' counts are scanned in
// shared memory, so every run gives the same rows.  Rows no assignment takes
// (the padding) hold -1.
//
// Gather (nvfp4_moe_gather): one 16-byte unit of codes per thread (128-bit
// loads and stores), one 4-byte word of the tensor-core scale layout per
// thread; padding rows become zeros (code 0 and scale 0 decode to 0, so
// their GEMM rows are 0).  Every index read from row_src is bounds-checked:
// a value outside the assignments gives a padding row, never a stray load.
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kChunk = 2048;            // assignments per chunk
constexpr int kRouteThreads = 256;      // 8 warps; a chunk takes kChunk / 256 rounds
constexpr int kRouteWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kThreads) k_fill_i32(int32_t* __restrict__ p, int64_t n, int32_t v) {
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads)
    p[i] = v;
}

// Pass 1: counts[c * E + e] = assignments of chunk c routed to expert e.
__global__ void __launch_bounds__(kRouteThreads)
    k_route_count(const int32_t* __restrict__ ids, int64_t A, int E, int32_t* __restrict__ counts) {
  extern __shared__ int32_t hist[];  // [E]
  for (int e = threadIdx.x; e < E; e += kRouteThreads) hist[e] = 0;
  __syncthreads();
  const int64_t a0 = (int64_t)blockIdx.x * kChunk;
  for (int r = 0; r < kChunk / kRouteThreads; ++r) {
    const int64_t a = a0 + r * kRouteThreads + threadIdx.x;
    if (a < A) {
      const int32_t e = __ldg(ids + a);
      if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kRouteThreads) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// Pass 2a: per expert (one warp each), counts -> exclusive prefix over the
// chunks (in place) and the expert's total in totals[e].
__global__ void __launch_bounds__(kRouteThreads)
    k_route_scan_chunks(int32_t* __restrict__ counts, int64_t chunks, int E,
                        int32_t* __restrict__ totals) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  if (e >= E) return;
  int32_t run = 0;
  for (int64_t c0 = 0; c0 < chunks; c0 += 32) {
    const int64_t c = c0 + lane;
    const int32_t v = c < chunks ? counts[c * E + e] : 0;
    int32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += t;
    }
    if (c < chunks) counts[c * E + e] = run + incl - v;
    run += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  if (lane == 0) totals[e] = run;
}

// Pass 2b (one CTA of 1024 threads, E <= 1024): expert_rows[e] = sum over
// e' < e of totals[e'] rounded up to 128.
__global__ void __launch_bounds__(1024)
    k_route_offsets(const int32_t* __restrict__ totals, int E, int32_t* __restrict__ expert_rows) {
  __shared__ int32_t warp_sum[32];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int32_t v = t < E ? (totals[t] + 127) / 128 * 128 : 0;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_sum[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t s = warp_sum[lane], si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t x = __shfl_up_sync(0xFFFFFFFFu, si, o);
      if (lane >= o) si += x;
    }
    warp_sum[lane] = si - s;  // exclusive prefix of the warps
  }
  __syncthreads();
  if (t < E) expert_rows[t + 1] = warp_sum[w] + incl;
  if (t == 0) expert_rows[0] = 0;
}

// Pass 3: stable placement of chunk c's assignments.
__global__ void __launch_bounds__(kRouteThreads)
    k_route_place(const int32_t* __restrict__ ids, int64_t A, int E,
                  const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ expert_rows,
                  int32_t* __restrict__ row_src, int32_t* __restrict__ assign_row) {
  extern __shared__ int32_t sm[];
  int32_t* cur = sm;       // [E]: rows of this chunk already placed, per expert
  int32_t* wcnt = sm + E;  // [8][E]: this round's per-warp counts, then their prefix
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  for (int e = t; e < E; e += kRouteThreads) cur[e] = 0;
  const int64_t c = blockIdx.x, a0 = c * kChunk;
  for (int r = 0; r < kChunk / kRouteThreads; ++r) {
    for (int i = t; i < kRouteWarps * E; i += kRouteThreads) wcnt[i] = 0;
    __syncthreads();
    const int64_t a = a0 + r * kRouteThreads + t;
    const int32_t id = a < A ? __ldg(ids + a) : -1;
    const bool ok = id >= 0 && id < E;
    const int32_t key = ok ? id : -1;
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
    const int rank = __popc(peers & lt);
    if (ok && rank == 0) wcnt[w * E + id] = __popc(peers);
    __syncthreads();
    for (int e = t; e < E; e += kRouteThreads) {
      int32_t run = cur[e];
#pragma unroll
      for (int ww = 0; ww < kRouteWarps; ++ww) {
        const int32_t v = wcnt[ww * E + e];
        wcnt[ww * E + e] = run;
        run += v;
      }
      cur[e] = run;
    }
    __syncthreads();
    if (ok) {
      const int32_t row = expert_rows[id] + chunk_base[c * E + id] + wcnt[w * E + id] + rank;
      row_src[row] = (int32_t)a;
      assign_row[a] = row;
    } else if (a < A) {
      assign_row[a] = -1;
    }
    __syncthreads();
  }
}

// Gather, codes: unit u = (row r, 16-byte column j) of the grouped rows.
__global__ void __launch_bounds__(kThreads)
    k_gather_codes(const uint4* __restrict__ codes, int64_t row_units, const int32_t* __restrict__ row_src,
                   int64_t m_cap, int64_t A, int64_t top_k, uint4* __restrict__ out) {
  const int64_t units = m_cap * row_units;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * kThreads) {
    const int64_t r = u / row_units, j = u - r * row_units;
    const int32_t a = __ldg(row_src + r);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (a >= 0 && a < A) v = __ldg(codes + (a / top_k) * row_units + j);
    out[u] = v;
  }
}

// Gather, scales: word w = (row r, scale tile kt) of the tensor-core layout
// (128 x 4 tiles; scale (r, c) at (r % 32) * 16 + (r % 128 / 32) * 4 + c % 4).
__global__ void __launch_bounds__(kThreads)
    k_gather_scales(const uint32_t* __restrict__ scales, int64_t col_tiles,
                    const int32_t* __restrict__ row_src, int64_t m_cap, int64_t A, int64_t top_k,
                    uint8_t* __restrict__ out) {
  const int64_t words = m_cap * col_tiles;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < words;
       i += (int64_t)gridDim.x * kThreads) {
    const int64_t r = i / col_tiles, kt = i - r * col_tiles;
    const int32_t a = __ldg(row_src + r);
    uint32_t v = 0u;
    if (a >= 0 && a < A) v = __ldg(scales + (a / top_k) * col_tiles + kt);  // 4 scales of the token row
    const int64_t rr = r & 127;
    *reinterpret_cast<uint32_t*>(out + ((r >> 7) * col_tiles + kt) * 512 + (rr & 31) * 16 + (rr >> 5) * 4) = v;
  }
}

int64_t route_chunks(int64_t A) { return A == 0 ? 1 : (A + kChunk - 1) / kChunk; }

cudaError_t launch_moe_route(const int32_t* ids, int64_t A, int E, int32_t* ws, int32_t* expert_rows,
                             int32_t* row_src, int64_t m_cap, int32_t* assign_row, cudaStream_t s) {
  const int64_t chunks = route_chunks(A);
  int32_t* counts = ws;                    // [chunks * E]
  int32_t* totals = ws + chunks * E;       // [E]
  k_fill_i32<<<grid_for(m_cap, kThreads, 4), kThreads, 0, s>>>(row_src, m_cap, -1);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem_count = (size_t)E * sizeof(int32_t);
  k_route_count<<<(unsigned)chunks, kRouteThreads, smem_count, s>>>(ids, A, E, counts);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  k_route_scan_chunks<<<(E + kRouteWarps - 1) / kRouteWarps, kRouteThreads, 0, s>>>(counts, chunks, E, totals);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  k_route_offsets<<<1, 1024, 0, s>>>(totals, E, expert_rows);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const size_t smem_place = (size_t)(1 + kRouteWarps) * E * sizeof(int32_t);
  k_route_place<<<(unsigned)chunks, kRouteThreads, smem_place, s>>>(ids, A, E, counts, expert_rows,
                                                                     row_src, assign_row);
  return cudaGetLastError();
}

cudaError_t launch_moe_gather(const uint8_t* codes, const uint8_t* scales, int64_t k,
                              const int32_t* row_src, int64_t m_cap, int64_t A, int64_t top_k,
                              uint8_t* a_codes, uint8_t* a_scales_mma, cudaStream_t s) {
  const int64_t row_units = k / 32, col_tiles = k / 64;
  k_gather_codes<<<grid_for(m_cap * row_units, kThreads, 4), kThreads, 0, s>>>(
      reinterpret_cast<const uint4*>(codes), row_units, row_src, m_cap, A, top_k,
      reinterpret_cast<uint4*>(a_codes));
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  k_gather_scales<<<grid_for(m_cap * col_tiles, kThreads, 4), kThreads, 0, s>>>(
      reinterpret_cast<const uint32_t*>(scales), col_tiles, row_src, m_cap, A, top_k, a_scales_mma);
  return cudaGetLastError();
}

}  // namespace nvfp4
