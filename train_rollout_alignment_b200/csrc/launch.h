// launch.h -- host-side launchers shared by the C-ABI layer (api.cu) and the
// kernel translation units.  Every launcher enqueues on `s` and returns the
// launch status (cudaGetLastError after the launch).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4_trace.h"

namespace nvfp4 {

// Argument checks shared by nvfp4_sr_transpose_requant and its no-allocation
// form (everything except the scratch words); NVFP4_OK for batch == 0.
nvfp4_status check_sr_transpose_args(const uint8_t* codes, const uint8_t* scales,
                                     const float* tensor_scale, int64_t batch, int64_t rows,
                                     int64_t cols, const uint8_t* codes_t, const uint8_t* scales_t,
                                     const float* tensor_scale_t);

// Streaming grid: `ctas_per_sm` resident CTAs on every SM, capped by the work.
int grid_for(int64_t work_items, int items_per_cta, int ctas_per_sm);
int sm_count();

cudaError_t launch_amax_bf16(const uint16_t* x, int64_t nblk, uint32_t* ws, cudaStream_t s);
cudaError_t launch_quantize_rtn(const uint16_t* x, int64_t nblk, const uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                uint8_t* hints, int hint_bits, cudaStream_t s);
cudaError_t launch_guided(const uint16_t* x, int64_t nblk, const uint8_t* hints, int hint_bits,
                          const uint32_t* ws, uint8_t* codes, uint8_t* scales,
                          float* tensor_scale, unsigned long long* stats4, cudaStream_t s);
// Guided re-quantization (plain round-to-nearest without hints) that also
// adds the mismatch counters against the rollout tensor (rcodes, rscales,
// *rts) to stats8.
cudaError_t launch_guided_stats(const uint16_t* x, int64_t nblk, const uint8_t* hints,
                                int hint_bits, const uint32_t* ws, uint8_t* codes, uint8_t* scales,
                                float* tensor_scale, unsigned long long* stats4,
                                const uint8_t* rcodes, const uint8_t* rscales, const float* rts,
                                unsigned long long* stats8, cudaStream_t s);
cudaError_t launch_emit_hint(const uint8_t* codes, int64_t nblk, int hint_bits, uint8_t* hints,
                             cudaStream_t s);
cudaError_t launch_mismatch_stats(const uint8_t* ca, const uint8_t* sa, const float* ta,
                                  const uint8_t* cb, const uint8_t* sb, const float* tb,
                                  int64_t nblk, unsigned long long* stats8, cudaStream_t s);
cudaError_t launch_sr_transpose(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                int64_t batch, int64_t rows, int64_t cols, uint64_t seed,
                                uint32_t draw, uint32_t* ws, uint8_t* codes_t,
                                uint8_t* scales_t, float* ts_t, cudaStream_t s);
cudaError_t launch_rht_quantize(const uint16_t* x, int64_t nblk, uint64_t seed, uint32_t* ws,
                                uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                float* y_out, cudaStream_t s);
cudaError_t launch_quantize_tile16(const uint16_t* x, int64_t rows, int64_t cols, const uint32_t* ws,
                                   uint8_t* codes, uint8_t* tscales, float* tensor_scale,
                                   cudaStream_t s);
cudaError_t launch_transpose_tile16(const uint8_t* codes, const uint8_t* tscales, int64_t batch,
                                    int64_t rows, int64_t cols, uint8_t* codes_t,
                                    uint8_t* tscales_t, cudaStream_t s);
cudaError_t launch_mxfp8_sr_transpose(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                      int64_t batch, int64_t rows, int64_t cols, uint64_t seed,
                                      uint32_t draw, uint8_t* q_t, uint8_t* e8_t, cudaStream_t s);
cudaError_t launch_dequant_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* ts,
                                 int64_t rows, int64_t cols, int tile16, float* out,
                                 cudaStream_t s);
cudaError_t launch_dequant_mxfp8(const uint8_t* q, const uint8_t* e8, int64_t n, float* out,
                                 cudaStream_t s);
cudaError_t launch_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* hints_in,
                                 int hint_bits, bool guided, uint8_t* codes, uint8_t* scales,
                                 float* row_scales, uint8_t* hints_out,
                                 unsigned long long* stats4, cudaStream_t s);
cudaError_t launch_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t sf_cols,
                                 uint8_t* out, cudaStream_t s);
// group_rows: device prefix offsets [groups + 1] of the A rows of each group
// (multiples of 128); null with groups == 1 for a plain GEMM.  B holds the
// groups' weights stacked [groups * n, k], b_ts one tensor scale per group.
cudaError_t launch_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_ts,
                                 const uint8_t* b_codes, const uint8_t* b_sf, const float* b_ts,
                                 const int32_t* group_rows, int64_t groups, int64_t m, int64_t n,
                                 int64_t k, uint32_t* ws, uint8_t* codes, uint8_t* scales,
                                 uint8_t* scales_mma, float* tensor_scale, uint8_t* hints,
                                 int hint_bits, float* d_out, cudaStream_t s);
cudaError_t launch_wait_selftest(uint32_t* ws, cudaStream_t s);
cudaError_t launch_measure_mul_wide(int ctas, int iters, unsigned long long* cycles, uint32_t* sink,
                                    cudaStream_t s);
// MoE dispatch on one GPU: stable grouping of the top-k assignments by expert
// (ws: route_ws_words(A, E) words) and the gather of the routed NVFP4 rows.
constexpr int kRouteMaxExperts = 1024;
int64_t route_chunks(int64_t assignments);
cudaError_t launch_moe_route(const int32_t* ids, int64_t A, int E, int32_t* ws, int32_t* expert_rows,
                             int32_t* row_src, int64_t m_cap, int32_t* assign_row, cudaStream_t s);
cudaError_t launch_moe_gather(const uint8_t* codes, const uint8_t* scales, int64_t k,
                              const int32_t* row_src, int64_t m_cap, int64_t A, int64_t top_k,
                              uint8_t* a_codes, uint8_t* a_scales_mma, cudaStream_t s);
// Hint transport: gathers `count` device streams (srcs/sizes are host arrays)
// into `staging`, each stream starting on a 16-byte boundary, padding zeroed.
constexpr int kPackMaxStreams = 128;  // streams per launch (more take several launches)
cudaError_t launch_hint_pack(const uint8_t* const* srcs, const int64_t* sizes, int64_t count,
                             uint8_t* staging, cudaStream_t s);
cudaError_t launch_set_f32(float* dst, float value, cudaStream_t s);

// Records e (when not cudaSuccess) as the calling thread's last CUDA error
// (nvfp4_last_cuda_error) and returns the matching status.
nvfp4_status status_from_cuda(cudaError_t e);

}  // namespace nvfp4
