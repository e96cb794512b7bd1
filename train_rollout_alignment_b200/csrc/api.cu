// api.cu -- the C ABI of libnvfp4trace.so (declared in include/nvfp4_trace.h).
// Validates every argument before anything is enqueued, then launches the
// kernels on the caller's stream.  No allocation, no synchronisation, no host
// copies of device data.
#include <cstdint>

#include "../../include/nvfp4_trace.h"
#include "launch.h"

namespace {
// The CUDA error behind the calling thread's most recent NVFP4_ERR_CUDA.
thread_local int g_last_cuda_error = 0;
}  // namespace

nvfp4_status nvfp4::status_from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  g_last_cuda_error = static_cast<int>(e);
  return NVFP4_ERR_CUDA;
}

namespace {

constexpr int64_t kMaxElems = int64_t(1) << 40;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

nvfp4_status from_cuda(cudaError_t e) { return nvfp4::status_from_cuda(e); }

// Shape checks shared by the [rows, cols] entry points.
nvfp4_status check_shape(int64_t rows, int64_t cols, int64_t col_multiple) {
  if (rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (cols % col_multiple != 0) return NVFP4_ERR_SHAPE;
  if (rows != 0 && cols > kMaxElems / rows) return NVFP4_ERR_SHAPE;
  return NVFP4_OK;
}

nvfp4_status check_hint_bits(int hint_bits) {
  return (hint_bits == 1 || hint_bits == 2 || hint_bits == 4) ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED;
}

// Output buffers that every quantizing call writes.
nvfp4_status check_quant_outputs(const uint32_t* ws, const uint8_t* codes, const uint8_t* scales,
                                 const float* tensor_scale) {
  if (!ws || !codes || !scales || !tensor_scale) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ws, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(tensor_scale, 4))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

// Empty tensor: A = 0, so s_t = 1 is the only output.
nvfp4_status write_unit_scale(float* tensor_scale, void* stream) {
  if (!tensor_scale) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(tensor_scale, 4)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_set_f32(tensor_scale, 1.0f, static_cast<cudaStream_t>(stream)));
}

}  // namespace

namespace nvfp4 {

// Argument checks of the SR transpose entry points other than the scratch
// words (shared by the allocating and the no-allocation forms, so both return
// the same status for the same arguments).  batch == 0 passes with any
// pointers: such a call does nothing.
nvfp4_status check_sr_transpose_args(const uint8_t* codes, const uint8_t* scales,
                                     const float* tensor_scale, int64_t batch, int64_t rows,
                                     int64_t cols, const uint8_t* codes_t, const uint8_t* scales_t,
                                     const float* tensor_scale_t) {
  if (batch < 0 || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (rows % 16 != 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (batch > 65535 || rows / 64 >= 65535) return NVFP4_ERR_SHAPE;
  if (rows != 0 && cols > kMaxElems / rows) return NVFP4_ERR_SHAPE;
  if (batch != 0 && rows * cols > kMaxElems / batch) return NVFP4_ERR_SHAPE;
  if (batch == 0) return NVFP4_OK;
  if (!codes || !scales || !tensor_scale || !codes_t || !scales_t || !tensor_scale_t)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(codes_t, 16) ||
      !aligned(scales_t, 16) || !aligned(tensor_scale, 4) || !aligned(tensor_scale_t, 4))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

}  // namespace nvfp4

extern "C" {

const char* nvfp4_status_string(nvfp4_status status) {
  switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad flag)";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer";
    case NVFP4_ERR_SHAPE: return "unsupported shape";
    case NVFP4_ERR_CUDA: return "CUDA launch failed";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported hint_bits (expected 1, 2 or 4)";
    case NVFP4_ERR_SCRATCH_LIMIT:
      return "batch exceeds the fixed scratch of the no-allocation entry point "
             "(NVFP4_SR_NOALLOC_MAX_BATCH matrices)";
    default: return "unknown status";
  }
}

int nvfp4_last_cuda_error(void) { return g_last_cuda_error; }

const char* nvfp4_last_cuda_error_string(void) {
  return g_last_cuda_error == 0 ? "no error" : cudaGetErrorString(static_cast<cudaError_t>(g_last_cuda_error));
}

nvfp4_status nvfp4_tensor_amax(const uint16_t* x_bf16, int64_t n, uint32_t* ws, void* stream) {
  if (!ws || (n > 0 && !x_bf16)) return NVFP4_ERR_INVALID_ARG;
  if (n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n % 16 != 0 || n >= kMaxElems) return NVFP4_ERR_SHAPE;
  if (!aligned(ws, 16) || !aligned(x_bf16, 32)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_amax_bf16(x_bf16, n / 16, ws, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_quantize_rtn(const uint16_t* x_bf16, int64_t rows, int64_t cols, uint32_t* ws,
                                int flags, uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                uint8_t* hints, int hint_bits, void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if ((flags & ~NVFP4_AMAX_PRECOMPUTED) != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows * cols == 0) return write_unit_scale(tensor_scale, stream);
  if (!x_bf16) return NVFP4_ERR_INVALID_ARG;
  if ((st = check_quant_outputs(ws, codes, scales, tensor_scale)) != NVFP4_OK) return st;
  if (hints) {
    if ((st = check_hint_bits(hint_bits)) != NVFP4_OK) return st;
    if (!aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  }
  if (!aligned(x_bf16, 32)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  if (!(flags & NVFP4_AMAX_PRECOMPUTED)) {
    st = nvfp4_tensor_amax(x_bf16, n, ws, stream);
    if (st != NVFP4_OK) return st;
  }
  return from_cuda(nvfp4::launch_quantize_rtn(x_bf16, n / 16, ws, codes, scales, tensor_scale,
                                              hints, hints ? hint_bits : 0, s));
}

nvfp4_status nvfp4_emit_hint(const uint8_t* codes, int64_t n, int hint_bits, uint8_t* hints,
                             void* stream) {
  if (n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n > 0 && (!codes || !hints)) return NVFP4_ERR_INVALID_ARG;
  nvfp4_status st = check_hint_bits(hint_bits);
  if (st != NVFP4_OK) return st;
  if (n % 16 != 0 || n >= kMaxElems) return NVFP4_ERR_SHAPE;
  if (!aligned(codes, 16) || !aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_emit_hint(codes, n / 16, hint_bits, hints,
                                           static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_guided_requant(const uint16_t* x_train_bf16, int64_t rows, int64_t cols,
                                  const uint8_t* hints, int hint_bits, uint32_t* ws, int flags,
                                  uint8_t* codes, uint8_t* scales, float* tensor_scale,
                                  uint64_t* stats4, void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if ((flags & ~NVFP4_AMAX_PRECOMPUTED) != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows * cols == 0) return write_unit_scale(tensor_scale, stream);
  if (!x_train_bf16) return NVFP4_ERR_INVALID_ARG;
  if ((st = check_quant_outputs(ws, codes, scales, tensor_scale)) != NVFP4_OK) return st;
  if (hints) {
    if ((st = check_hint_bits(hint_bits)) != NVFP4_OK) return st;
    if (!aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  }
  if (!aligned(x_train_bf16, 32)) return NVFP4_ERR_MISALIGNED;
  if (stats4 && !aligned(stats4, 8)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  if (!(flags & NVFP4_AMAX_PRECOMPUTED)) {
    st = nvfp4_tensor_amax(x_train_bf16, n, ws, stream);
    if (st != NVFP4_OK) return st;
  }
  return from_cuda(nvfp4::launch_guided(x_train_bf16, n / 16, hints, hint_bits, ws, codes, scales,
                                        tensor_scale,
                                        reinterpret_cast<unsigned long long*>(stats4), s));
}

nvfp4_status nvfp4_guided_requant_stats(const uint16_t* x_train_bf16, int64_t rows, int64_t cols,
                                        const uint8_t* hints, int hint_bits, uint32_t* ws,
                                        int flags, uint8_t* codes, uint8_t* scales,
                                        float* tensor_scale, uint64_t* stats4,
                                        const uint8_t* roll_codes, const uint8_t* roll_scales,
                                        const float* roll_tensor_scale, uint64_t* stats8,
                                        void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if ((flags & ~NVFP4_AMAX_PRECOMPUTED) != 0) return NVFP4_ERR_INVALID_ARG;
  if (rows * cols == 0) return write_unit_scale(tensor_scale, stream);
  if (!x_train_bf16 || !roll_codes || !roll_scales || !roll_tensor_scale || !stats8)
    return NVFP4_ERR_INVALID_ARG;
  if ((st = check_quant_outputs(ws, codes, scales, tensor_scale)) != NVFP4_OK) return st;
  if (hints) {
    if ((st = check_hint_bits(hint_bits)) != NVFP4_OK) return st;
    if (!aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  }
  if (!aligned(x_train_bf16, 32) || !aligned(roll_codes, 16) || !aligned(roll_scales, 16) ||
      !aligned(roll_tensor_scale, 4) || !aligned(stats8, 8) || (stats4 && !aligned(stats4, 8)))
    return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  if (!(flags & NVFP4_AMAX_PRECOMPUTED)) {
    st = nvfp4_tensor_amax(x_train_bf16, n, ws, stream);
    if (st != NVFP4_OK) return st;
  }
  return from_cuda(nvfp4::launch_guided_stats(
      x_train_bf16, n / 16, hints, hint_bits, ws, codes, scales, tensor_scale,
      reinterpret_cast<unsigned long long*>(stats4), roll_codes, roll_scales, roll_tensor_scale,
      reinterpret_cast<unsigned long long*>(stats8), s));
}

nvfp4_status nvfp4_mismatch_stats(const uint8_t* codes_a, const uint8_t* scales_a,
                                  const float* ts_a, const uint8_t* codes_b,
                                  const uint8_t* scales_b, const float* ts_b, int64_t rows,
                                  int64_t cols, uint64_t* stats8, void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if (rows * cols == 0) return NVFP4_OK;
  if (!codes_a || !scales_a || !ts_a || !codes_b || !scales_b || !ts_b || !stats8)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes_a, 16) || !aligned(codes_b, 16) || !aligned(scales_a, 16) ||
      !aligned(scales_b, 16) || !aligned(ts_a, 4) || !aligned(ts_b, 4) || !aligned(stats8, 8))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_mismatch_stats(codes_a, scales_a, ts_a, codes_b, scales_b, ts_b,
                                                rows * cols / 16,
                                                reinterpret_cast<unsigned long long*>(stats8),
                                                static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                        const float* tensor_scale, int64_t batch, int64_t rows,
                                        int64_t cols, uint64_t seed, uint32_t draw, uint32_t* ws,
                                        uint8_t* codes_t, uint8_t* scales_t,
                                        float* tensor_scale_t, void* stream) {
  nvfp4_status st = nvfp4::check_sr_transpose_args(codes, scales, tensor_scale, batch, rows, cols,
                                                    codes_t, scales_t, tensor_scale_t);
  if (st != NVFP4_OK || batch == 0) return st;
  if (!ws) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_sr_transpose(codes, scales, tensor_scale, batch, rows, cols, seed,
                                              draw, ws, codes_t, scales_t, tensor_scale_t,
                                              static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_rht_quantize(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                uint64_t sign_seed, uint32_t* ws, uint8_t* codes, uint8_t* scales,
                                float* tensor_scale, float* y_out, void* stream) {
  nvfp4_status st = check_shape(rows, cols, 32);
  if (st != NVFP4_OK) return st;
  if (rows * cols == 0) return write_unit_scale(tensor_scale, stream);
  if (!x_bf16) return NVFP4_ERR_INVALID_ARG;
  if ((st = check_quant_outputs(ws, codes, scales, tensor_scale)) != NVFP4_OK) return st;
  if (!aligned(x_bf16, 32) || (y_out && !aligned(y_out, 32))) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_rht_quantize(x_bf16, rows * cols / 16, sign_seed, ws, codes,
                                              scales, tensor_scale, y_out,
                                              static_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------------------------- KV-cache rows
namespace {
nvfp4_status check_rows(const uint16_t* x, int64_t rows, int64_t cols, const uint8_t* codes,
                        const uint8_t* scales, const float* row_scales) {
  if (rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (cols != 16 && cols != 32 && cols != 64 && cols != 128 && cols != 256 && cols != 512)
    return NVFP4_ERR_SHAPE;
  if (rows > kMaxElems / cols) return NVFP4_ERR_SHAPE;
  if (rows == 0) return NVFP4_OK;
  if (!x || !codes || !scales || !row_scales) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(x, 32) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(row_scales, 4))
    return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}
}  // namespace

nvfp4_status nvfp4_quantize_rtn_rows(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                     uint8_t* codes, uint8_t* scales, float* row_scales,
                                     uint8_t* hints, int hint_bits, void* stream) {
  nvfp4_status st = check_rows(x_bf16, rows, cols, codes, scales, row_scales);
  if (st != NVFP4_OK || rows == 0) return st;
  if (hints) {
    if ((st = check_hint_bits(hint_bits)) != NVFP4_OK) return st;
    if (!aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  }
  return from_cuda(nvfp4::launch_quantize_rows(x_bf16, rows, cols, nullptr, hint_bits, false, codes,
                                               scales, row_scales, hints, nullptr,
                                               static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_guided_requant_rows(const uint16_t* x_bf16, int64_t rows, int64_t cols,
                                       const uint8_t* hints, int hint_bits, uint8_t* codes,
                                       uint8_t* scales, float* row_scales, uint64_t* stats4,
                                       void* stream) {
  nvfp4_status st = check_rows(x_bf16, rows, cols, codes, scales, row_scales);
  if (st != NVFP4_OK || rows == 0) return st;
  if (hints) {
    if ((st = check_hint_bits(hint_bits)) != NVFP4_OK) return st;
    if (!aligned(hints, 16)) return NVFP4_ERR_MISALIGNED;
  }
  if (stats4 && !aligned(stats4, 8)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!hints)  // no guidance: round-to-nearest
    return from_cuda(nvfp4::launch_quantize_rows(x_bf16, rows, cols, nullptr, 0, false, codes, scales,
                                                 row_scales, nullptr, nullptr, s));
  return from_cuda(nvfp4::launch_quantize_rows(x_bf16, rows, cols, hints, hint_bits, true, codes,
                                               scales, row_scales, nullptr,
                                               reinterpret_cast<unsigned long long*>(stats4), s));
}

// ----------------------------------------------------------------- alternatives to SR transpose
nvfp4_status nvfp4_quantize_tile16(const uint16_t* x_bf16, int64_t rows, int64_t cols, uint32_t* ws,
                                   int flags, uint8_t* codes, uint8_t* tile_scales,
                                   float* tensor_scale, void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if (rows % 16 != 0) return NVFP4_ERR_SHAPE;
  if (flags & ~NVFP4_AMAX_PRECOMPUTED) return NVFP4_ERR_INVALID_ARG;
  if (rows * cols == 0) return write_unit_scale(tensor_scale, stream);
  if (!x_bf16) return NVFP4_ERR_INVALID_ARG;
  if ((st = check_quant_outputs(ws, codes, tile_scales, tensor_scale)) != NVFP4_OK) return st;
  if (!aligned(x_bf16, 32)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!(flags & NVFP4_AMAX_PRECOMPUTED)) {
    if ((st = from_cuda(nvfp4::launch_amax_bf16(x_bf16, rows * cols / 16, ws, s))) != NVFP4_OK)
      return st;
  }
  return from_cuda(nvfp4::launch_quantize_tile16(x_bf16, rows, cols, ws, codes, tile_scales,
                                                 tensor_scale, s));
}

nvfp4_status nvfp4_transpose_tile16(const uint8_t* codes, const uint8_t* tile_scales, int64_t batch,
                                    int64_t rows, int64_t cols, uint8_t* codes_t,
                                    uint8_t* tile_scales_t, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (rows % 16 != 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (batch > 65535 || rows / 128 >= 65535) return NVFP4_ERR_SHAPE;
  if (rows != 0 && cols > kMaxElems / rows) return NVFP4_ERR_SHAPE;
  if (batch != 0 && rows * cols > kMaxElems / batch) return NVFP4_ERR_SHAPE;
  if (batch == 0 || rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !tile_scales || !codes_t || !tile_scales_t) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(tile_scales, 16) || !aligned(codes_t, 16) ||
      !aligned(tile_scales_t, 16))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_transpose_tile16(codes, tile_scales, batch, rows, cols, codes_t,
                                                  tile_scales_t, static_cast<cudaStream_t>(stream)));
}

nvfp4_status mxfp8_sr_transpose_requant(const uint8_t* codes, const uint8_t* scales,
                                        const float* tensor_scale, int64_t batch, int64_t rows,
                                        int64_t cols, uint64_t seed, uint32_t draw, uint8_t* q_t,
                                        uint8_t* e8_t, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (rows % 32 != 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (batch > 65535 || rows / 128 >= 65535) return NVFP4_ERR_SHAPE;
  if (rows != 0 && cols > kMaxElems / rows) return NVFP4_ERR_SHAPE;
  if (batch != 0 && rows * cols > kMaxElems / batch) return NVFP4_ERR_SHAPE;
  if (batch == 0 || rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !scales || !tensor_scale || !q_t || !e8_t) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(q_t, 16) || !aligned(e8_t, 16) ||
      !aligned(tensor_scale, 4))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_mxfp8_sr_transpose(codes, scales, tensor_scale, batch, rows, cols,
                                                    seed, draw, q_t, e8_t,
                                                    static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale,
                              int64_t rows, int64_t cols, int scale_layout, float* out,
                              void* stream) {
  nvfp4_status st = check_shape(rows, cols, 16);
  if (st != NVFP4_OK) return st;
  if (scale_layout != NVFP4_SCALES_BLOCK16 && scale_layout != NVFP4_SCALES_TILE16)
    return NVFP4_ERR_INVALID_ARG;
  if (scale_layout == NVFP4_SCALES_TILE16 && rows % 16 != 0) return NVFP4_ERR_SHAPE;
  if (rows * cols == 0) return NVFP4_OK;
  if (!codes || !scales || !tensor_scale || !out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(tensor_scale, 4) || !aligned(out, 32))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_dequant_nvfp4(codes, scales, tensor_scale, rows, cols,
                                               scale_layout == NVFP4_SCALES_TILE16, out,
                                               static_cast<cudaStream_t>(stream)));
}

nvfp4_status mxfp8_dequantize(const uint8_t* q, const uint8_t* e8, int64_t n, float* out,
                              void* stream) {
  if (n < 0) return NVFP4_ERR_INVALID_ARG;
  if (n % 32 != 0 || n >= kMaxElems) return NVFP4_ERR_SHAPE;
  if (n == 0) return NVFP4_OK;
  if (!q || !e8 || !out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(e8, 16) || !aligned(out, 32)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_dequant_mxfp8(q, e8, n, out, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t sf_cols,
                                 uint8_t* scales_mma, void* stream) {
  if (rows < 0 || sf_cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (rows != 0 && sf_cols > kMaxElems / 16 / rows) return NVFP4_ERR_SHAPE;
  if (rows == 0 || sf_cols == 0) return NVFP4_OK;
  if (!scales || !scales_mma) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(scales_mma, 16)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_scales_to_mma(scales, rows, sf_cols, scales_mma,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

nvfp4_status gemm_quantize(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                           const float* a_tensor_scale, const uint8_t* b_codes,
                           const uint8_t* b_scales_mma, const float* b_tensor_scales,
                           const int32_t* group_rows, int64_t groups, int64_t m, int64_t n,
                           int64_t k, uint32_t* ws, uint8_t* codes, uint8_t* scales,
                           uint8_t* scales_mma, float* tensor_scale, uint8_t* hints,
                           int hint_bits, float* d_out, void* stream) {
  if (m < 0 || n < 0 || k < 0) return NVFP4_ERR_INVALID_ARG;
  if (m % 128 != 0 || n % 128 != 0 || k % 256 != 0 || k == 0) return NVFP4_ERR_SHAPE;
  if (m >= kMaxElems || n >= kMaxElems || k >= (int64_t(1) << 31) ||
      (m != 0 && n > kMaxElems / m) || (m != 0 && k > kMaxElems / m) ||
      (n != 0 && k > kMaxElems / n) || (n != 0 && groups > kMaxElems / n / k))
    return NVFP4_ERR_SHAPE;
  if (!ws || !tensor_scale) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ws, 16) || !aligned(tensor_scale, 4)) return NVFP4_ERR_MISALIGNED;
  if (hints != nullptr) {
    nvfp4_status st = check_hint_bits(hint_bits);
    if (st != NVFP4_OK) return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m == 0 || n == 0)
    return from_cuda(nvfp4::launch_gemm_quantize(nullptr, nullptr, nullptr, nullptr, nullptr,
                                                 nullptr, nullptr, 1, m, n, k, ws, nullptr,
                                                 nullptr, nullptr, tensor_scale, nullptr, 0,
                                                 nullptr, s));
  if (!a_codes || !a_scales_mma || !a_tensor_scale || !b_codes || !b_scales_mma ||
      !b_tensor_scales || !codes || !scales || (groups > 1 && !group_rows))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales_mma, 16) || !aligned(a_tensor_scale, 4) ||
      !aligned(b_codes, 16) || !aligned(b_scales_mma, 16) || !aligned(b_tensor_scales, 4) ||
      !aligned(group_rows, 4) || !aligned(codes, 32) || !aligned(scales, 16) ||
      !aligned(scales_mma, 16) || !aligned(hints, 32) || !aligned(d_out, 32))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_gemm_quantize(
      a_codes, a_scales_mma, a_tensor_scale, b_codes, b_scales_mma, b_tensor_scales,
      groups > 1 ? group_rows : nullptr, groups, m, n, k, ws, codes, scales, scales_mma,
      tensor_scale, hints, hint_bits, d_out, s));
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                 const float* a_tensor_scale, const uint8_t* b_codes,
                                 const uint8_t* b_scales_mma, const float* b_tensor_scale,
                                 int64_t m, int64_t n, int64_t k, uint32_t* ws, uint8_t* codes,
                                 uint8_t* scales, uint8_t* scales_mma, float* tensor_scale,
                                 uint8_t* hints, int hint_bits, float* d_out, void* stream) {
  return gemm_quantize(a_codes, a_scales_mma, a_tensor_scale, b_codes, b_scales_mma,
                       b_tensor_scale, nullptr, 1, m, n, k, ws, codes, scales, scales_mma,
                       tensor_scale, hints, hint_bits, d_out, stream);
}

nvfp4_status nvfp4_moe_gemm_quantize(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                     const float* a_tensor_scale, const uint8_t* w_codes,
                                     const uint8_t* w_scales_mma, const float* w_tensor_scales,
                                     const int32_t* expert_rows, int64_t experts, int64_t m,
                                     int64_t n, int64_t k, uint32_t* ws, uint8_t* codes,
                                     uint8_t* scales, uint8_t* scales_mma, float* tensor_scale,
                                     uint8_t* hints, int hint_bits, float* d_out, void* stream) {
  if (experts < 1 || experts > 65536) return NVFP4_ERR_INVALID_ARG;
  return gemm_quantize(a_codes, a_scales_mma, a_tensor_scale, w_codes, w_scales_mma,
                       w_tensor_scales, expert_rows, experts, m, n, k, ws, codes, scales,
                       scales_mma, tensor_scale, hints, hint_bits, d_out, stream);
}

int64_t nvfp4_hint_pack_size(const int64_t* sizes, int64_t count) {
  if (count < 0 || (count > 0 && !sizes)) return -1;
  int64_t total = 0;
  for (int64_t i = 0; i < count; ++i) {
    if (sizes[i] < 0 || sizes[i] >= kMaxElems) return -1;
    total += (sizes[i] + 15) / 16 * 16;
    if (total >= kMaxElems) return -1;
  }
  return total;
}

nvfp4_status nvfp4_hint_pack(const uint8_t* const* srcs, const int64_t* sizes, int64_t count,
                             uint8_t* staging, uint8_t* host_dst, void* stream) {
  if (count < 0 || (count > 0 && (!srcs || !sizes))) return NVFP4_ERR_INVALID_ARG;
  for (int64_t i = 0; i < count; ++i) {
    if (sizes[i] < 0) return NVFP4_ERR_INVALID_ARG;
    if (sizes[i] > 0 && !srcs[i]) return NVFP4_ERR_INVALID_ARG;
  }
  const int64_t total = nvfp4_hint_pack_size(sizes, count);
  if (total < 0) return NVFP4_ERR_SHAPE;
  if (total == 0) return NVFP4_OK;
  if (!staging) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(staging, 16)) return NVFP4_ERR_MISALIGNED;
  for (int64_t i = 0; i < count; ++i)
    if (sizes[i] > 0 && !aligned(srcs[i], 16)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  nvfp4_status st = from_cuda(nvfp4::launch_hint_pack(srcs, sizes, count, staging, s));
  if (st != NVFP4_OK || !host_dst) return st;
  return from_cuda(cudaMemcpyAsync(host_dst, staging, (size_t)total, cudaMemcpyDeviceToHost, s));
}

int64_t nvfp4_moe_rows_cap(int64_t assignments, int64_t experts) {
  if (assignments < 0 || experts < 1 || experts > nvfp4::kRouteMaxExperts ||
      assignments >= (int64_t(1) << 31) - 128 * 1024)
    return -1;
  return (assignments + 127 * experts) / 128 * 128;  // each group adds < 128 padding rows
}

int64_t nvfp4_moe_route_ws_words(int64_t assignments, int64_t experts) {
  if (nvfp4_moe_rows_cap(assignments, experts) < 0) return -1;
  return (nvfp4::route_chunks(assignments) + 1) * experts;
}

nvfp4_status nvfp4_moe_route(const int32_t* topk_ids, int64_t tokens, int64_t top_k, int64_t experts,
                             int32_t* ws, int32_t* expert_rows, int32_t* row_src, int64_t m_cap,
                             int32_t* assign_row, void* stream) {
  if (tokens < 0 || top_k < 1 || experts < 1) return NVFP4_ERR_INVALID_ARG;
  if (experts > nvfp4::kRouteMaxExperts || top_k > (int64_t(1) << 20)) return NVFP4_ERR_SHAPE;
  if (tokens > (int64_t(1) << 31) / top_k) return NVFP4_ERR_SHAPE;
  const int64_t A = tokens * top_k;
  const int64_t cap = nvfp4_moe_rows_cap(A, experts);
  if (cap < 0) return NVFP4_ERR_SHAPE;
  if (m_cap < cap) return NVFP4_ERR_SHAPE;   // too small to hold every possible grouping
  if (!ws || !expert_rows || !row_src || (A > 0 && (!topk_ids || !assign_row)))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ws, 16) || !aligned(expert_rows, 4) || !aligned(row_src, 4) ||
      !aligned(topk_ids, 4) || !aligned(assign_row, 4))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_moe_route(topk_ids, A, (int)experts, ws, expert_rows, row_src, m_cap,
                                           assign_row, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_moe_gather(const uint8_t* codes, const uint8_t* scales, int64_t tokens, int64_t k,
                              const int32_t* row_src, int64_t m_cap, int64_t top_k, uint8_t* a_codes,
                              uint8_t* a_scales_mma, void* stream) {
  if (tokens < 0 || k < 0 || m_cap < 0 || top_k < 1) return NVFP4_ERR_INVALID_ARG;
  if (k % 64 != 0 || m_cap % 128 != 0) return NVFP4_ERR_SHAPE;
  if (tokens > (int64_t(1) << 31) / top_k || (k != 0 && m_cap > kMaxElems / k) ||
      (k != 0 && tokens > kMaxElems / k))
    return NVFP4_ERR_SHAPE;
  if (m_cap == 0 || k == 0) return NVFP4_OK;
  if (!row_src || !a_codes || !a_scales_mma || (tokens > 0 && (!codes || !scales)))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(scales, 16) || !aligned(row_src, 4) || !aligned(a_codes, 16) ||
      !aligned(a_scales_mma, 16))
    return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_moe_gather(codes, scales, k, row_src, m_cap, tokens * top_k, top_k,
                                            a_codes, a_scales_mma, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_measure_mul_wide(int64_t ctas, int64_t iters, uint64_t* cycles, uint32_t* sink,
                                    void* stream) {
  if (ctas < 1 || ctas > 65535 || iters < 1 || iters > (int64_t(1) << 24) || !cycles || !sink)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(cycles, 8) || !aligned(sink, 4)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_measure_mul_wide((int)ctas, (int)iters,
                                                  reinterpret_cast<unsigned long long*>(cycles), sink,
                                                  static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_wait_selftest(uint32_t* ws, void* stream) {
  if (!ws) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(ws, 16)) return NVFP4_ERR_MISALIGNED;
  return from_cuda(nvfp4::launch_wait_selftest(ws, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
