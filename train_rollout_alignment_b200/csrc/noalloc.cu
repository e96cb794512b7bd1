// noalloc.cu -- nvfp4_sr_transpose_requant_noalloc: the SR transpose
// re-quantization for callers that cannot allocate device memory.
//
// Some callers have no way to hand this library a scratch buffer: a rollout or
// serving engine that reserved (nearly) all of HBM for its weight and KV-cache
// pools at start-up and forbids any later cudaMalloc, or plain C/C++ code that
// links only this library, has no caching allocator, and must not pay the
// device-wide synchronisation that cudaMalloc/cudaFree can imply in the middle
// of a step.  For them, the per-matrix scratch words that
// nvfp4_sr_transpose_requant takes as `ws` live instead in the file-scope
// array below, a fixed NVFP4_SR_NOALLOC_MAX_BATCH words (16 KiB) that every GPU
// which loads this library keeps until the process exits.
//
// Host code must not use the array's name as a pointer (on the host it is a
// stand-in, not a device address): its device address is fetched once per
// device with cudaGetSymbolAddress, with that device current, and cached.  The
// cached address belongs to the device's primary context as it was at that
// first call; a process that resets the device (cudaDeviceReset) or otherwise
// destroys and recreates its primary context must not call this entry point
// afterwards.
#include <cstdint>
#include <mutex>

#include "../../include/nvfp4_trace.h"
#include "launch.h"

static __device__ __align__(256) uint32_t g_sr_scratch[NVFP4_SR_NOALLOC_MAX_BATCH];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
uint32_t* g_scratch_addr[kMaxDevices] = {};

// Device address of g_sr_scratch on the current device (set up on first use).
nvfp4_status scratch_on_current_device(uint32_t** out) {
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return nvfp4::status_from_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return nvfp4::status_from_cuda(cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t ea = cudaGetSymbolAddress(&p, g_sr_scratch);
    if (ea != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return nvfp4::status_from_cuda(ea != cudaSuccess ? ea : cudaErrorInvalidSymbol);
    }
    g_scratch_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_addr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_sr_transpose_requant_noalloc(
    const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t batch,
    int64_t rows, int64_t cols, uint64_t seed, uint32_t draw, uint8_t* codes_t, uint8_t* scales_t,
    float* tensor_scale_t, void* stream) {
  // The allocating entry point's own checks first, so both forms return the
  // same status for the same arguments; an empty batch does nothing and needs
  // no scratch.
  nvfp4_status st = nvfp4::check_sr_transpose_args(codes, scales, tensor_scale, batch, rows, cols,
                                                    codes_t, scales_t, tensor_scale_t);
  if (st != NVFP4_OK || batch == 0) return st;
  if (batch > NVFP4_SR_NOALLOC_MAX_BATCH) return NVFP4_ERR_SCRATCH_LIMIT;
  uint32_t* ws = nullptr;
  if ((st = scratch_on_current_device(&ws)) != NVFP4_OK) return st;
  // Same kernels as the allocating entry point; it clears the `batch`
  // scratch words on `stream` before the kernels use them.
  return nvfp4_sr_transpose_requant(codes, scales, tensor_scale, batch, rows, cols, seed, draw, ws,
                                    codes_t, scales_t, tensor_scale_t, stream);
}
