// transport.cu -- moving the rollout's guidance off the GPU (TRACE explainer,
// guidance-volume paragraph: the guidance of every step leaves the GPU for
// host memory or storage, and its size and that transfer decide the cost;
// compaction paragraph: only the low bits of the codes, and only for the back
// half of the layers, are shipped).
//
// The hint streams of the layers that ship guidance are separate device
// buffers (one per layer, or per layer and token in decoding).  Many small
// copies to the host are bound by per-copy latency, so one kernel first
// gathers them, back to back, into one contiguous staging buffer and one
// copy then moves it to (pinned) host memory.  Layout of the staging buffer:
// stream i starts at byte off_i = sum over j < i of round_up(size_j, 16), the
// bytes between the end of a stream and the next 16-byte boundary are zero.
// Every 16-byte unit of the staging buffer is one thread's 128-bit load and
// store (a stream's last, partial unit by bytes), so the gather streams at
// HBM bandwidth whatever the stream sizes.
#include "launch.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

constexpr int kPackCtasPerSm = 4;
constexpr int kPackUnroll = 4;

// Kernel parameters of one launch (at most kPackMaxStreams streams, well
// inside the 4 KiB parameter space); unit offsets are cumulative, off[count]
// is the launch's total number of 16-byte units.
struct PackArgs {
  const uint8_t* src[kPackMaxStreams];
  int64_t size[kPackMaxStreams];
  int64_t off[kPackMaxStreams + 1];
  int count;
};

__device__ __forceinline__ uint4 pack_unit(const PackArgs& a, int64_t u) {
  int lo = 0, hi = a.count;  // the stream s with off[s] <= u < off[s + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.off[mid] <= u) lo = mid;
    else hi = mid;
  }
  const int64_t b0 = (u - a.off[lo]) * 16;
  const int64_t left = a.size[lo] - b0;
  if (left >= 16) return __ldg(reinterpret_cast<const uint4*>(a.src[lo] + b0));
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int k = 0; k < (int)left; ++k) w[k >> 2] |= (uint32_t)__ldg(a.src[lo] + b0 + k) << (8 * (k & 3));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(kThreads, kPackCtasPerSm)
    k_hint_pack(const __grid_constant__ PackArgs a, uint4* __restrict__ dst) {
  const int64_t units = a.off[a.count];
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (; u + (kPackUnroll - 1) * stride < units; u += kPackUnroll * stride) {
    uint4 v[kPackUnroll];
#pragma unroll
    for (int k = 0; k < kPackUnroll; ++k) v[k] = pack_unit(a, u + k * stride);
#pragma unroll
    for (int k = 0; k < kPackUnroll; ++k) dst[u + k * stride] = v[k];
  }
  for (; u < units; u += stride) dst[u] = pack_unit(a, u);
}

cudaError_t launch_hint_pack(const uint8_t* const* srcs, const int64_t* sizes, int64_t count,
                             uint8_t* staging, cudaStream_t s) {
  int64_t dst_unit = 0;
  for (int64_t first = 0; first < count; first += kPackMaxStreams) {
    PackArgs a;
    a.count = (int)((count - first) < kPackMaxStreams ? (count - first) : kPackMaxStreams);
    a.off[0] = 0;
    for (int i = 0; i < a.count; ++i) {
      a.src[i] = srcs[first + i];
      a.size[i] = sizes[first + i];
      a.off[i + 1] = a.off[i] + (sizes[first + i] + 15) / 16;
    }
    for (int i = a.count; i < kPackMaxStreams; ++i) {
      a.src[i] = nullptr;
      a.size[i] = 0;
      a.off[i + 1] = a.off[a.count];
    }
    const int64_t units = a.off[a.count];
    if (units > 0) {
      k_hint_pack<<<grid_for(units, kThreads, kPackCtasPerSm), kThreads, 0, s>>>(
          a, reinterpret_cast<uint4*>(staging) + dst_unit);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    dst_unit += units;
  }
  return cudaSuccess;
}

}  // namespace nvfp4
