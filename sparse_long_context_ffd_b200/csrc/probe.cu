// probe.cu -- streaming-read bandwidth probe.
//
// Not part of the method: a reference point for the decode kernel's roofline.
// The decode step is almost entirely a one-pass read of HBM (packed keys,
// scales, K and V), while the usual bandwidth figure is a copy (read +
// write).  This kernel reads a buffer once, with 16-byte non-allocating loads
// spread over a grid of 4 CTAs x 512 threads per SM and eight loads in flight
// per thread, and folds the data into a word that is stored only if it equals
// a constant (so no load can be dropped as dead code).
#include <cuda_runtime.h>

#include <cstdint>

#include "ffd.h"

namespace ffd {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__device__ __forceinline__ uint4 load_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kProbeThreads) read_probe_kernel(const uint4 *__restrict__ buf, size_t n16,
                                                                   uint32_t *sink) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0u;
  for (; i + (kProbeUnroll - 1) * stride < n16; i += kProbeUnroll * stride) {
    uint4 v[kProbeUnroll];
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) v[u] = load_stream(buf + i + u * stride);
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = load_stream(buf + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (acc == 0x9E3779B9u) sink[0] = acc;
}

}  // namespace
}  // namespace ffd

extern "C" ffd_status ffd_read_probe(const void *buf, size_t bytes, uint32_t *sink, void *cuda_stream) {
  if (buf == nullptr || sink == nullptr || bytes == 0 || (bytes & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(buf) & 15u) != 0)
    return FFD_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FFD_ERR_CUDA;
  const size_t n16 = bytes / 16;
  const size_t per_wave = static_cast<size_t>(sms) * 4 * ffd::kProbeThreads;
  const unsigned grid = static_cast<unsigned>(n16 < per_wave ? (n16 + ffd::kProbeThreads - 1) / ffd::kProbeThreads
                                                             : static_cast<size_t>(sms) * 4);
  ffd::read_probe_kernel<<<grid, ffd::kProbeThreads, 0, static_cast<cudaStream_t>(cuda_stream)>>>(
      static_cast<const uint4 *>(buf), n16, sink);
  return cudaGetLastError() == cudaSuccess ? FFD_OK : FFD_ERR_CUDA;
}
