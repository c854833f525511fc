// no_alloc.cu -- ffd_decode_no_alloc: the fused decode step for callers that
// cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a plug-in inside an
// inference engine that is handed only its input and output buffers, or a
// serving loop that forbids cudaMalloc after start-up because an allocation
// can synchronise the device and stall every stream.  This entry point runs
// the same kernel as ffd_decode, with the kernel's scratch (split partials,
// per-split selection bits, arrival counters, error word) placed in a fixed
// device array that is part of this library's image.
//
// The array costs kNoAllocScratchBytes (16 MiB) on every GPU that loads the
// library, for the life of the process.  All calls on a device share it and
// it keeps whatever the previous call left; the counters and the error word
// are cleared on the stream at the start of every call that passes its host
// checks.  Calls whose executions overlap on the GPU (different streams, or
// different host threads without ordering) race on the array and give
// undefined results.  ffd_no_alloc_device_status reads the error word that the
// last call left (a bad length, or a bounded wait that ran out).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "ffd.h"
#include "ffd_internal.h"

namespace ffd {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up with the
// device current: on every call made outside a stream capture (a device reset
// reloads this library's image, and the array may then sit elsewhere), and
// from the copy cached by the last such call while `stream` is being captured
// (a lookup may load the module, which a capture does not allow).
void *scratch_for_current_device(cudaStream_t stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool capturing =
      cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!capturing) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
  } else {
    (void)cudaGetLastError();  // (a failed capture query leaves no sticky error)
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace ffd

extern "C" ffd_status ffd_decode_no_alloc(const ffd_shape *s, const void *q_bf16, const void *k_bf16,
                                          const void *v_bf16, const void *k_packed,
                                          const void *k_scales, const int32_t *d_lengths, float delta,
                                          void *out_bf16, uint32_t *mask, void *cuda_stream) {
  const size_t need = ffd_decode_workspace_bytes(s);
  if (need == 0)  // invalid shape: let ffd_decode report which check failed
    return ffd_decode(s, q_bf16, k_bf16, v_bf16, k_packed, k_scales, d_lengths, delta, out_bf16,
                      mask, nullptr, 0, cuda_stream);
  if (need > ffd::kNoAllocScratchBytes) return FFD_ERR_WORKSPACE;
  if (s->batch == 0)
    return ffd_decode(s, q_bf16, k_bf16, v_bf16, k_packed, k_scales, d_lengths, delta, out_bf16,
                      mask, nullptr, need, cuda_stream);
  void *scratch = ffd::scratch_for_current_device(static_cast<cudaStream_t>(cuda_stream));
  if (scratch == nullptr) return FFD_ERR_CUDA;
  // every host check first; the array's error word and counters are cleared
  // on the stream only once the launch is certain, so a rejected call leaves
  // the array (and any call still running on it) alone
  return ffd::decode_shared_scratch(s, q_bf16, k_bf16, v_bf16, k_packed, k_scales, d_lengths, delta,
                                    out_bf16, mask, scratch, need, cuda_stream);
}

extern "C" ffd_status ffd_no_alloc_device_status(uint32_t *flags_out, void *cuda_stream) {
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
    return FFD_ERR_INVALID_ARG;  // it synchronises the stream
  void *scratch = ffd::scratch_for_current_device(stream);
  if (scratch == nullptr) return FFD_ERR_CUDA;
  return ffd_check_device_status(scratch, flags_out, cuda_stream);
}
