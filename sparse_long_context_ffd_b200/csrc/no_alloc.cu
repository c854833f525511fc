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
// are cleared on the stream at the start of every call.  Calls whose
// executions overlap on the GPU (different streams, or different host
// threads without ordering) race on the array and give undefined results.
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
// symbol is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
void *scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
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
  void *scratch = ffd::scratch_for_current_device();
  if (scratch == nullptr) return FFD_ERR_CUDA;
  // error word and arrival counters must start at zero
  const ffd::WorkspaceLayout L = ffd::workspace_layout(
      s->batch, s->num_kv_heads, s->num_q_heads / s->num_kv_heads, s->capacity, s->block_size,
      s->split_blocks);
  if (cudaMemsetAsync(scratch, 0, L.split_bits, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FFD_ERR_CUDA;
  return ffd_decode(s, q_bf16, k_bf16, v_bf16, k_packed, k_scales, d_lengths, delta, out_bf16, mask,
                    scratch, need, cuda_stream);
}
