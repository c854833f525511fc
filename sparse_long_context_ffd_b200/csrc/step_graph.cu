// step_graph.cu -- one layer's whole decode step as a native CUDA graph.
//
// The system part of the method (Faster Than Flash, gist.science explainer,
// Methodology 3, "Fused Kernel and System Optimization": the decoding step is
// captured whole in a CUDA graph so that small batches pay no CPU launch
// overhead), done without any framework in the loop.  The graph holds the
// H2D copy of the step's query and new K/V rows from pinned host memory, the
// optional length increment, the fused append + re-quantisation + decode
// launch, and the D2H copy of the output rows and mask (or none, when the
// kernel writes them into mapped pinned host memory); ffd_step_graph_run
// launches it and waits on its private stream.
#include <cuda_runtime.h>

#include <cstdint>
#include <new>

#include "ffd.h"
#include "ffd_internal.h"

struct ffd_step_graph {
  cudaStream_t stream = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

namespace ffd {
namespace {

__global__ void advance_lengths_kernel(int32_t *lengths, int32_t batch) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) lengths[b] += 1;
}

void destroy_parts(ffd_step_graph *g) {
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  if (g->stream) cudaStreamDestroy(g->stream);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace ffd

extern "C" {

ffd_status ffd_step_graph_create(const ffd_shape *s, int32_t format, int32_t reference, float delta,
                                 int32_t advance, const void *host_in, void *dev_in, void *k_bf16,
                                 void *v_bf16, void *k_copy, void *k_resid, void *k_scales,
                                 int32_t *d_lengths, void *dev_result, void *host_result,
                                 size_t mask_offset, void *workspace, size_t workspace_bytes,
                                 ffd_step_graph **graph_out) {
  if (graph_out == nullptr) return FFD_ERR_INVALID_ARG;
  *graph_out = nullptr;
  if (s == nullptr || ffd_decode_workspace_bytes(s) == 0) return FFD_ERR_INVALID_ARG;
  if (format != 0 && format != 1) return FFD_ERR_INVALID_ARG;
  if (advance != 0 && advance != 1) return FFD_ERR_INVALID_ARG;
  if (s->batch == 0) return FFD_ERR_INVALID_ARG;
  if (host_in == nullptr || dev_in == nullptr || host_result == nullptr || d_lengths == nullptr ||
      !ffd::aligned16(dev_in) || !ffd::aligned16(dev_result) || !ffd::aligned16(host_result) ||
      (mask_offset & 15u) != 0)
    return FFD_ERR_INVALID_ARG;
  const size_t D = ffd::kHeadDim;
  const size_t nq = static_cast<size_t>(s->batch) * s->num_q_heads * D;
  const size_t nk = static_cast<size_t>(s->batch) * s->num_kv_heads * D;
  const size_t out_bytes = nq * 2;
  if (mask_offset < out_bytes) return FFD_ERR_INVALID_ARG;
  const size_t result_bytes = mask_offset + ffd_mask_words(s) * 4;
  const uint8_t *in_h = static_cast<const uint8_t *>(host_in);
  uint8_t *in_d = static_cast<uint8_t *>(dev_in);
  // without a device result buffer the kernel writes the results straight
  // into the pinned host buffer (no D2H copy node), through the device
  // address the runtime reports for it; memory that is not mapped is refused
  void *res_ptr = dev_result;
  if (res_ptr == nullptr) {
    if (cudaHostGetDevicePointer(&res_ptr, host_result, 0) != cudaSuccess || res_ptr == nullptr ||
        !ffd::aligned16(res_ptr)) {
      cudaGetLastError();  // clear the sticky-free error of the query
      return FFD_ERR_INVALID_ARG;
    }
  }
  uint8_t *res_d = static_cast<uint8_t *>(res_ptr);
  const int group = s->num_q_heads / s->num_kv_heads;
  if (ffd::prepare_decode(s->block_size, group, format) != cudaSuccess) return FFD_ERR_CUDA;

  ffd_step_graph *g = new (std::nothrow) ffd_step_graph();
  if (g == nullptr) return FFD_ERR_CUDA;
  ffd_status st = FFD_OK;
  if (cudaStreamCreateWithFlags(&g->stream, cudaStreamNonBlocking) != cudaSuccess) {
    ffd::destroy_parts(g);
    delete g;
    return FFD_ERR_CUDA;
  }
  if (cudaStreamBeginCapture(g->stream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    ffd::destroy_parts(g);
    delete g;
    return FFD_ERR_CUDA;
  }
  const bool copy_ok = cudaMemcpyAsync(in_d, in_h, (nq + 2 * nk) * 2, cudaMemcpyHostToDevice, g->stream) ==
                       cudaSuccess;
  if (copy_ok && advance) ffd::advance_lengths_kernel<<<(s->batch + 127) / 128, 128, 0, g->stream>>>(d_lengths, s->batch);
  if (copy_ok) {
    const void *q = in_d;
    const void *k_new = in_d + nq * 2;
    const void *v_new = in_d + (nq + nk) * 2;
    uint32_t *mask = reinterpret_cast<uint32_t *>(res_d + mask_offset);
    st = format == 1
             ? ffd_decode_append_tr(s, reference, q, k_new, v_new, k_bf16, v_bf16, k_copy, k_resid, k_scales,
                                    d_lengths, delta, res_d, mask, workspace, workspace_bytes, g->stream)
             : ffd_decode_append(s, reference, q, k_new, v_new, k_bf16, v_bf16, k_copy, k_scales, d_lengths,
                                 delta, res_d, mask, workspace, workspace_bytes, g->stream);
  }
  const bool back_ok = copy_ok && st == FFD_OK &&
                       (dev_result == nullptr ||
                        cudaMemcpyAsync(host_result, res_d, result_bytes, cudaMemcpyDeviceToHost, g->stream) ==
                            cudaSuccess);
  const bool end_ok = cudaStreamEndCapture(g->stream, &g->graph) == cudaSuccess;
  if (!copy_ok || st != FFD_OK || !back_ok || !end_ok) {
    ffd::destroy_parts(g);
    delete g;
    return st != FFD_OK ? st : FFD_ERR_CUDA;
  }
  if (cudaGraphInstantiate(&g->exec, g->graph, 0) != cudaSuccess) {
    ffd::destroy_parts(g);
    delete g;
    return FFD_ERR_CUDA;
  }
  *graph_out = g;
  return FFD_OK;
}

ffd_status ffd_step_graph_run(ffd_step_graph *g) {
  if (g == nullptr || g->exec == nullptr) return FFD_ERR_INVALID_ARG;
  if (cudaGraphLaunch(g->exec, g->stream) != cudaSuccess) return FFD_ERR_CUDA;
  if (cudaStreamSynchronize(g->stream) != cudaSuccess) return FFD_ERR_CUDA;
  return FFD_OK;
}

void ffd_step_graph_destroy(ffd_step_graph *g) {
  if (g == nullptr) return;
  cudaStreamSynchronize(g->stream);
  ffd::destroy_parts(g);
  delete g;
}

}  // extern "C"
