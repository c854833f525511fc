// quantize.cu -- the low-bit key copies the selector scans.
//
// Two formats (Faster Than Flash, gist.science explainer, Methodology 1
// "Content-Aware Scanning via Low-Bit Quantization"): symmetric int4 codes in
// [-7, 7] with one bf16 scale per (block, channel), scanned beside a bf16 K
// cache; or the pages' own split of K into 2-bit thumbnails and 8-bit
// residuals (the computer then reconstructs K from the two).
//
// One CTA of 256 threads per (block j, kv-head g, sequence b) runs the block
// quantiser of ffd_quant.cuh; every load and store covers whole rows per
// warp.
#include "ffd_internal.h"
#include "ffd_quant.cuh"

namespace ffd {
namespace {

template <int T, int F>
__global__ void __launch_bounds__(256) quantize_kernel(const QuantizeParams p) {
  __shared__ float red[8 * kHeadDim];
  __shared__ float scale_s[kHeadDim];

  const int b = blockIdx.z, g = blockIdx.y;
  const int len = p.lengths[b];
  if (len < 0 || len > p.capacity) return;  // reported by the decode kernel
  const int nb = (len + T - 1) / T;
  const int j = p.block_begin < 0 ? nb - 1 : p.block_begin + static_cast<int>(blockIdx.x);
  if (j < 0 || j >= nb) return;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  const size_t tok0 = row * static_cast<size_t>(p.capacity) + static_cast<size_t>(j) * T;
  uint16_t *scale_row = p.scales + (row * static_cast<size_t>(p.capacity / T) + j) * kHeadDim;
  if constexpr (F == kFormatThumbResid) {
    quantize_block_tr<T, 256>(p.k + tok0 * kHeadDim, min(T, len - j * T), p.packed + tok0 * kThumbRowBytes,
                              p.resid + tok0 * kResidRowBytes, scale_row, red, scale_s,
                              static_cast<int>(threadIdx.x), 1);
  } else {
    quantize_block<T, 256>(p.k + tok0 * kHeadDim, min(T, len - j * T), p.packed + tok0 * kPackedRowBytes,
                           scale_row, red, scale_s, static_cast<int>(threadIdx.x), 1);
  }
}

template <int F>
void launch_f(const QuantizeParams &p, int block_size, dim3 grid, cudaStream_t stream) {
  if (block_size == 64) {
    quantize_kernel<64, F><<<grid, 256, 0, stream>>>(p);
  } else {
    quantize_kernel<128, F><<<grid, 256, 0, stream>>>(p);
  }
}

}  // namespace

cudaError_t launch_quantize(const QuantizeParams &p, int block_size, dim3 grid,
                            cudaStream_t stream) {
  if (p.format == kFormatThumbResid)
    launch_f<kFormatThumbResid>(p, block_size, grid, stream);
  else
    launch_f<kFormatInt4>(p, block_size, grid, stream);
  return cudaGetLastError();
}

}  // namespace ffd
