// quantize.cu -- int4 key copy with per-block-per-channel bf16 scales.
//
// The low-bit key "thumbnail" that the selector scans (Faster Than Flash,
// gist.science explainer, Methodology 1 "Content-Aware Scanning via Low-Bit
// Quantization"); the pages use 2-bit thumbnails, this path uses symmetric
// int4 codes in [-7, 7] with one bf16 scale per (block, channel).
//
// One CTA of 256 threads per (block j, kv-head g, batch b).  Thread
// (rg = tid / 16, cg = tid % 16) owns channels 8cg..8cg+7 of token rows
// rg, rg+16, ...: one 16-byte load per row (a warp reads two whole 256-byte
// rows), one 4-byte store of 8 nibbles per row (a warp writes two whole
// 64-byte packed rows).  Every arithmetic step is a single correctly rounded
// IEEE operation, so codes and scales are bit-identical to a scalar CPU
// implementation of the same steps.
#include <cuda_bf16.h>

#include "ffd_internal.h"

namespace ffd {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int T>
__global__ void __launch_bounds__(256) quantize_kernel(const QuantizeParams p) {
  __shared__ float red[8][kHeadDim];
  __shared__ float scale_s[kHeadDim];

  const int b = blockIdx.z, g = blockIdx.y;
  const int len = p.lengths[b];
  if (len < 0 || len > p.capacity) return;  // reported by the decode kernel
  const int nb = (len + T - 1) / T;
  const int j = p.block_begin < 0 ? nb - 1 : p.block_begin + static_cast<int>(blockIdx.x);
  if (j < 0 || j >= nb) return;
  const int valid = min(T, len - j * T);

  const int tid = threadIdx.x;
  const int cg = tid & 15;
  const int rg = tid >> 4;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  const size_t tok0 = row * static_cast<size_t>(p.capacity) + static_cast<size_t>(j) * T;

  constexpr int R = T / 16;
  uint4 x[R];
  float amax[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) amax[c] = 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = rg + 16 * r;
    if (t < valid) {
      x[r] = *reinterpret_cast<const uint4 *>(p.k + (tok0 + t) * kHeadDim + 8 * cg);
      const uint32_t w[4] = {x[r].x, x[r].y, x[r].z, x[r].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        amax[2 * e] = fmaxf(amax[2 * e], fabsf(bf16_lo(w[e])));
        amax[2 * e + 1] = fmaxf(amax[2 * e + 1], fabsf(bf16_hi(w[e])));
      }
    } else {
      x[r] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // rows rg and rg+1 of a warp differ in bit 4 of the lane id
#pragma unroll
  for (int c = 0; c < 8; ++c) amax[c] = fmaxf(amax[c], __shfl_xor_sync(0xFFFFFFFFu, amax[c], 16));
  const int warp = tid >> 5;
  if ((tid & 16) == 0) {
#pragma unroll
    for (int c = 0; c < 8; ++c) red[warp][8 * cg + c] = amax[c];
  }
  __syncthreads();
  if (tid < kHeadDim) {
    float a = red[0][tid];
#pragma unroll
    for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w][tid]);
    const __nv_bfloat16 s = __float2bfloat16_rn(__fdiv_rn(a, 7.0f));
    p.scales[(row * static_cast<size_t>(p.capacity / T) + j) * kHeadDim + tid] =
        __bfloat16_as_ushort(s);
    scale_s[tid] = __bfloat162float(s);
  }
  __syncthreads();

  float sf[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) sf[c] = scale_s[8 * cg + c];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = rg + 16 * r;
    const uint32_t w[4] = {x[r].x, x[r].y, x[r].z, x[r].w};
    uint32_t nibbles = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float v = (c & 1) ? bf16_hi(w[c >> 1]) : bf16_lo(w[c >> 1]);
      int code = 0;
      if (t < valid && sf[c] != 0.0f) {
        code = __float2int_rn(__fdiv_rn(v, sf[c]));
        code = min(7, max(-7, code));
      }
      nibbles |= static_cast<uint32_t>(code + 8) << (4 * c);
    }
    *reinterpret_cast<uint32_t *>(p.packed + (tok0 + t) * kPackedRowBytes + 4 * cg) = nibbles;
  }
}

}  // namespace

cudaError_t launch_quantize(const QuantizeParams &p, int block_size, dim3 grid,
                            cudaStream_t stream) {
  if (block_size == 64) {
    quantize_kernel<64><<<grid, 256, 0, stream>>>(p);
  } else {
    quantize_kernel<128><<<grid, 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace ffd
