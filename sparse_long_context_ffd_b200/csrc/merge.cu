// merge.cu -- log-sum-exp merge of split partials gathered from context
// shards (sequence parallelism across GPUs).
//
// Each GPU decodes a contiguous shard of every sequence's context (shards
// start at split boundaries, so the Top-delta selection of a split never
// looks across a shard) and writes its split partials (m, l, acc[128] per
// query head; m in base-2 logit units) and selection bits.  After the
// partials of all shards are gathered, this kernel merges them per
// (sequence, kv-head): M = max m, L = sum l 2^(m - M), o = sum acc 2^(m - M) / L
// -- the flash-decoding split merge, across GPUs -- and assembles the mask
// over the global capacity.  One CTA of 128 threads per (kv-head, sequence).
#include <cuda_bf16.h>

#include "ffd_internal.h"
#include "ffd_ptx.cuh"

namespace ffd {
namespace {

constexpr int kMergeThreads = 128;
constexpr uint32_t kFullMask = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

template <int T, int G>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeParams p) {
  extern __shared__ float smem_f[];
  float *stats = smem_f;    // [G][2]: M*, L*
  float *wts = smem_f + 16;  // [num_shards * nsplit_max][G]
  const int g = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_q_heads = p.num_kv_heads * G;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  uint16_t *out_rows = p.out + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G) * kHeadDim;
  const int len = p.lengths[b];
  const int global_cap = p.capacity * p.num_shards;
  const int nblk_local = p.capacity / T;
  if (len <= 0 || len > global_cap) {  // empty (or invalid) sequence: zero rows, empty mask
    for (int i = threadIdx.x; i < G * kHeadDim; i += kMergeThreads) out_rows[i] = 0;
    for (int w = threadIdx.x; w < p.mask_words; w += kMergeThreads) p.mask[row * p.mask_words + w] = 0u;
    return;
  }
  const int nflat = p.num_shards * p.nsplit_max;
  auto shard_splits = [&](int r) {
    const int lr = min(max(len - r * p.capacity, 0), p.capacity);
    const int nbr = (lr + T - 1) / T;
    return (nbr + p.split_blocks - 1) / p.split_blocks;
  };
  auto partial_ptr = [&](int f, int h) {
    const int r = f / p.nsplit_max, s = f - r * p.nsplit_max;
    return reinterpret_cast<const float *>(p.gathered + r * p.region_bytes + p.partials_offset) +
           ((row * p.nsplit_max + s) * G + h) * kPartialStride;
  };
  // 1. per head: pairwise (max, sum) combination over every valid split of every shard
  for (int h = warp; h < G; h += kMergeThreads / 32) {
    float m = -INFINITY, l = 0.0f;
    for (int f = lane; f < nflat; f += 32) {
      const int r = f / p.nsplit_max, s = f - r * p.nsplit_max;
      float ms = -INFINITY;
      if (s < shard_splits(r)) {
        const float *ps = partial_ptr(f, h);
        ms = __ldcg(ps + 128);
        const float ls = __ldcg(ps + 129);
        const float mn = fmaxf(m, ms);
        if (mn != -INFINITY) {
          l = (m == -INFINITY ? 0.0f : l * exp2f(m - mn)) + (ms == -INFINITY ? 0.0f : ls * exp2f(ms - mn));
          m = mn;
        }
      }
      wts[f * G + h] = ms;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float mo = __shfl_xor_sync(kFullMask, m, off), lo = __shfl_xor_sync(kFullMask, l, off);
      const float mn = fmaxf(m, mo);
      if (mn != -INFINITY) {
        l = (m == -INFINITY ? 0.0f : l * exp2f(m - mn)) + (mo == -INFINITY ? 0.0f : lo * exp2f(mo - mn));
        m = mn;
      }
    }
    if (lane == 0) {
      stats[2 * h] = m;
      stats[2 * h + 1] = l;
    }
  }
  __syncthreads();
  // 2. weights 2^(m - M*) / L*; splits that do not exist or kept nothing get 0
  for (int i = threadIdx.x; i < nflat * G; i += kMergeThreads) {
    const int h = i % G;
    const float ms = wts[i];
    wts[i] = ms == -INFINITY ? 0.0f : exp2f(ms - stats[2 * h]) / stats[2 * h + 1];
  }
  __syncthreads();
  // 3. each thread accumulates four output channels (float4) of one head
  for (int fi = threadIdx.x; fi < G * 32; fi += kMergeThreads) {
    const int h = fi >> 5, c4 = fi & 31;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int f0 = 0; f0 < nflat; f0 += 8) {
      float4 v[8];
      float wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int f = f0 + u;
        wv[u] = f < nflat ? wts[f * G + h] : 0.0f;
        v[u] = wv[u] != 0.0f ? __ldcg(reinterpret_cast<const float4 *>(partial_ptr(f, h)) + c4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc.x += wv[u] * v[u].x;
        acc.y += wv[u] * v[u].y;
        acc.z += wv[u] * v[u].z;
        acc.w += wv[u] * v[u].w;
      }
    }
    *reinterpret_cast<uint2 *>(out_rows + h * kHeadDim + 4 * c4) =
        make_uint2(pack2_bf16(acc.x, acc.y), pack2_bf16(acc.z, acc.w));
  }
  // 4. mask over the global capacity: global block j lives in shard j / nblk_local
  const int nb = (len + T - 1) / T;
  for (int w = threadIdx.x; w < p.mask_words; w += kMergeThreads) {
    uint32_t bits = 0, cached = 0;
    int key = -1;
    for (int k = 0; k < 32; ++k) {
      const int j = 32 * w + k;
      if (j >= nb) break;
      const int r = j / nblk_local, jl = j - r * nblk_local;
      const int s = jl / p.split_blocks, i = jl - s * p.split_blocks;
      const int kk = r * 65536 + s * p.split_words + (i >> 5);  // cache key
      if (kk != key) {
        const uint32_t *bits_r = reinterpret_cast<const uint32_t *>(p.gathered + r * p.region_bytes);
        cached = __ldcg(bits_r + (row * p.nsplit_max + s) * p.split_words + (i >> 5));
        key = kk;
      }
      bits |= ((cached >> (i & 31)) & 1u) << k;
    }
    p.mask[row * p.mask_words + w] = bits;
  }
}

template <int T>
cudaError_t launch_t(const MergeParams &p, int group, dim3 grid, size_t smem, cudaStream_t stream) {
  switch (group) {
    case 1: merge_kernel<T, 1><<<grid, kMergeThreads, smem, stream>>>(p); break;
    case 2: merge_kernel<T, 2><<<grid, kMergeThreads, smem, stream>>>(p); break;
    case 4: merge_kernel<T, 4><<<grid, kMergeThreads, smem, stream>>>(p); break;
    case 8: merge_kernel<T, 8><<<grid, kMergeThreads, smem, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const MergeParams &p, int block_size, int group, dim3 grid,
                         cudaStream_t stream) {
  const size_t smem = 4 * (16 + static_cast<size_t>(p.num_shards) * p.nsplit_max * group);
  if (block_size == 64) return launch_t<64>(p, group, grid, smem, stream);
  if (block_size == 128) return launch_t<128>(p, group, grid, smem, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ffd
