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
// over the global capacity.  One CTA of 256 threads per (query head,
// kv-head, sequence): one round of loads for every split's (m, l), then eight
// thread groups share the partials' float4 loads.
#include <cuda_bf16.h>

#include "ffd_internal.h"
#include "ffd_ptx.cuh"

namespace ffd {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kGroups = kMergeThreads / 32;  // thread groups, each one float4 per lane of a head
constexpr uint32_t kFullMask = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// One CTA per (query head h of the group, kv-head g, sequence b).  Warps are
// thread groups: group q handles partials f = q, q + kGroups, ...; a lane holds
// four output channels.
template <int T, int G>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeParams p) {
  extern __shared__ float smem_f[];
  const int nflat = p.num_shards * p.nsplit_max;
  float *ms_s = smem_f;                   // [nflat] split maxima (base 2), -inf if absent
  float *ls_s = ms_s + nflat;             // [nflat] split sums
  float *stats = ls_s + nflat;            // [2]: M*, L*
  // [kGroups][32] float4, 16-byte aligned whatever nflat is
  float4 *red = reinterpret_cast<float4 *>(smem_f + ((2 * nflat + 4 + 3) & ~3));
  const float **part_s = reinterpret_cast<const float **>(red + kGroups * 32);  // [nflat]
  const int h = blockIdx.x % G, g = blockIdx.x / G, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_q_heads = p.num_kv_heads * G;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  uint16_t *out_row = p.out + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G + h) * kHeadDim;
  const int len = p.lengths[b];
  const int global_cap = p.capacity * p.num_shards;
  const int nblk_local = p.capacity / T;
  if (len <= 0 || len > global_cap) {  // empty (or invalid) sequence: zero row, empty mask
    for (int i = threadIdx.x; i < kHeadDim; i += kMergeThreads) out_row[i] = 0;
    if (h == 0)
      for (int w = threadIdx.x; w < p.mask_words; w += kMergeThreads) p.mask[row * p.mask_words + w] = 0u;
    return;
  }
  auto partial_ptr = [&](int f) {
    const int r = f / p.nsplit_max, s = f - r * p.nsplit_max;
    return reinterpret_cast<const float *>(p.gathered + r * p.region_bytes + p.partials_offset) +
           ((row * p.nsplit_max + s) * G + h) * kPartialStride;
  };
  // 1. every split's (m, l) in one round of independent loads; absent or
  //    empty splits get m = -inf
  for (int f = threadIdx.x; f < nflat; f += kMergeThreads) {
    const int r = f / p.nsplit_max, s = f - r * p.nsplit_max;
    const int lr = min(max(len - r * p.capacity, 0), p.capacity);
    const int nsr = ((lr + T - 1) / T + p.split_blocks - 1) / p.split_blocks;
    float m = -INFINITY, l = 0.0f;
    const float *ps = partial_ptr(f);
    if (s < nsr) {
      m = __ldcg(ps + 128);
      l = __ldcg(ps + 129);
    }
    ms_s[f] = m;
    ls_s[f] = l;
    part_s[f] = ps;
  }
  __syncthreads();
  // 2. M* = max m, L* = sum l 2^(m - M*) (warp 0, from shared memory)
  if (warp == 0) {
    float m = -INFINITY;
    for (int f = lane; f < nflat; f += 32) m = fmaxf(m, ms_s[f]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    float l = 0.0f;
    for (int f = lane; f < nflat; f += 32)
      if (ms_s[f] != -INFINITY) l += ls_s[f] * exp2f(ms_s[f] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFullMask, l, off);
    if (lane == 0) {
      stats[0] = m;
      stats[1] = l;
    }
  }
  __syncthreads();
  // 3. weights 2^(m - M*) / L* in place of the maxima
  for (int f = threadIdx.x; f < nflat; f += kMergeThreads)
    ms_s[f] = ms_s[f] == -INFINITY ? 0.0f : exp2f(ms_s[f] - stats[0]) / stats[1];
  __syncthreads();
  // 4. group `warp` accumulates partials f = warp, warp + kGroups, ... ; lane
  //    holds channels 4*lane .. 4*lane+3
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int f0 = warp; f0 < nflat; f0 += 8 * kGroups) {
    float4 v[8];
    float wv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = f0 + u * kGroups;
      wv[u] = f < nflat ? ms_s[f] : 0.0f;
      v[u] = wv[u] != 0.0f ? __ldcg(reinterpret_cast<const float4 *>(part_s[f]) + lane)
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
  red[warp * 32 + lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float4 o = red[lane];
#pragma unroll
    for (int q = 1; q < kGroups; ++q) {
      const float4 x = red[q * 32 + lane];
      o.x += x.x;
      o.y += x.y;
      o.z += x.z;
      o.w += x.w;
    }
    *reinterpret_cast<uint2 *>(out_row + 4 * lane) = make_uint2(pack2_bf16(o.x, o.y), pack2_bf16(o.z, o.w));
  }
  // 5. the mask row (head 0's CTA): global block j lives in shard j / nblk_local
  if (h != 0) return;
  const int nb = (len + T - 1) / T;
  // shards start at split boundaries, so the global split index j / S is
  // shard * nsplit_max + the shard's split index
  (void)nblk_local;
  auto load_word = [&](int gs, int wd) {
    const int r = gs / p.nsplit_max, s = gs - r * p.nsplit_max;
    const uint32_t *bits_r = reinterpret_cast<const uint32_t *>(p.gathered + r * p.region_bytes);
    return __ldcg(bits_r + (row * p.nsplit_max + s) * p.split_words + wd);
  };
  for (int w = threadIdx.x; w < p.mask_words; w += kMergeThreads)
    p.mask[row * p.mask_words + w] = gather_mask_word(w, nb, p.split_blocks, load_word);
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

size_t merge_smem_bytes(int num_shards, int nsplit_max) {
  const size_t nflat = static_cast<size_t>(num_shards) * nsplit_max;
  const size_t floats = (2 * nflat + 4 + 3) & ~static_cast<size_t>(3);
  return 4 * floats + 16 * kGroups * 32 + 8 * nflat;
}

cudaError_t launch_merge(const MergeParams &p, int block_size, int group, dim3 grid,
                         cudaStream_t stream) {
  const dim3 g(grid.x * group, grid.y);  // one CTA per query head
  const size_t smem = merge_smem_bytes(p.num_shards, p.nsplit_max);
  if (block_size == 64) return launch_t<64>(p, group, g, smem, stream);
  if (block_size == 128) return launch_t<128>(p, group, g, smem, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ffd
