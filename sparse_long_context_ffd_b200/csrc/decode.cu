// decode.cu -- the fused FFD decode kernel: selector + computer + split merge
// in one launch.
//
// Method (Faster Than Flash, gist.science explainer, Methodology 3 "Fused
// Kernel and System Optimization"): a selector streams the low-bit keys,
// computes tentative block scores and filters blocks against a threshold; the
// computer fetches full-precision K/V only for the kept blocks and computes
// exact attention.  The threshold is delta below a running maximum inside a
// fixed split of blocks (Methodology 2, Mechanism), so splits never wait for
// one another; splits are merged with log-sum-exp (flash-decoding split-K).
//
// One CTA per work unit (split s, kv-head g, sequence b), 4 consumer warps +
// 1 producer warp:
//   phase 1 (selector, skipped when dense): the producer streams the split's
//     packed-key tiles and scales with 1-D bulk copies into a ring of shared
//     memory stages; each consumer warp folds the query group into int8 for
//     one block, runs the integer dot products on the tensor cores
//     (mma m16n8k32, u8 nibbles x s8 query) and keeps the block maximum.
//   phase 2: warp 0 turns the block scores into keep bits with a warp-wide
//     prefix maximum per head and the union over the group (no HBM traffic:
//     the scan's decision stays on chip).
//   phase 3 (computer): the producer fetches the kept blocks' K and V in
//     64-token stages with 2-D TMA copies (128-byte swizzle); each consumer
//     warp owns 16 tokens of every stage, runs q.K^T and P.V on the tensor
//     cores (mma m16n8k16 bf16, the query group as the M dimension) with an
//     online softmax in base 2.
//   phase 4: the warps' partial softmax states are merged in shared memory
//     and written as the split partial; the last CTA to finish for (b, g)
//     merges all splits, writes the bf16 output rows and the mask row.
#include <cuda_bf16.h>

#include <atomic>
#include <climits>

#include "ffd.h"
#include "ffd_internal.h"
#include "ffd_ptx.cuh"

namespace ffd {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr float kRsqrtD = 0.08838834764831845f;     // nearest float to 1/sqrt(128)
constexpr float kScaleLog2 = 0.12751743074195287f;  // log2(e) / sqrt(128)

template <int T>
struct ScanGeom {
  static constexpr int kStageBytes = T * kPackedRowBytes + kScaleRowBytes;
  static constexpr int kStages = kRingBytes / kStageBytes;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ int clamp127(int x) { return min(127, max(-127, x)); }

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat162 v) {
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ void raise_timeout(const DecodeParams &p, volatile int *flags) {
  flags[1] = 1;
  atomicOr(p.err, kFlagTimeout);
}

// Wait for the most recent fill of each ring stage (bounded), so that no
// bulk copy is still writing this CTA's shared memory when it exits.
__device__ __forceinline__ void drain_ring(uint64_t *full, int stages, int issued) {
  for (int u = issued > stages ? issued - stages : 0; u < issued; ++u)
    mbar_wait(&full[u % stages], static_cast<uint32_t>(u / stages) & 1u, kWaitLimitNs);
}

// Selector for one block: fold the group's query with the block's channel
// scales into int8, integer-score every token on the tensor cores, and
// write score_j for each head of the group.
//
// Lane (gid = lane / 4, t4 = lane % 4) folds head gid over channels
// 32*t4 .. 32*t4 + 31, which are exactly the channels its mma B fragments
// hold: k-step s takes packed word s of the lane's 16-byte chunk of a token
// row, whose low nibbles are channels 32*t4 + 8s + {0,2,4,6} and high
// nibbles channels 32*t4 + 8s + {1,3,5,7}.
template <int T, int G>
__device__ __forceinline__ void scan_block(const uint8_t *tile, const uint16_t *scl,
                                           const uint32_t (&qreg)[16], int valid_rows, int lane,
                                           float *score_out) {
  const int gid = lane >> 2, t4 = lane & 3;
  float pc[32];
  float a = 0.0f;
  const uint4 *s4 = reinterpret_cast<const uint4 *>(scl) + 4 * t4;
#pragma unroll
  for (int w4 = 0; w4 < 4; ++w4) {
    const uint4 sv = s4[w4];
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k = 8 * w4 + 2 * e;
      const uint32_t qw = qreg[k >> 1];
      pc[k] = __fmul_rn(bf16_lo(qw), bf16_lo(sw[e]));
      pc[k + 1] = __fmul_rn(bf16_hi(qw), bf16_hi(sw[e]));
      a = fmaxf(a, fmaxf(fabsf(pc[k]), fabsf(pc[k + 1])));
    }
  }
  a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
  a = fmaxf(a, __shfl_xor_sync(kFull, a, 2));

  uint32_t bq[4][2];
  int sumq = 0;
  float cf = 0.0f;
  if (gid < G && a > 0.0f) {
    const float inv = __fdiv_rn(127.0f, a);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = clamp127(__float2int_rn(__fmul_rn(pc[8 * s + 2 * e], inv)));
        const int qh = clamp127(__float2int_rn(__fmul_rn(pc[8 * s + 2 * e + 1], inv)));
        sumq += ql + qh;
        lo |= (static_cast<uint32_t>(ql) & 0xFFu) << (8 * e);
        hi |= (static_cast<uint32_t>(qh) & 0xFFu) << (8 * e);
      }
      bq[s][0] = lo;
      bq[s][1] = hi;
    }
    cf = __fmul_rn(__fdiv_rn(a, 127.0f), kRsqrtD);
  } else {
#pragma unroll
    for (int s = 0; s < 4; ++s) bq[s][0] = bq[s][1] = 0u;
  }
  sumq += __shfl_xor_sync(kFull, sumq, 1);
  sumq += __shfl_xor_sync(kFull, sumq, 2);

  // sum_c qi_c * (u_c - 8) = sum_c qi_c * u_c - 8 * sum_c qi_c, and the
  // correction commutes with the max over tokens.
  int best0 = INT_MIN, best1 = INT_MIN;  // heads 2*t4, 2*t4 + 1
#pragma unroll
  for (int mt = 0; mt < T / 16; ++mt) {
    const int r0 = 16 * mt + gid, r1 = r0 + 8;
    const uint4 u0 = *reinterpret_cast<const uint4 *>(tile + r0 * kPackedRowBytes + 16 * t4);
    const uint4 u1 = *reinterpret_cast<const uint4 *>(tile + r1 * kPackedRowBytes + 16 * t4);
    const uint32_t w0[4] = {u0.x, u0.y, u0.z, u0.w};
    const uint32_t w1[4] = {u1.x, u1.y, u1.z, u1.w};
    int acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      mma_u8s8_16x8x32(acc, w0[s] & 0x0F0F0F0Fu, w1[s] & 0x0F0F0F0Fu, (w0[s] >> 4) & 0x0F0F0F0Fu,
                       (w1[s] >> 4) & 0x0F0F0F0Fu, bq[s][0], bq[s][1]);
    }
    if (r0 < valid_rows) {
      best0 = max(best0, acc[0]);
      best1 = max(best1, acc[1]);
    }
    if (r1 < valid_rows) {
      best0 = max(best0, acc[2]);
      best1 = max(best1, acc[3]);
    }
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    best0 = max(best0, __shfl_xor_sync(kFull, best0, off));
    best1 = max(best1, __shfl_xor_sync(kFull, best1, off));
  }
  const int h0 = 2 * t4, h1 = 2 * t4 + 1;
  const int sq0 = __shfl_sync(kFull, sumq, h0 << 2);
  const int sq1 = __shfl_sync(kFull, sumq, h1 << 2);
  const float c0 = __shfl_sync(kFull, cf, h0 << 2);
  const float c1 = __shfl_sync(kFull, cf, h1 << 2);
  if (gid == 0) {
    if (h0 < G) score_out[h0] = __fmul_rn(__int2float_rn(best0 - 8 * sq0), c0);
    if (h1 < G) score_out[h1] = __fmul_rn(__int2float_rn(best1 - 8 * sq1), c1);
  }
}

// Byte address of 16-byte chunk `cc` (0..15) of row `r` in a K or V stage
// tile: two 64-channel halves of 64 rows x 128 bytes, 128-byte swizzled.
__device__ __forceinline__ uint32_t kv_chunk_addr(uint32_t base, int r, int cc) {
  return base + static_cast<uint32_t>((cc >> 3) * 8192 + r * 128 + (((cc & 7) ^ (r & 7)) << 4));
}

template <int T, int G>
__global__ void __launch_bounds__(kDecodeThreads, 2)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int NS1 = ScanGeom<T>::kStages;
  constexpr int kScanStage = ScanGeom<T>::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *full1 = reinterpret_cast<uint64_t *>(smem + kRingBytes);
  uint64_t *empty1 = full1 + NS1;
  uint64_t *full3 = empty1 + NS1;
  uint64_t *empty3 = full3 + kKvStages;
  volatile int *flags = reinterpret_cast<volatile int *>(empty3 + kKvStages);  // is_last, abort
  uint32_t *keepbits = reinterpret_cast<uint32_t *>(empty3 + kKvStages) + 4;
  float *scores = reinterpret_cast<float *>(keepbits + ((p.split_words + 3) & ~3));

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_q_heads = p.num_kv_heads * G;
  const int len = p.lengths[b];
  const bool bad = len < 0 || len > p.capacity;
  const int nb = bad ? 0 : (len + T - 1) / T;
  const int nsplit = (nb + p.split_blocks - 1) / p.split_blocks;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  uint16_t *out_rows = p.out + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G) * kHeadDim;

  if (split >= nsplit) {
    // Empty or invalid sequence: split 0 writes zero rows and an empty mask.
    if (split == 0) {
      if (bad && threadIdx.x == 0 && g == 0) atomicOr(p.err, kFlagBadLength);
      for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) out_rows[i] = 0;
      for (int w = threadIdx.x; w < p.mask_words; w += blockDim.x) p.mask[row * p.mask_words + w] = 0u;
    }
    return;
  }
  const int j0 = split * p.split_blocks;
  const int nbs = min(p.split_blocks, nb - j0);
  const bool dense = p.dense != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS1; ++s) {
      mbar_init(&full1[s], 1);
      mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&full3[s], 1);
      mbar_init(&empty3[s], kConsumerWarps);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  __syncthreads();

  // ---------------------------------------------------------- phase 1: scan
  if (!dense) {
    if (warp == kConsumerWarps) {
      if (lane == 0) {
        const uint8_t *src_p =
            p.packed + (row * p.capacity + static_cast<size_t>(j0) * T) * kPackedRowBytes;
        const uint16_t *src_s =
            p.scales + (row * static_cast<size_t>(p.capacity / T) + j0) * kHeadDim;
        int i = 0;
        for (; i < nbs; ++i) {
          const int st = i % NS1;
          const uint32_t use = static_cast<uint32_t>(i / NS1);
          if (use > 0 && !mbar_wait(&empty1[st], (use - 1) & 1u, kWaitLimitNs)) {
            raise_timeout(p, flags);
            break;
          }
          uint8_t *dst = ring + st * kScanStage;
          mbar_arrive_expect_tx(&full1[st], kScanStage);
          bulk_g2s(dst, src_p + static_cast<size_t>(i) * T * kPackedRowBytes, T * kPackedRowBytes,
                   &full1[st]);
          bulk_g2s(dst + T * kPackedRowBytes, src_s + static_cast<size_t>(i) * kHeadDim,
                   kScaleRowBytes, &full1[st]);
          if (flags[1]) {
            ++i;
            break;
          }
        }
        drain_ring(full1, NS1, i);
      }
    } else {
      const int gid = lane >> 2, t4 = lane & 3;
      uint32_t qreg[16];
      if (gid < G) {
        const uint4 *qsrc = reinterpret_cast<const uint4 *>(
            p.q + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G + gid) * kHeadDim +
            32 * t4);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 x = qsrc[v];
          qreg[4 * v] = x.x;
          qreg[4 * v + 1] = x.y;
          qreg[4 * v + 2] = x.z;
          qreg[4 * v + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int v = 0; v < 16; ++v) qreg[v] = 0u;
      }
      for (int i = warp; i < nbs; i += kConsumerWarps) {
        const int st = i % NS1;
        const uint32_t use = static_cast<uint32_t>(i / NS1);
        if (!mbar_wait(&full1[st], use & 1u, kWaitLimitNs)) {
          raise_timeout(p, flags);
          break;
        }
        const uint8_t *tile = ring + st * kScanStage;
        scan_block<T, G>(tile, reinterpret_cast<const uint16_t *>(tile + T * kPackedRowBytes), qreg,
                         min(T, len - (j0 + i) * T), lane, scores + i * G);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty1[st]);
        if (flags[1]) break;
      }
    }
  }
  fence_proxy_async_smem();  // generic reads of the ring before TMA reuses it
  __syncthreads();

  // ------------------------------------------- phase 2: Top-delta keep bits
  if (warp == 0) {
    float carry[G];
#pragma unroll
    for (int h = 0; h < G; ++h) carry[h] = -INFINITY;
    for (int base = 0; base < nbs; base += 32) {
      const int i = base + lane;
      const bool valid = i < nbs;
      bool keep = dense && valid;
      if (!dense) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float s = valid ? scores[i * G + h] : -INFINITY;
          float m = s;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(kFull, m, off);
            if (lane >= off) m = fmaxf(m, o);
          }
          m = fmaxf(m, carry[h]);
          carry[h] = __shfl_sync(kFull, m, 31);
          keep = keep || (valid && s >= __fsub_rn(m, p.delta));
        }
      }
      const uint32_t bits = __ballot_sync(kFull, keep);
      if (lane == 0) keepbits[base >> 5] = bits;
    }
  }
  __syncthreads();

  // ------------------------------------------- phase 3: attention (computer)
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      int it = 0;
      bool ok = flags[1] == 0;
      for (int w = 0; ok && w < p.split_words; ++w) {
        uint32_t bits = keepbits[w];
        while (ok && bits) {
          const int i = 32 * w + __ffs(bits) - 1;
          bits &= bits - 1;
#pragma unroll 1
          for (int u = 0; u < T / kSubTokens; ++u) {
            const int tok = (j0 + i) * T + u * kSubTokens;
            if (tok >= len) break;
            const int st = it % kKvStages;
            const uint32_t use = static_cast<uint32_t>(it / kKvStages);
            if (use > 0 && !mbar_wait(&empty3[st], (use - 1) & 1u, kWaitLimitNs)) {
              raise_timeout(p, flags);
              ok = false;
              break;
            }
            uint8_t *dst = ring + st * kKvStageBytes;
            mbar_arrive_expect_tx(&full3[st], kKvStageBytes);
            const int y = static_cast<int>(row * p.capacity) + tok;
            tma_load_2d(dst, &tmap_k, 0, y, &full3[st]);
            tma_load_2d(dst + 8192, &tmap_k, 64, y, &full3[st]);
            tma_load_2d(dst + 16384, &tmap_v, 0, y, &full3[st]);
            tma_load_2d(dst + 24576, &tmap_v, 64, y, &full3[st]);
            ++it;
          }
        }
      }
      drain_ring(full3, kKvStages, it);
    }
    return;
  }

  const int gid = lane >> 2, t4 = lane & 3;
  uint32_t qa[8][2];
  {
    const uint32_t *qh = reinterpret_cast<const uint32_t *>(
        p.q + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G + (gid < G ? gid : 0)) *
                  kHeadDim);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      qa[s][0] = gid < G ? qh[8 * s + t4] : 0u;      // channels 16s + 2*t4, +1
      qa[s][1] = gid < G ? qh[8 * s + 4 + t4] : 0u;  // channels 16s + 8 + 2*t4, +1
    }
  }
  float m_run = -INFINITY, l_run = 0.0f;
  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  const uint32_t ring_addr = smem_addr(ring);
  int it = 0;
  bool ok = flags[1] == 0;
  for (int w = 0; ok && w < p.split_words; ++w) {
    uint32_t bits = keepbits[w];
    while (ok && bits) {
      const int i = 32 * w + __ffs(bits) - 1;
      bits &= bits - 1;
#pragma unroll 1
      for (int u = 0; u < T / kSubTokens; ++u) {
        const int tok = (j0 + i) * T + u * kSubTokens;
        if (tok >= len) break;
        const int st = it % kKvStages;
        const uint32_t use = static_cast<uint32_t>(it / kKvStages);
        if (!mbar_wait(&full3[st], use & 1u, kWaitLimitNs)) {
          raise_timeout(p, flags);
          ok = false;
          break;
        }
        const uint32_t kbase = ring_addr + st * kKvStageBytes;
        const uint32_t vbase = kbase + 16384;

        // S = Q K^T over this warp's 16 tokens (two n-tiles of 8)
        float sacc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            uint32_t kb[4];
            ldmatrix_x4(kb, kv_chunk_addr(kbase, 16 * warp + 8 * nt + (lane & 7), 4 * kk + (lane >> 3)));
            mma_bf16_16x8x16(sacc[nt], qa[2 * kk][0], 0u, qa[2 * kk][1], 0u, kb[0], kb[1]);
            mma_bf16_16x8x16(sacc[nt], qa[2 * kk + 1][0], 0u, qa[2 * kk + 1][1], 0u, kb[2], kb[3]);
          }
        }
        // online softmax in base 2; tokens past the length are masked out
        const int tw = tok + 16 * warp;
        float x[2][2];
        float mt = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int t = tw + 8 * nt + 2 * t4 + e;
            x[nt][e] = t < len ? sacc[nt][e] * kScaleLog2 : -INFINITY;
            mt = fmaxf(mt, x[nt][e]);
          }
        }
        mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 2));
        const float m_new = fmaxf(m_run, mt);
        float corr = 1.0f;
        float pv[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
        if (m_new != -INFINITY) {
          corr = exp2f(m_run - m_new);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) pv[nt][e] = exp2f(x[nt][e] - m_new);
        }
        // P is rounded to bf16 once; the same weights feed P.V and the sum
        const __nv_bfloat162 p01 = __floats2bfloat162_rn(pv[0][0], pv[0][1]);
        const __nv_bfloat162 p23 = __floats2bfloat162_rn(pv[1][0], pv[1][1]);
        const float2 f01 = __bfloat1622float2(p01);
        const float2 f23 = __bfloat1622float2(p23);
        l_run = l_run * corr + ((f01.x + f01.y) + (f23.x + f23.y));
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          acc[n][0] *= corr;
          acc[n][1] *= corr;
        }
        const uint32_t pa0 = pack_bf16x2(p01), pa2 = pack_bf16x2(p23);
#pragma unroll
        for (int cc2 = 0; cc2 < 8; ++cc2) {
          const int mi = lane >> 3;
          uint32_t vb[4];
          ldmatrix_x4_trans(vb, kv_chunk_addr(vbase, 16 * warp + (lane & 7) + 8 * (mi & 1), 2 * cc2 + (mi >> 1)));
          mma_bf16_16x8x16(acc[2 * cc2], pa0, 0u, pa2, 0u, vb[0], vb[1]);
          mma_bf16_16x8x16(acc[2 * cc2 + 1], pa0, 0u, pa2, 0u, vb[2], vb[3]);
        }
        m_run = m_new;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty3[st]);
        ++it;
      }
    }
  }
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);

  // ------------------------------ phase 4: split partial and the final merge
  const uint32_t nthreads = kConsumerWarps * 32;
  named_barrier(1, nthreads);  // every stage consumed: the ring becomes scratch
  float *wm = reinterpret_cast<float *>(ring);  // [warp][8]
  float *wl = wm + kConsumerWarps * 8;          // [warp][8]
  float *wacc = wl + kConsumerWarps * 8;        // [warp][8][128]
  if (gid < G) {
    if (t4 == 0) {
      wm[warp * 8 + gid] = m_run;
      wl[warp * 8 + gid] = l_run;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      wacc[(warp * 8 + gid) * kHeadDim + 8 * n + 2 * t4] = acc[n][0];
      wacc[(warp * 8 + gid) * kHeadDim + 8 * n + 2 * t4 + 1] = acc[n][1];
    }
  }
  named_barrier(1, nthreads);
  const size_t unit = row * p.nsplit_max + split;
  float *part = p.partials + unit * G * kPartialStride;
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += nthreads) {
    const int h = idx >> 7, c = idx & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, wm[w * 8 + h]);
    float L = 0.0f, A = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = wm[w * 8 + h];
      if (mw != -INFINITY) {
        const float f = exp2f(mw - M);
        L += wl[w * 8 + h] * f;
        A += wacc[(w * 8 + h) * kHeadDim + c] * f;
      }
    }
    part[h * kPartialStride + c] = A;
    if (c == 0) {
      part[h * kPartialStride + 128] = M;
      part[h * kPartialStride + 129] = L;
    }
  }
  if (static_cast<int>(threadIdx.x) < p.split_words)
    p.split_bits[unit * p.split_words + threadIdx.x] = keepbits[threadIdx.x];
  __threadfence();
  named_barrier(1, nthreads);
  if (threadIdx.x == 0)
    flags[0] = atomicAdd(&p.counters[row], 1u) == static_cast<unsigned>(nsplit - 1) ? 1 : 0;
  named_barrier(1, nthreads);
  if (!flags[0]) return;
  __threadfence();

  // last CTA of (b, g): log-sum-exp merge over the splits
  const float *row_parts = p.partials + row * p.nsplit_max * G * kPartialStride;
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += nthreads) {
    const int h = idx >> 7, c = idx & 127;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(row_parts + (s * G + h) * kPartialStride + 128));
    float L = 0.0f, A = 0.0f;
    for (int s = 0; s < nsplit; ++s) {
      const float *ps = row_parts + (s * G + h) * kPartialStride;
      const float f = exp2f(__ldcg(ps + 128) - M);
      L += __ldcg(ps + 129) * f;
      A += __ldcg(ps + c) * f;
    }
    out_rows[h * kHeadDim + c] = __bfloat16_as_ushort(__float2bfloat16_rn(A / L));
  }
  const uint32_t *row_bits = p.split_bits + row * p.nsplit_max * p.split_words;
  for (int w = threadIdx.x; w < p.mask_words; w += nthreads) {
    uint32_t bits = 0;
    for (int k = 0; k < 32; ++k) {
      const int j = 32 * w + k;
      if (j < nb) {
        const int s = j / p.split_blocks, i = j - s * p.split_blocks;
        bits |= ((__ldcg(row_bits + s * p.split_words + (i >> 5)) >> (i & 31)) & 1u) << k;
      }
    }
    p.mask[row * p.mask_words + w] = bits;
  }
  if (threadIdx.x == 0) p.counters[row] = 0u;
}

template <int T, int G>
cudaError_t launch_tg(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, dim3 grid,
                      size_t smem, cudaStream_t stream) {
  auto kern = decode_kernel<T, G>;
  // Raise the dynamic shared memory cap once per device, to the largest
  // split this build accepts, so later launches (and graph captures) need
  // no attribute call.
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit == 0 || (configured.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(decode_smem_bytes(T, G, FFD_MAX_SPLIT_BLOCKS)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  kern<<<grid, kDecodeThreads, smem, stream>>>(p, tk, tv);
  return cudaGetLastError();
}

template <int T>
cudaError_t launch_t(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int group,
                     dim3 grid, size_t smem, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_tg<T, 1>(p, tk, tv, grid, smem, stream);
    case 2: return launch_tg<T, 2>(p, tk, tv, grid, smem, stream);
    case 4: return launch_tg<T, 4>(p, tk, tv, grid, smem, stream);
    case 8: return launch_tg<T, 8>(p, tk, tv, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t decode_smem_bytes(int block_size, int group, int split_blocks) {
  const int stage = block_size * kPackedRowBytes + kScaleRowBytes;
  const int ns1 = kRingBytes / stage;
  const int split_words = (split_blocks + 31) / 32;
  return 1024 + kRingBytes + 8 * (2 * ns1 + 2 * kKvStages) + 16 +
         4 * static_cast<size_t>((split_words + 3) & ~3) +
         4 * static_cast<size_t>(split_blocks) * group;
}

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                          int block_size, int group, dim3 grid, size_t smem_bytes, cudaStream_t stream) {
  if (block_size == 64) return launch_t<64>(p, tmap_k, tmap_v, group, grid, smem_bytes, stream);
  if (block_size == 128) return launch_t<128>(p, tmap_k, tmap_v, group, grid, smem_bytes, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ffd
