// ffd_quant.cuh -- quantisation of one key block to the int4 scan copy or to
// the thumbnail + residual format, shared by the quantize kernel and the fused
// decode step.
//
// The low-bit key "thumbnail" (Faster Than Flash, gist.science explainer,
// Methodology 1): symmetric int4 codes in [-7, 7] with one bf16 scale per
// (block, channel), scale = bf16_rne(amax / 7) by IEEE division, code =
// clamp(rint_even(k / scale), -7, 7), nibble = code + 8, byte i of a token row
// = channel 2i (low nibble) | channel 2i+1 (high nibble).  Tokens at or past
// the sequence length are excluded from amax and stored as code 0.  Every
// step is one correctly rounded IEEE operation, so the result is bit-exact.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ffd_internal.h"
#include "ffd_ptx.cuh"

namespace ffd {

__device__ __forceinline__ float q_bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float q_bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// NT threads (a multiple of 32, at least 32, tid in [0, NT)) quantise one
// block of T token rows.  Thread (rg = tid / 16, cg = tid % 16) owns channels
// 8cg .. 8cg+7 of rows rg, rg + NT/16, ...: one 16-byte load and one 4-byte
// store of 8 nibbles per row.  red holds NT/32 x 128 floats and scale_s 128
// floats of shared memory; `bar_id` names a barrier used by exactly these NT
// threads.  When last_row is not null it replaces the block's last valid row
// (the token being appended, not yet visible in k_rows to this CTA).
template <int T, int NT>
__device__ __forceinline__ void quantize_block(const uint16_t *k_rows, int valid, uint8_t *packed_rows,
                                               uint16_t *scale_row, float *red, float *scale_s, int tid,
                                               uint32_t bar_id, const uint16_t *last_row = nullptr) {
  static_assert(NT % 32 == 0 && NT >= 32 && T % (NT / 16) == 0, "thread layout");
  constexpr int RG = NT / 16;  // row groups
  constexpr int R = T / RG;    // rows per thread
  const int cg = tid & 15;
  const int rg = tid >> 4;
  uint4 x[R];
  float amax[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) amax[c] = 0.0f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = rg + RG * r;
    if (t < valid) {
      const uint16_t *src = (last_row != nullptr && t == valid - 1) ? last_row
                                                                     : k_rows + static_cast<size_t>(t) * kHeadDim;
      x[r] = *reinterpret_cast<const uint4 *>(src + 8 * cg);
      const uint32_t w[4] = {x[r].x, x[r].y, x[r].z, x[r].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        amax[2 * e] = fmaxf(amax[2 * e], fabsf(q_bf16_lo(w[e])));
        amax[2 * e + 1] = fmaxf(amax[2 * e + 1], fabsf(q_bf16_hi(w[e])));
      }
    } else {
      x[r] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // row groups rg and rg ^ 1 share a warp and differ in bit 4 of the lane id
#pragma unroll
  for (int c = 0; c < 8; ++c) amax[c] = fmaxf(amax[c], __shfl_xor_sync(0xFFFFFFFFu, amax[c], 16));
  const int warp = tid >> 5;
  if ((tid & 16) == 0) {
#pragma unroll
    for (int c = 0; c < 8; ++c) red[warp * kHeadDim + 8 * cg + c] = amax[c];
  }
  named_barrier(bar_id, NT);
  if (tid < kHeadDim) {
    float a = red[tid];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) a = fmaxf(a, red[w * kHeadDim + tid]);
    const __nv_bfloat16 s = __float2bfloat16_rn(__fdiv_rn(a, 7.0f));
    scale_row[tid] = __bfloat16_as_ushort(s);
    scale_s[tid] = __bfloat162float(s);
  }
  named_barrier(bar_id, NT);
  float sf[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) sf[c] = scale_s[8 * cg + c];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = rg + RG * r;
    const uint32_t w[4] = {x[r].x, x[r].y, x[r].z, x[r].w};
    uint32_t nibbles = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float v = (c & 1) ? q_bf16_hi(w[c >> 1]) : q_bf16_lo(w[c >> 1]);
      int code = 0;
      if (t < valid && sf[c] != 0.0f) {
        code = __float2int_rn(__fdiv_rn(v, sf[c]));
        code = min(7, max(-7, code));
      }
      nibbles |= static_cast<uint32_t>(code + 8) << (4 * c);
    }
    *reinterpret_cast<uint32_t *>(packed_rows + static_cast<size_t>(t) * kPackedRowBytes + 4 * cg) =
        nibbles;
  }
}

// The pages' own split of the K cache (Faster Than Flash, gist.science
// explainer, Methodology 1: 2-bit thumbnails for the scan, 8-bit residuals to
// reconstruct the keys).  Per (block, channel) s = bf16_rne(amax / 1.5); per
// element y = k / s, code u = clamp(floor(y) + 2, 0, 3) (level (u - 1.5) s),
// residual e = clamp(rint_even((y - (u - 1.5)) * 254), -127, 127) stored as
// e + 128; s == 0 gives u = 2, e = 0.  Thumbnail packing: channel 16w + i of
// a token row in 32-bit word w at bit 2 (i / 2) + 16 (i % 2).  Tokens at or
// past the length are zero bytes.  Every step is one IEEE operation, so the
// result is bit-exact.
//
// NT threads quantise one block of T rows.  Thread (rg = tid / 8, cg = tid % 8)
// owns channels 16cg .. 16cg+15 (thumbnail word cg, residual bytes 16cg ..) of
// rows rg, rg + NT/8, ...  Rows are loaded four at a time with all loads in
// flight together; up to four rows per thread stay in registers between the
// amax pass and the code pass, more are re-read (from L1/L2) four at a time.
// resid_rows may be null (a scan-only copy).  red holds NT/32 x 128 floats,
// scale_s 128 floats.  last_row as for quantize_block.
template <int T, int NT>
__device__ __forceinline__ void quantize_block_tr(const uint16_t *k_rows, int valid, uint8_t *thumb_rows,
                                                  uint8_t *resid_rows, uint16_t *scale_row, float *red,
                                                  float *scale_s, int tid, uint32_t bar_id,
                                                  const uint16_t *last_row = nullptr) {
  static_assert(NT % 32 == 0 && NT >= 32 && T % (NT / 8) == 0, "thread layout");
  constexpr int RG = NT / 8;  // row groups
  constexpr int R = T / RG;   // rows per thread
  constexpr int RC = R < 4 ? R : 4;  // rows per load round
  const int cg = tid & 7;
  const int rg = tid >> 3;
  uint4 x[RC][2];
  auto load_rows = [&](int r0) {
#pragma unroll
    for (int i = 0; i < RC; ++i) {
      const int t = rg + RG * (r0 + i);
      if (t < valid) {
        const uint16_t *row = (last_row != nullptr && t == valid - 1) ? last_row
                                                                       : k_rows + static_cast<size_t>(t) * kHeadDim;
        const uint4 *src = reinterpret_cast<const uint4 *>(row + 16 * cg);
        x[i][0] = src[0];
        x[i][1] = src[1];
      } else {
        x[i][0] = x[i][1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  float amax[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) amax[c] = 0.0f;
#pragma unroll
  for (int r0 = 0; r0 < R; r0 += RC) {
    load_rows(r0);
#pragma unroll
    for (int i = 0; i < RC; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t w[4] = {x[i][h].x, x[i][h].y, x[i][h].z, x[i][h].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          amax[8 * h + 2 * e] = fmaxf(amax[8 * h + 2 * e], fabsf(q_bf16_lo(w[e])));
          amax[8 * h + 2 * e + 1] = fmaxf(amax[8 * h + 2 * e + 1], fabsf(q_bf16_hi(w[e])));
        }
      }
    }
  }
  // the four row groups of a warp differ in lane bits 3 and 4
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    amax[c] = fmaxf(amax[c], __shfl_xor_sync(0xFFFFFFFFu, amax[c], 8));
    amax[c] = fmaxf(amax[c], __shfl_xor_sync(0xFFFFFFFFu, amax[c], 16));
  }
  const int warp = tid >> 5;
  if ((tid & 24) == 0) {
#pragma unroll
    for (int c = 0; c < 16; ++c) red[warp * kHeadDim + 16 * cg + c] = amax[c];
  }
  named_barrier(bar_id, NT);
  if (tid < kHeadDim) {
    float a = red[tid];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) a = fmaxf(a, red[w * kHeadDim + tid]);
    const __nv_bfloat16 s = __float2bfloat16_rn(__fdiv_rn(a, 1.5f));
    scale_row[tid] = __bfloat16_as_ushort(s);
    scale_s[tid] = __bfloat162float(s);
  }
  named_barrier(bar_id, NT);
  float sf[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) sf[c] = scale_s[16 * cg + c];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int i = r % RC;
    if (R > RC && i == 0) load_rows(r);
    const int t = rg + RG * r;
    uint32_t word = 0u;
    uint32_t rb[4] = {0u, 0u, 0u, 0u};
    if (t < valid) {
      const uint32_t w[8] = {x[i][0].x, x[i][0].y, x[i][0].z, x[i][0].w,
                             x[i][1].x, x[i][1].y, x[i][1].z, x[i][1].w};
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float v = (c & 1) ? q_bf16_hi(w[c >> 1]) : q_bf16_lo(w[c >> 1]);
        uint32_t u = 2u, eb = 128u;
        if (sf[c] != 0.0f) {
          const float y = __fdiv_rn(v, sf[c]);
          const float uf = fminf(fmaxf(__fadd_rn(floorf(y), 2.0f), 0.0f), 3.0f);
          const float d = __fsub_rn(y, __fsub_rn(uf, 1.5f));
          const float e = fminf(fmaxf(rintf(__fmul_rn(d, 254.0f)), -127.0f), 127.0f);
          u = static_cast<uint32_t>(uf);
          eb = static_cast<uint32_t>(static_cast<int>(e) + 128);
        }
        word |= u << (2 * (c >> 1) + 16 * (c & 1));
        rb[c >> 2] |= eb << (8 * (c & 3));
      }
    }
    *reinterpret_cast<uint32_t *>(thumb_rows + static_cast<size_t>(t) * kThumbRowBytes + 4 * cg) = word;
    if (resid_rows != nullptr)
      *reinterpret_cast<uint4 *>(resid_rows + static_cast<size_t>(t) * kResidRowBytes + 16 * cg) =
          make_uint4(rb[0], rb[1], rb[2], rb[3]);
  }
}

}  // namespace ffd
