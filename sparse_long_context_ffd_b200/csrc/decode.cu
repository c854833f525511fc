// decode.cu -- the fused FFD decode kernel: selector + computer + split merge
// in one launch.
//
// Method (Faster Than Flash, gist.science explainer, Methodology 3 "Fused
// Kernel and System Optimization"): a selector streams the low-bit keys,
// computes tentative block scores and filters blocks against a threshold; the
// computer fetches full-precision K/V only for the kept blocks and computes
// exact attention, reusing the scan's decision without a memory round trip
// (arXiv abstract).  The threshold is delta below a running maximum inside a
// fixed split of blocks (Methodology 2, Mechanism), so splits never wait for
// one another; splits are merged with log-sum-exp (flash-decoding split-K).
//
// One CTA per work unit (split s, kv-head g, sequence b); three warp roles
// run concurrently as a pipeline:
//   producer warp (one lane): an event loop that streams the split's packed
//     key tiles and scales into the scan ring with 1-D bulk copies and, as
//     kept blocks appear in the selection queue, their K and V into the
//     attention ring with one 3-D TMA copy each (128-byte swizzle);
//   scan warp: folds the query group into int8 for each block, scores all
//     tokens on the tensor cores (mma m16n8k32, u8 nibbles x s8 query), keeps
//     the per-head running maximum in registers, applies the Top-delta test,
//     takes the union over the group and appends kept blocks to the queue --
//     the decision never leaves shared memory;
//   attention warps: each takes whole K/V stages round-robin and runs
//     S^T = K Q^T (tokens as the mma M dimension), an online softmax in base 2
//     and O^T += V^T P^T on the tensor cores (mma m16n8k16 bf16).
// At the end the attention warps merge their softmax states, write the split
// partial, and the last CTA to finish for (b, g) merges all splits and writes
// the bf16 output rows and the mask row.  No CTA ever waits for another.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <atomic>
#include <climits>

#include "ffd.h"
#include "ffd_internal.h"
#include "ffd_ptx.cuh"
#include "ffd_quant.cuh"

namespace ffd {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;

// Debug build (FFD_DEBUG): every global index the kernel computes is checked
// against the extent the shape implies; a violation sets kFlagBounds in the
// sticky word and the access is skipped (a skipped copy leaves its barrier
// short, so the waits end at their limit).  Without FFD_DEBUG the checks
// compile away.
#ifdef FFD_DEBUG
#define FFD_IN_BOUNDS(params, cond) ((cond) || (atomicOr((params).err, kFlagBounds), false))
#else
#define FFD_IN_BOUNDS(params, cond) true
#endif
constexpr float kRsqrtD = 0.08838834764831845f;     // nearest float to 1/sqrt(128)
constexpr float kFltMax = 3.4028234663852886e38f;
constexpr float kScaleLog2 = 0.12751743074195287f;  // log2(e) / sqrt(128)

// Pipeline geometry.
constexpr int kAttnWarps = 4;
constexpr int kScanWarp = kAttnWarps;
constexpr int kProducerWarp = kAttnWarps + 1;
constexpr int kThreads = (kAttnWarps + 2) * 32;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kKvTok = kKvBoxRows;                  // tokens per attention stage
constexpr int kKvHalfBytes = kKvTok * 128;          // one 64-channel half of K or V
constexpr int kMergeBytes = kAttnWarps * (8 + 8 + 8 * kHeadDim) * 4;
// block quantiser scratch for the attention warps: per-warp channel maxima + scales
constexpr int kRequantScratchBytes = (kAttnWarps + 1) * kHeadDim * 4;
// Scored scan entries waiting for the in-order Top-delta decision: entry e
// uses slot e % kScanSlots, so at most kScanSlots entries are claimed ahead of
// the decision frontier.
constexpr int kScanSlots = 16;
// Thumbnail format: longest split (tokens) whose sparse steps load the
// attention stages' thumbnail rows and scale rows from L2 (KvGeom).
constexpr int kTrL2MaxSplitTokens = 4096;

// One attention stage (kKvTok tokens of one kept block) per key format and
// variant (C: the sparse-step variant, below).
template <int F, bool C>
struct KvGeom;
template <bool C>
struct KvGeom<kFormatInt4, C> {  // K lo, K hi, V lo, V hi (bf16, 128-byte swizzle): 16 KiB
  static constexpr int kVOffset = 2 * kKvHalfBytes;
  static constexpr int kTx = 4 * kKvHalfBytes;
  static constexpr int kStageBytes = kTx;
  static constexpr int kStages = 5;
};
template <>
struct KvGeom<kFormatThumbResid, false> {
  // residual rows (128 B, 128-byte swizzle) | V lo | V hi | thumbnail rows | scale row
  static constexpr int kVOffset = kKvTok * kResidRowBytes;
  static constexpr int kThumbOffset = kVOffset + 2 * kKvHalfBytes;
  static constexpr int kScaleOffset = kThumbOffset + kKvTok * kThumbRowBytes;
  static constexpr int kTx = kScaleOffset + kScaleRowBytes;
  static constexpr int kStageBytes = (kTx + 1023) / 1024 * 1024;  // swizzled tiles stay 1 KiB aligned
  static constexpr int kStages = 6;
};
template <>
struct KvGeom<kFormatThumbResid, true> {
  // residual rows | V lo | V hi: 12 KiB.  The stage's thumbnail rows and scale
  // row (1.25 KiB) stay out of it: in a sparse step with short splits the scan
  // read them shortly before, so the attention warp loads them from L2 into
  // registers while the stage is in flight.  No small copies per stage, and
  // one stage more in the same shared memory.
  static constexpr int kVOffset = kKvTok * kResidRowBytes;
  static constexpr int kTx = kVOffset + 2 * kKvHalfBytes;
  static constexpr int kStageBytes = kTx;
  static constexpr int kStages = 7;
};

// With the cooperative selector (C) the ring has as many stages as fit beside
// the K/V ring with two CTAs per SM, since several warps hold stages at once;
// with the scan warp alone, fewer.
template <int T, int F, bool C>
struct ScanGeom {
  static constexpr int kRowBytes = F == kFormatThumbResid ? kThumbRowBytes : kPackedRowBytes;
  static constexpr int kStageBytes = T * kRowBytes + kScaleRowBytes;
  static constexpr int kStages = C ? (F == kFormatThumbResid ? (T == 64 ? 9 : 5) : (T == 64 ? 6 : 3))
                                   : (F == kFormatThumbResid ? 2 : 1) * (T == 64 ? 4 : 2);
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(kRingBytes >= kMergeBytes, "merge scratch aliases the scan ring");
};

template <int T, int F, bool C>
struct SmemLayout {
  static constexpr int NKV = KvGeom<F, C>::kStages;
  static constexpr int kKvRing = 0;
  static constexpr int kScanRing = NKV * KvGeom<F, C>::kStageBytes;
  static constexpr int kBars = kScanRing + ScanGeom<T, F, C>::kRingBytes;
  static constexpr int kNumBars = 2 * ScanGeom<T, F, C>::kStages + 2 * NKV;
  static constexpr int kMeta = kBars + 8 * kNumBars;  // int [NKV] token offsets
  static constexpr int kSeq = kMeta + 4 * NKV;        // int [NKV] item indices
  // qcount, sel_done, is_last, abort, requant_done, scan claim, scan decided,
  // attention warps help the scan
  static constexpr int kCtrl = (kSeq + 4 * NKV + 15) / 16 * 16;
  static constexpr int kScanSeq = kCtrl + 32;                // int [NSA] scan entry per stage
  static constexpr int kSlotSeq = kScanSeq + 4 * kScanSlots;  // int [kScanSlots] entry per slot
  static constexpr int kScores = kSlotSeq + 4 * kScanSlots;   // float [kScanSlots][8]
  static constexpr int kQRows = kScores + 32 * kScanSlots;    // bf16 [8][128]: the query group
  static constexpr int kRequant = kQRows + 8 * kHeadDim * 2;  // re-quantisation scratch (attention warps)
  static constexpr int kKeep = kRequant + kRequantScratchBytes;  // u32 [split_words]
  // queue of kept block indices (u16 [split_blocks]) follows keep bits
  static_assert(ScanGeom<T, F, C>::kStages <= kScanSlots, "one sequence word per scan stage");
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ int clamp127(int x) { return min(127, max(-127, x)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Reconstructed key codes z = 254 u - 381 + e of two channels as an f16 pair.
// `w_shifted` holds the two 2-bit codes at bits 0 and 16; `resid_word` the two
// residual bytes (e + 128) at byte positions picked by `sel` (0x4140: bytes 0
// and 1, 0x4342: bytes 2 and 3).  The byte permute puts 0x64 above each byte,
// so a lane reads as the f16 1024 + (e + 128) + 254 u = z + 1533 exactly (all
// below 2048); one f16x2 subtraction of 1533 (0x65FD) leaves z exactly.
__device__ __forceinline__ uint32_t key_pair(uint32_t w_shifted, uint32_t resid_word, uint32_t sel) {
  const uint32_t u = w_shifted & 0x00030003u;
  const uint32_t e = __byte_perm(resid_word, 0x64646464u, sel);
  return sub_f16x2(u * 254u + e, 0x65FD65FDu);
}

__device__ __forceinline__ void raise_timeout(const DecodeParams &p, volatile int *ctrl) {
  ctrl[3] = 1;
  atomicOr(p.err, kFlagTimeout);
}

// Spin (bounded) until the producer has published item `it` in a stage.
__device__ __forceinline__ bool wait_item_published(volatile int *seq, int st, int it, uint64_t limit_ns) {
  if (seq[st] == it) return true;
  const uint64_t t0 = global_timer_ns();
  while (seq[st] != it) {
    if (global_timer_ns() - t0 > limit_ns) return false;
    __nanosleep(20);
  }
  return true;
}

// Wait for the most recent fill of each ring stage (bounded), so that no
// copy is still writing this CTA's shared memory when it exits.
__device__ __forceinline__ void drain_ring(uint64_t *full, int stages, int issued) {
  for (int u = issued > stages ? issued - stages : 0; u < issued; ++u)
    mbar_wait(&full[u % stages], static_cast<uint32_t>(u / stages) & 1u, kWaitLimitNs);
}

// Block index of scan entry e: with nref reference entries first (the sink
// block 0, then the local block nb - 1), then the split's blocks from j0.
__device__ __forceinline__ int scan_block_index(int e, int nref, int nb, int j0) {
  return e < nref ? (e == 0 ? 0 : nb - 1) : j0 + (e - nref);
}

// Query fold of the selector (the per-block int8 query: p_c = q_c s_c,
// a = max |p_c|, qi_c = rint(p_c 127 / a)), spread over the warp.  Lane
// (gid, t4) folds head gid % G over part r = gid / G of the 32 channels
// 32*t4 .. 32*t4 + 31 that its mma B fragments cover, R parts per head so
// that every lane group works when G < 8; the int8 words are then gathered
// into the B fragments of lanes gid < G (lanes gid >= G feed output columns
// of heads that do not exist, so their fragments are left as they fall).
//
// B word positions pos = 0..7 (the order of the fragment registers):
//   int4 format   pos = 2s + x: k-step s, x = 0 for the low nibbles
//                 (channels 8s + {0,2,4,6}), 1 for the high ones (+1);
//   thumbnail     pos = 4h + k: k-step k, word group h, bytes channels
//                 16h + {2k, 8+2k, 2k+1, 9+2k}.
// Part r owns positions r*NW .. r*NW + NW - 1.  Its channels are
// base(r) + off(ci), ci = 0..NC-1 (the lane's compact order), and byte j of
// its word w is compact index idx(w, j).
template <int G, int F>
struct ScanFold {
  static constexpr bool kTR = F == kFormatThumbResid;
  static constexpr int R = G >= 8 ? 1 : (G == 4 ? 2 : 4);
  static constexpr int NC = 32 / R;  // channels folded per lane
  static constexpr int NW = NC / 4;  // int8 B words per lane
  // the thumbnail format with 4 parts takes channels base + {0..3, 8..11}
  static constexpr bool kSplitRuns = kTR && R == 4;
  __device__ static int part(int gid) { return (gid / G) & (R - 1); }
  __device__ static int base(int r) { return kSplitRuns ? 16 * (r >> 1) + 4 * (r & 1) : r * NC; }
  static constexpr int off(int ci) { return kSplitRuns && ci >= 4 ? ci + 4 : ci; }
  static constexpr int idx(int w, int j) {
    if (!kTR) return 8 * (w >> 1) + 2 * j + (w & 1);
    if (kSplitRuns) return j == 0 ? 2 * w : j == 1 ? 4 + 2 * w : j == 2 ? 2 * w + 1 : 5 + 2 * w;
    const int k = w & 3, h16 = 16 * (w >> 2);
    return h16 + (j == 0 ? 2 * k : j == 1 ? 8 + 2 * k : j == 2 ? 2 * k + 1 : 9 + 2 * k);
  }
  // the lane's NC bf16 values of a channel row (query or scales) as pairs
  template <typename Src>
  __device__ static void load_pairs(const Src *row_t4, int r, uint32_t (&v)[NC / 2]) {
    const uint16_t *src = reinterpret_cast<const uint16_t *>(row_t4) + base(r);
    if constexpr (kSplitRuns) {
      const uint2 x = *reinterpret_cast<const uint2 *>(src);
      const uint2 y = *reinterpret_cast<const uint2 *>(src + 8);
      v[0] = x.x;
      v[1] = x.y;
      v[2] = y.x;
      v[3] = y.y;
    } else {
#pragma unroll
      for (int m = 0; m < NC / 8; ++m) {
        const uint4 x = reinterpret_cast<const uint4 *>(src)[m];
        v[4 * m] = x.x;
        v[4 * m + 1] = x.y;
        v[4 * m + 2] = x.z;
        v[4 * m + 3] = x.w;
      }
    }
  }
};

// Low byte of four words packed into one (bytes 0..3 from a, b, c, d).
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

// Fold one block's scales into the int8 query (see ScanFold).  qv: the lane's
// query channels in compact order, as bf16 pairs.  Returns the B fragments in bq
// (lanes gid < G), the head's sum of qi in sumq and a in a_out (every lane of
// the head; a == 0 gives qi = 0).
//
// Rounding: with the fp32 product x = p * (127 / a), |x| <= 127 (1 + 2^-24)^2
// < 127.5, so the fp32 sum x + 1.5 * 2^23 is 1.5 * 2^23 + rint(x) exactly
// (round to nearest even, as rint), its low byte is qi as int8 and the clamp
// to +-127 never acts.  When 127 / a overflows (a below about 3.7e-37), or a
// itself is infinite, the conversion is done the direct way instead.
template <int G, int F>
__device__ __forceinline__ void fold_block_sv(const uint32_t (&sv)[ScanFold<G, F>::NC / 2],
                                              const uint32_t (&qv)[ScanFold<G, F>::NC / 2], int lane,
                                              uint32_t (&bq)[8], int &sumq, float &a_out) {
  using SF = ScanFold<G, F>;
  constexpr int NC = SF::NC, NW = SF::NW, R = SF::R;
  // p_c is recomputed where it is used (an exact product) rather than kept
  auto pc = [&](int c) {
    return (c & 1) ? __fmul_rn(bf16_hi(qv[c >> 1]), bf16_hi(sv[c >> 1])) : __fmul_rn(bf16_lo(qv[c >> 1]), bf16_lo(sv[c >> 1]));
  };
  float am0 = 0.0f, am1 = 0.0f;
#pragma unroll
  for (int c = 0; c < NC; c += 2) {
    am0 = fmaxf(am0, fabsf(pc(c)));
    am1 = fmaxf(am1, fabsf(pc(c + 1)));
  }
  float a = fmaxf(am0, am1);
  a = fmaxf(a, __shfl_xor_sync(kFull, a, 1));
  a = fmaxf(a, __shfl_xor_sync(kFull, a, 2));
#pragma unroll
  for (int m = 1; m < R; m <<= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, 4 * G * m));
  uint32_t words[NW];
  int sq = 0;
  if (a > 0.0f) {
    const float inv = __fdiv_rn(127.0f, a);
    if (a <= kFltMax && inv <= kFltMax) {
      uint32_t acc = 0u;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        uint32_t y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          y[j] = __float_as_uint(__fadd_rn(__fmul_rn(pc(SF::idx(w, j)), inv), 12582912.0f));
          acc += y[j];
        }
        words[w] = low_bytes4(y[0], y[1], y[2], y[3]);
      }
      sq = static_cast<int>(acc - static_cast<uint32_t>(NC) * 0x4B400000u);
    } else {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        uint32_t y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = clamp127(__float2int_rn(__fmul_rn(pc(SF::idx(w, j)), inv)));
          sq += v;
          y[j] = static_cast<uint32_t>(v);
        }
        words[w] = low_bytes4(y[0], y[1], y[2], y[3]);
      }
    }
  } else {
#pragma unroll
    for (int w = 0; w < NW; ++w) words[w] = 0u;
  }
  sq += __shfl_xor_sync(kFull, sq, 1);
  sq += __shfl_xor_sync(kFull, sq, 2);
#pragma unroll
  for (int m = 1; m < R; m <<= 1) sq += __shfl_xor_sync(kFull, sq, 4 * G * m);
  // gather: position pos comes from part pos / NW, NW words on
#pragma unroll
  for (int pos = 0; pos < 8; ++pos) {
    if (pos < NW)
      bq[pos] = words[pos];
    else
      bq[pos] = __shfl_sync(kFull, words[pos % NW], (lane + 4 * G * (pos / NW)) & 31);
  }
  sumq = sq;
  a_out = a;
}

// fold_block_sv with the lane's scale pairs read from a block's scale row.
template <int G, int F>
__device__ __forceinline__ void fold_block(const uint16_t *scl, const uint32_t (&qv)[ScanFold<G, F>::NC / 2],
                                           int lane, uint32_t (&bq)[8], int &sumq, float &a_out) {
  using SF = ScanFold<G, F>;
  uint32_t sv[SF::NC / 2];
  SF::load_pairs(scl + 32 * (lane & 3), SF::part(lane >> 2), sv);
  fold_block_sv<G, F>(sv, qv, lane, bq, sumq, a_out);
}

// Selector, tensor-core part: the integer score sum_c qi_c u_c of every token
// of a block, maxed over the valid tokens, for heads 2*t4 and 2*t4 + 1 of the
// lane's output columns (reduced over the warp at the end).
//
// int4 format: k-step s takes packed word s of the lane's 16-byte chunk of a
// token row (channels 32*t4 + 8s .. +7), whose low nibbles are channels
// 8s + {0,2,4,6} and high nibbles 8s + {1,3,5,7}: B positions 2s and 2s + 1.
// Thumbnail format: the lane reads thumbnail words 2*t4 + h (h = 0, 1) of its
// token rows; (w >> 2k) & 0x03030303 puts channels 16h + {2k, 8+2k, 2k+1,
// 9+2k} (relative to 32*t4) in bytes 0..3, so k-step k takes a0 from word
// 2*t4 and a2 from word 2*t4 + 1, with B positions k and 4 + k.
template <int T, int F>
__device__ __forceinline__ void block_best(const uint8_t *tile, const uint32_t (&bq)[8], int valid_rows,
                                           int lane, int &best0, int &best1) {
  const int gid = lane >> 2, t4 = lane & 3;
  best0 = INT_MIN;
  best1 = INT_MIN;
#pragma unroll
  for (int mt = 0; mt < T / 16; ++mt) {
    const int r0 = 16 * mt + gid, r1 = r0 + 8;
    int acc[4] = {0, 0, 0, 0};
    if constexpr (F == kFormatThumbResid) {
      const uint2 u0 = *reinterpret_cast<const uint2 *>(tile + r0 * kThumbRowBytes + 8 * t4);
      const uint2 u1 = *reinterpret_cast<const uint2 *>(tile + r1 * kThumbRowBytes + 8 * t4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        mma_u8s8_16x8x32(acc, (u0.x >> (2 * k)) & 0x03030303u, (u1.x >> (2 * k)) & 0x03030303u,
                         (u0.y >> (2 * k)) & 0x03030303u, (u1.y >> (2 * k)) & 0x03030303u, bq[k], bq[4 + k]);
      }
    } else {
      const uint4 u0 = *reinterpret_cast<const uint4 *>(tile + r0 * kPackedRowBytes + 16 * t4);
      const uint4 u1 = *reinterpret_cast<const uint4 *>(tile + r1 * kPackedRowBytes + 16 * t4);
      const uint32_t w0[4] = {u0.x, u0.y, u0.z, u0.w};
      const uint32_t w1[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        mma_u8s8_16x8x32(acc, w0[s] & 0x0F0F0F0Fu, w1[s] & 0x0F0F0F0Fu, (w0[s] >> 4) & 0x0F0F0F0Fu,
                         (w1[s] >> 4) & 0x0F0F0F0Fu, bq[2 * s], bq[2 * s + 1]);
      }
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
}

// Selector, last part: the block scores of heads 2*t4 and 2*t4 + 1 from the
// per-lane maxima, the head's sum of qi and a (every lane).
//   int4 format:  I = sum_c qi_c (u_c - 8) = sum qi u - 8 sum qi (the
//                 correction commutes with the max over tokens), score =
//                 float(max_t I_t) * (a / 127) / sqrt(D);
//   thumbnails:   the level of code u is (2u - 3) s / 2, so I = 2 sum qi u -
//                 3 sum qi and score = float(max_t I_t) * (a / 254) / sqrt(D).
template <int F>
__device__ __forceinline__ void block_scores(int best0, int best1, int sumq, float a, int lane, float &score0,
                                             float &score1) {
  constexpr bool kTR = F == kFormatThumbResid;
  const int t4 = lane & 3;
  const float cf = a > 0.0f ? __fmul_rn(__fdiv_rn(a, kTR ? 254.0f : 127.0f), kRsqrtD) : 0.0f;
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
  if constexpr (kTR) {
    score0 = __fmul_rn(__int2float_rn(2 * best0 - 3 * sq0), c0);
    score1 = __fmul_rn(__int2float_rn(2 * best1 - 3 * sq1), c1);
  } else {
    score0 = __fmul_rn(__int2float_rn(best0 - 8 * sq0), c0);
    score1 = __fmul_rn(__int2float_rn(best1 - 8 * sq1), c1);
  }
}

// ------------------------------------------------------------------------
// Cooperative selector.  Scoring a block (fold + integer scan + block score)
// is independent from block to block; only the Top-delta decision runs in
// block order (the running maximum).  So the scan warp and, while they wait
// for K/V, the attention warps all score scan entries: a warp claims the next
// entry (ctrl[5], in order), scores it from its ring stage, releases the
// stage and leaves the head scores in slot e % kScanSlots with e written
// last into the slot's sequence word.  The scan warp alone decides, entry by
// entry in order, from the slots (ctrl[6] counts the decided entries and
// frees their slots).  Max is taken in the same order as a single scanning
// warp would, so the selection is bit-identical to it.

struct ScanShared {
  volatile int *ctrl;       // [5] next entry to claim, [6] entries decided
  volatile int *scan_seq;   // [stage]: entry whose tile the producer put there
  volatile int *slot_seq;   // [slot]: entry whose scores the slot holds
  float *scores;            // [slot][8 heads]
  const uint16_t *q_rows;   // [G][128]: the query group
};

// Lane 0 claims the next scan entry; the whole warp gets the result: the
// entry, -1 once every entry is claimed, -2 if none can be taken now (the
// slot window is full, or -- when `landed_only` -- its tile has not landed).
template <int NSA>
__device__ __forceinline__ int claim_scan_entry(const ScanShared &sh, uint64_t *full_a, int total, bool landed_only,
                                                int lane) {
  int e = -2;
  if (lane == 0) {
    const int c = sh.ctrl[5];
    if (c >= total) {
      e = -1;
    } else if (c < sh.ctrl[6] + kScanSlots) {
      const int st = c % NSA;
      const bool ready = !landed_only ||
                         (sh.scan_seq[st] == c && mbar_test_wait(&full_a[st], static_cast<uint32_t>(c / NSA) & 1u));
      if (ready && atomicCAS(const_cast<int *>(&sh.ctrl[5]), c, c + 1) == c) e = c;
    }
  }
  return __shfl_sync(kFull, e, 0);
}

// Score scan entry e (block jb, valid_rows tokens): wait for its tile (the
// producer's sequence word, then the stage's fill, both bounded), fold the
// query with the block's scales, scan, release the stage.  s0, s1: the
// scores of heads 2 t4 and 2 t4 + 1 (every lane).  False if a wait ran out.
template <int T, int G, int F, bool C>
__device__ __forceinline__ bool score_scan_entry(const ScanShared &sh, uint8_t *scan_ring, uint64_t *full_a,
                                                 uint64_t *empty_a, int e, int valid_rows, int lane,
                                                 uint64_t limit_ns, float &s0, float &s1) {
  using SG = ScanGeom<T, F, C>;
  using SF = ScanFold<G, F>;
  constexpr int NSA = SG::kStages;
  const int st = e % NSA;
  if (!wait_item_published(sh.scan_seq, st, e, limit_ns) ||
      !mbar_wait(&full_a[st], static_cast<uint32_t>(e / NSA) & 1u, limit_ns))
    return false;
  const int gid = lane >> 2, t4 = lane & 3;
  const uint8_t *tile = scan_ring + st * SG::kStageBytes;
  uint32_t qv[SF::NC / 2];
  SF::load_pairs(sh.q_rows + (gid % G) * kHeadDim + 32 * t4, SF::part(gid), qv);
  uint32_t bq[8];
  int sq, best0, best1;
  float am;
  fold_block<G, F>(reinterpret_cast<const uint16_t *>(tile + T * SG::kRowBytes), qv, lane, bq, sq, am);
  block_best<T, F>(tile, bq, valid_rows, lane, best0, best1);
  __syncwarp();
  if (lane == 0) mbar_arrive(&empty_a[st]);
  block_scores<F>(best0, best1, sq, am, lane, s0, s1);
  return true;
}

// Leave scan entry e's head scores in its slot, e written last into the
// slot's sequence word (for the scan warp's in-order decision).
__device__ __forceinline__ void publish_scan_scores(const ScanShared &sh, int e, float s0, float s1, int lane) {
  float *slot = sh.scores + (e % kScanSlots) * 8;
  if (lane < 4) {  // lane t4 holds heads 2 t4 and 2 t4 + 1
    slot[2 * lane] = s0;
    slot[2 * lane + 1] = s1;
  }
  __syncwarp();
  if (lane == 0) {
    __threadfence_block();
    sh.slot_seq[e % kScanSlots] = e;
  }
}

// The attention warps' call: kept out of line, so that the registers it needs
// do not raise the attention loop's own allocation (the live registers of the
// caller are saved around the call, which happens only while it waits).
template <int T, int G, int F>
__device__ __noinline__ bool score_scan_entry_helper(const ScanShared &sh, uint8_t *scan_ring, uint64_t *full_a,
                                                     uint64_t *empty_a, int e, int valid_rows, int lane,
                                                     uint64_t limit_ns) {
  float s0, s1;
  if (!score_scan_entry<T, G, F, true>(sh, scan_ring, full_a, empty_a, e, valid_rows, lane, limit_ns, s0, s1))
    return false;
  publish_scan_scores(sh, e, s0, s1, lane);
  return true;
}

// Thumbnail format: keys are rebuilt from thumbnail + residual as k_hat =
// s z / 254 with the integer z = 254 u - 381 + e (exact in f16).  The block's
// scales go into the query instead: q'_c = f16(q_c s_c 2^E / 254), E per head
// so that max |q'| is about 2^13 (no f16 overflow or underflow), and the scores
// are scaled back by 2^-E in fp32.  qb: the lane's query pairs (channels
// 32*t4 + 2i, +1 of head gid, i = 2ks + j at qb[ks][j]); scale4(w4): the lane's
// scales of channels 32*t4 + 8*w4 .. +7.  Returns q' as f16 pairs in qh and
// the logit scales of heads 2*t4, 2*t4 + 1 (every lane).
template <typename ScaleFn>
__device__ __forceinline__ void fold_query_tr(const uint32_t (&qb)[8][2], int t4, ScaleFn scale4, uint32_t (&qh)[16],
                                              float &sc0, float &sc1) {
  float fq[32];
  float am = 0.0f;
#pragma unroll
  for (int w4 = 0; w4 < 4; ++w4) {
    const uint4 sv = scale4(w4);
    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = 4 * w4 + e;  // channel pair 32*t4 + 2i
      const uint32_t qw = qb[i >> 1][i & 1];
      fq[2 * i] = __fmul_rn(bf16_lo(qw), bf16_lo(sw[e]));
      fq[2 * i + 1] = __fmul_rn(bf16_hi(qw), bf16_hi(sw[e]));
      am = fmaxf(am, fmaxf(fabsf(fq[2 * i]), fabsf(fq[2 * i + 1])));
    }
  }
  am = fmaxf(am, __shfl_xor_sync(kFull, am, 1));
  am = fmaxf(am, __shfl_xor_sync(kFull, am, 2));
  const int ea = static_cast<int>((__float_as_uint(am) >> 23) & 0xFFu);
  const int E = min(148 - ea, 126);  // am 2^E in [2^21, 2^22)
  const float mult = ea == 0 ? 0.0f : __uint_as_float(static_cast<uint32_t>(127 + E) << 23) * (1.0f / 254.0f);
  const float uns = ea == 0 ? 0.0f : __uint_as_float(static_cast<uint32_t>(127 - E) << 23) * kScaleLog2;
#pragma unroll
  for (int i = 0; i < 16; ++i) qh[i] = pack_f16x2(fq[2 * i] * mult, fq[2 * i + 1] * mult);
  sc0 = __shfl_sync(kFull, uns, (2 * t4) << 2);
  sc1 = __shfl_sync(kFull, uns, (2 * t4 + 1) << 2);
}

// C: the sparse-step variant for 64-token blocks: the cooperative selector
// (the attention warps score scan entries while they wait for K/V); without it
// (dense mode, 128-token blocks) the scan warp scores every entry itself.  In
// the thumbnail format (splits of at most 4096 tokens) the variant's attention
// stages also leave out the thumbnail rows and scale rows, which the attention
// warps load from L2 (KvGeom).
template <int T, int G, int F, bool C>
__global__ void __launch_bounds__(kThreads, 2)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
  using SG = ScanGeom<T, F, C>;
  using SL = SmemLayout<T, F, C>;
  using KG = KvGeom<F, C>;
  constexpr bool kTR = F == kFormatThumbResid;
  constexpr bool kCoop = C;          // the cooperative selector
  constexpr bool kTrL2 = C && kTR;   // thumbnails and scales from L2
  constexpr int NSA = SG::kStages;
  constexpr int NKV = KG::kStages;
  constexpr int kSubPerBlock = T / kKvTok;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *kv_ring = smem + SL::kKvRing;
  uint8_t *scan_ring = smem + SL::kScanRing;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SL::kBars);
  uint64_t *full_a = bars;
  uint64_t *empty_a = full_a + NSA;
  uint64_t *full_b = empty_a + NSA;
  uint64_t *empty_b = full_b + NKV;
  volatile int *meta = reinterpret_cast<volatile int *>(smem + SL::kMeta);
  volatile int *seq = reinterpret_cast<volatile int *>(smem + SL::kSeq);
  // qcount, sel_done, is_last, abort, requant_done
  volatile int *ctrl = reinterpret_cast<volatile int *>(smem + SL::kCtrl);
  uint32_t *keepbits = reinterpret_cast<uint32_t *>(smem + SL::kKeep);
  const ScanShared sh{ctrl, reinterpret_cast<volatile int *>(smem + SL::kScanSeq),
                      reinterpret_cast<volatile int *>(smem + SL::kSlotSeq),
                      reinterpret_cast<float *>(smem + SL::kScores),
                      reinterpret_cast<const uint16_t *>(smem + SL::kQRows)};
  volatile uint16_t *queue =
      reinterpret_cast<volatile uint16_t *>(keepbits + ((p.split_words + 3) & ~3));

  // R = p.parts CTAs per split when the splits alone leave SMs idle: every
  // one of them scans the whole split (so all take the same decisions, with
  // no exchange) and attends over its share of the kept blocks (kept-list
  // positions = part mod R); each writes its own partial.
  const int R = p.parts;
  const int split = blockIdx.x / R, part = blockIdx.x % R, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_q_heads = p.num_kv_heads * G;
  const int len = p.lengths[b];
  const bool bad = len < 0 || len > p.capacity;
  const int nb = bad ? 0 : (len + T - 1) / T;
  const int nsplit = (nb + p.split_blocks - 1) / p.split_blocks;
  const size_t row = static_cast<size_t>(b) * p.num_kv_heads + g;
  uint16_t *out_rows =
      p.out + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G) * kHeadDim;

  if (split >= nsplit) {
    // Empty or invalid sequence: split 0 writes zero rows and an empty mask.
    if (split == 0 && part == 0) {
      if (bad && threadIdx.x == 0 && g == 0) atomicOr(p.err, kFlagBadLength);
      if (!p.partials_only &&
          FFD_IN_BOUNDS(p, row < static_cast<size_t>(p.batch) * p.num_kv_heads)) {  // (a shard leaves them to the merge)
        for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) out_rows[i] = 0;
        for (int w = threadIdx.x; w < p.mask_words; w += blockDim.x) p.mask[row * p.mask_words + w] = 0u;
      }
    }
    return;
  }
  const int j0 = split * p.split_blocks;
  const int nbs = min(p.split_blocks, nb - j0);
  const bool dense = p.dense != 0;
  // pseudo-max reference: the scan first scores the sink block (0) and the
  // local block (nb - 1), then the split's own blocks
  const bool pseudo = p.reference != 0 && !dense;
  const int nref = pseudo ? (nb > 1 ? 2 : 1) : 0;
  // in the fused step the last block is being re-quantised by the CTA that
  // owns it; every other CTA builds that block's int4 tile itself from K
  const bool local_in_smem = pseudo && p.requant_last && nb > 1 && split != nsplit - 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSA; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&empty_a[s], 1);
    }
    for (int s = 0; s < NKV; ++s) {
      mbar_init(&full_b[s], 1);
      mbar_init(&empty_b[s], 1);
      seq[s] = -1;
    }
    for (int c = 0; c < 8; ++c) ctrl[c] = 0;
    for (int s = 0; s < NSA; ++s) sh.scan_seq[s] = -1;
    for (int s = 0; s < kScanSlots; ++s) sh.slot_seq[s] = -1;
    fence_mbar_init();
  }
  for (int w = threadIdx.x; w < p.split_words; w += blockDim.x) keepbits[w] = 0u;
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  // Fused decode step: the CTA that owns a sequence's last block re-quantises
  // it (the appended token changed it).  The attention warps do it while the
  // producer and the scan already stream the split's other blocks; only the
  // copies that read the rewritten block wait for the requant_done flag.
  const bool owner_requant = p.requant_last && split == nsplit - 1;
  __syncthreads();

  // ================================================================ producer
  if (warp == kProducerWarp) {
    if (lane != 0) return;
    const uint8_t *src_p = p.packed + row * p.capacity * SG::kRowBytes;
    const uint16_t *src_s = p.scales + row * static_cast<size_t>(p.capacity / T) * kHeadDim;
    const int row_tok0 = static_cast<int>(row * p.capacity);
    const bool row_ok = row < static_cast<size_t>(p.batch) * p.num_kv_heads;
    (void)row_ok;
    const int scan_total = dense ? 0 : nref + nbs;
    int sc_next = 0;                // scan tiles issued
    int it_next = 0;                // attention stages issued (items + end markers)
    int q_ptr = part, sub = 0;      // position in the kept-block list (this part's: part + k R)
    int ends_sent = 0;
    uint64_t idle_since = 0;
    // copies that read the last block's re-quantised data wait for the
    // attention warps' flag; seeing it, the producer orders their generic
    // stores before its own async-proxy reads
    bool requant_seen = !owner_requant;
    auto requant_ready = [&]() {
      if (!requant_seen && ctrl[4] != 0) {
        __threadfence_block();
        fence_proxy_async_global();
        requant_seen = true;
      }
      return requant_seen;
    };
    while (true) {
      bool progress = false;
      // scan tiles
      while (sc_next < scan_total) {
        if (sc_next == 1 && local_in_smem) {  // the attention warps build this tile
          ++sc_next;
          continue;
        }
        const int st = sc_next % NSA;
        const int use = sc_next / NSA;
        const int jb = scan_block_index(sc_next, nref, nb, j0);
        if (jb == nb - 1 && !requant_ready()) break;
        if (use > 0 && !mbar_test_wait(&empty_a[st], static_cast<uint32_t>(use - 1) & 1u)) break;
        uint8_t *dst = scan_ring + st * SG::kStageBytes;
        sh.scan_seq[st] = sc_next;
        mbar_arrive_expect_tx(&full_a[st], SG::kStageBytes);
        if (FFD_IN_BOUNDS(p, jb >= 0 && (jb + 1) * T <= p.capacity && row_ok)) {
          bulk_g2s(dst, src_p + static_cast<size_t>(jb) * T * SG::kRowBytes, T * SG::kRowBytes,
                   &full_a[st]);
          bulk_g2s(dst + T * SG::kRowBytes, src_s + static_cast<size_t>(jb) * kHeadDim,
                   kScaleRowBytes, &full_a[st]);
        }
        ++sc_next;
        progress = true;
      }
      // K/V stages for the kept blocks published so far
      // (acquire loads: the queue entries below are read after the count)
      const bool sel_done = dense || ld_acquire_cta(&ctrl[1]) != 0;
      const int avail = dense ? nbs : ld_acquire_cta(&ctrl[0]);
      while (q_ptr < avail) {
        const int j = dense ? q_ptr : static_cast<int>(queue[q_ptr]);
        const int tok = (j0 + j) * T + sub * kKvTok;
        if (sub >= kSubPerBlock || tok >= len) {
          q_ptr += R;  // this part's next kept block
          sub = 0;
          continue;
        }
        // (the int4 computer reads bf16 K/V, which only the fused append changes)
        if ((kTR || p.k_new != nullptr) && j0 + j == nb - 1 && !requant_ready()) break;
        const int st = it_next % NKV;
        const int use = it_next / NKV;
        if (use > 0 && !mbar_test_wait(&empty_b[st], static_cast<uint32_t>(use - 1) & 1u)) break;
        uint8_t *dst = kv_ring + st * KG::kStageBytes;
        meta[st] = tok;
        if constexpr (kTrL2) __threadfence_block();  // (the computer reads meta once seq shows the item)
        seq[st] = it_next;
        mbar_arrive_expect_tx(&full_b[st], KG::kTx);
        const int y = row_tok0 + tok;
        if (FFD_IN_BOUNDS(p, tok >= 0 && tok + kKvTok <= p.capacity && row_ok)) {
          if constexpr (kTR) {
            tma_load_2d(dst, &tmap_k, 0, y, &full_b[st]);  // residual rows
            if constexpr (!kTrL2) {
              bulk_g2s(dst + KG::kThumbOffset, src_p + static_cast<size_t>(tok) * kThumbRowBytes,
                       kKvTok * kThumbRowBytes, &full_b[st]);
              bulk_g2s(dst + KG::kScaleOffset, src_s + static_cast<size_t>(tok / T) * kHeadDim,
                       kScaleRowBytes, &full_b[st]);
            }
          } else {
            tma_load_3d(dst, &tmap_k, 0, y, 0, &full_b[st]);  // K: both halves
          }
          tma_load_3d(dst + KG::kVOffset, &tmap_v, 0, y, 0, &full_b[st]);  // V: both halves
        }
        ++it_next;
        ++sub;
        progress = true;
      }
      // once the selection is complete and every kept stage is issued, one
      // end marker per attention warp
      if (sel_done && q_ptr >= avail) {
        while (ends_sent < kAttnWarps) {
          const int st = it_next % NKV;
          const int use = it_next / NKV;
          if (use > 0 && !mbar_test_wait(&empty_b[st], static_cast<uint32_t>(use - 1) & 1u)) break;
          meta[st] = -1;
          if constexpr (kTrL2) __threadfence_block();
          seq[st] = it_next;
          mbar_arrive(&full_b[st]);
          ++it_next;
          ++ends_sent;
          progress = true;
        }
        if (ends_sent == kAttnWarps) break;
      }
      if (ctrl[3]) break;
      if (progress) {
        idle_since = 0;
      } else {
        const uint64_t now = global_timer_ns();
        if (idle_since == 0) {
          idle_since = now;
        } else if (now - idle_since > p.wait_limit_ns) {
          raise_timeout(p, ctrl);
          break;
        }
        __nanosleep(32);
      }
    }
    drain_ring(full_a, NSA, sc_next);  // (a skipped entry's phase is completed by its builders)
    drain_ring(full_b, NKV, it_next);
    return;
  }

  // ============================================================ scan warp
  if (warp == kScanWarp) {
    if (dense) return;
    const int gid = lane >> 2, t4 = lane & 3;
    float run0 = -INFINITY, run1 = -INFINITY;  // running max of heads 2*t4, 2*t4 + 1
    // the pages' rule: the pseudo-max is a fixed threshold (no running update)
    const bool fixed_ref = p.reference == 2;
    int qn = 0;
    // the Top-delta decision for scan entry e
    auto decide = [&](int e, float s0, float s1) {
      if (e < nref) {  // reference blocks: the pseudo-max is their max
        run0 = fmaxf(run0, s0);
        run1 = fmaxf(run1, s1);
        return;
      }
      const int i = e - nref;
      // Top-delta against the reference maximum, union over the group
      bool keep = false;
      if (gid == 0) {
        if (2 * t4 < G) {
          if (!fixed_ref) run0 = fmaxf(run0, s0);
          keep = s0 >= __fsub_rn(run0, p.delta);
        }
        if (2 * t4 + 1 < G) {
          if (!fixed_ref) run1 = fmaxf(run1, s1);
          keep = keep || (s1 >= __fsub_rn(run1, p.delta));
        }
      }
      if (__any_sync(kFull, keep)) {
        if (lane == 0) {
          keepbits[i >> 5] |= 1u << (i & 31);
          queue[qn] = static_cast<uint16_t>(i);
          __threadfence_block();
          ctrl[0] = qn + 1;
        }
        ++qn;
      }
    };
    const int total = nref + nbs;
    // Cooperative selector: the attention warps help the scan unless this
    // CTA's share of the split's kept blocks in the previous call on this
    // workspace (the split's selection bits are still there, and a part
    // attends over 1 / R of them) was at least 3/4 of the split (int4) or 1/8
    // (thumbnails, whose attention warps also rebuild every key): then the
    // attention warps are the bound and the scan warp keeps ahead alone.
    // This only spreads the work; the selection and the output do not depend
    // on it.  Decided here, after the pipeline has started, and published in
    // ctrl[7]: 1 = help (the query group is copied for the helpers first),
    // 2 = no help (the attention warps then wait plainly).
    bool help = false;
    if constexpr (kCoop) {
      // (both loads in flight together: the query group, 16 bytes x G x 16
      // over the lanes, and the split's previous bits)
      constexpr int kQv = (G * kHeadDim / 8 + 31) / 32;
      uint4 qrow[kQv];
      const uint4 *qsrc = reinterpret_cast<const uint4 *>(
          p.q + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G) * kHeadDim);
#pragma unroll
      for (int k = 0; k < kQv; ++k)
        if (lane + 32 * k < G * kHeadDim / 8) qrow[k] = qsrc[lane + 32 * k];
      int prev = 0;
      for (int w = lane; w < p.split_words; w += 32)
        prev += __popc(__ldcg(p.split_bits + (row * p.nsplit_max + split) * p.split_words + w));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) prev += __shfl_xor_sync(kFull, prev, off);
      help = kTR ? 8 * prev < nbs * R : 4 * prev < 3 * nbs * R;  // (a part attends over 1 / R of them)
      if (help) {
#pragma unroll
        for (int k = 0; k < kQv; ++k)
          if (lane + 32 * k < G * kHeadDim / 8) reinterpret_cast<uint4 *>(smem + SL::kQRows)[lane + 32 * k] = qrow[k];
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          ctrl[7] = 1;
        }
      } else if (lane == 0) {
        ctrl[7] = 2;
      }
    }
    if (!help) {
      // the scan warp alone: every entry in order, the query in registers
      using SF = ScanFold<G, F>;
      uint32_t qv[SF::NC / 2];
      SF::load_pairs(p.q + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G + gid % G) *
                               kHeadDim + 32 * t4,
                     SF::part(gid), qv);
      for (int e = 0; e < total; ++e) {
        const int st = e % NSA;
        if (!mbar_wait(&full_a[st], static_cast<uint32_t>(e / NSA) & 1u, p.wait_limit_ns)) {
          raise_timeout(p, ctrl);
          break;
        }
        const int jb = scan_block_index(e, nref, nb, j0);
        const uint8_t *tile = scan_ring + st * SG::kStageBytes;
        uint32_t bq[8];
        int sq, best0, best1;
        float am, s0, s1;
        fold_block<G, F>(reinterpret_cast<const uint16_t *>(tile + T * SG::kRowBytes), qv, lane, bq, sq, am);
        block_best<T, F>(tile, bq, min(T, len - jb * T), lane, best0, best1);
        block_scores<F>(best0, best1, sq, am, lane, s0, s1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_a[st]);
        decide(e, s0, s1);
        if (__shfl_sync(kFull, lane == 0 ? ctrl[3] : 0, 0)) break;
      }
      if (lane == 0) {
        __threadfence_block();
        ctrl[1] = 1;
      }
      return;
    }
    // score entries (the attention warps help while they wait for K/V) and
    // decide them in block order
    int decided = 0;
    uint64_t idle_since = 0;
    while (true) {
      bool progress = false;
      while (decided < total) {
        const int ready = __shfl_sync(kFull, lane == 0 ? sh.slot_seq[decided % kScanSlots] == decided : 0, 0);
        if (!ready) break;
        __threadfence_block();
        const float *slot = sh.scores + (decided % kScanSlots) * 8;
        decide(decided, slot[2 * t4], slot[2 * t4 + 1]);
        ++decided;
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          ctrl[6] = decided;  // frees the entry's slot
        }
        progress = true;
      }
      if (decided >= total || __shfl_sync(kFull, lane == 0 ? ctrl[3] : 0, 0)) break;
      // (the next entry whether or not its tile has landed: the scan warp
      // then waits on the stage's barrier rather than polling)
      const int e = claim_scan_entry<NSA>(sh, full_a, total, false, lane);
      if (e >= 0) {
        const int jb = scan_block_index(e, nref, nb, j0);
        float s0, s1;
        if (!score_scan_entry<T, G, F, C>(sh, scan_ring, full_a, empty_a, e, min(T, len - jb * T), lane,
                                          p.wait_limit_ns, s0, s1)) {
          raise_timeout(p, ctrl);
          break;
        }
        if (e == decided) {  // next in order: decide at once, no slot
          decide(e, s0, s1);
          ++decided;
          __syncwarp();
          if (lane == 0) {
            __threadfence_block();
            ctrl[6] = decided;
          }
        } else {
          publish_scan_scores(sh, e, s0, s1, lane);
        }
        progress = true;
      }
      if (progress) {
        idle_since = 0;
        continue;
      }
      const uint64_t now = global_timer_ns();
      if (idle_since == 0) {
        idle_since = now;
      } else if (now - idle_since > p.wait_limit_ns) {
        raise_timeout(p, ctrl);
        break;
      }
      __nanosleep(20);
    }
    if (lane == 0) {
      __threadfence_block();
      ctrl[1] = 1;
    }
    return;
  }

  // ======================================================= attention warps
  const int gid = lane >> 2, t4 = lane & 3;
  // int4 format -- Q^T as the bf16 mma B operand: k-step ks holds channels
  // 16ks + 2*t4 (+1) and 16ks + 8 + 2*t4 (+1) of head gid.
  // thumbnail format -- the bf16 pairs of channels 32*t4 + 2i (+1) of head gid,
  // folded with each block's scales into f16 per stage.
  uint32_t qb[8][2];
  {
    const uint32_t *qh = reinterpret_cast<const uint32_t *>(
        p.q + (static_cast<size_t>(b) * num_q_heads + static_cast<size_t>(g) * G + (gid < G ? gid : 0)) *
                  kHeadDim);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      if constexpr (kTR) {
        qb[ks][0] = gid < G ? qh[16 * t4 + 2 * ks] : 0u;
        qb[ks][1] = gid < G ? qh[16 * t4 + 2 * ks + 1] : 0u;
      } else {
        qb[ks][0] = gid < G ? qh[8 * ks + t4] : 0u;
        qb[ks][1] = gid < G ? qh[8 * ks + 4 + t4] : 0u;
      }
    }
  }
  // fused append: the new token's K row (read by the quantisers from k_new,
  // since this CTA's own cache store is not yet visible to them)
  const uint16_t *new_k_row = p.k_new != nullptr ? p.k_new + row * kHeadDim : nullptr;
  if (owner_requant) {
    // the last block's re-quantisation (see the prologue), after the append's
    // cache stores; all stores are fenced for the async proxy before the flag
    // releases the producer
    const int jl = nb - 1;
    const size_t tok0 = row * static_cast<size_t>(p.capacity) + static_cast<size_t>(jl) * T;
    if (new_k_row != nullptr && threadIdx.x < 32 && FFD_IN_BOUNDS(p, len >= 1 && len <= p.capacity)) {
      const size_t at = (row * static_cast<size_t>(p.capacity) + static_cast<size_t>(len - 1)) * kHeadDim;
      const int c = threadIdx.x & 15;
      if (threadIdx.x < 16)
        reinterpret_cast<uint4 *>(p.k_out + at)[c] = reinterpret_cast<const uint4 *>(new_k_row)[c];
      else
        reinterpret_cast<uint4 *>(p.v_out + at)[c] = reinterpret_cast<const uint4 *>(p.v_new + row * kHeadDim)[c];
    }
    float *red = reinterpret_cast<float *>(smem + SL::kRequant);
    uint16_t *scale_row = p.scales_out + (row * static_cast<size_t>(p.capacity / T) + jl) * kHeadDim;
    // (the condition is the same in every attention thread: the quantiser's
    // named barriers stay matched)
    if (FFD_IN_BOUNDS(p, jl >= 0 && (jl + 1) * T <= p.capacity &&
                             row < static_cast<size_t>(p.batch) * p.num_kv_heads)) {
      if constexpr (kTR)
        quantize_block_tr<T, kAttnThreads>(p.k + tok0 * kHeadDim, min(T, len - jl * T),
                                           p.packed_out + tok0 * kThumbRowBytes,
                                           p.resid_out + tok0 * kResidRowBytes, scale_row, red,
                                           red + kAttnWarps * kHeadDim, static_cast<int>(threadIdx.x), 2,
                                           new_k_row);
      else
        quantize_block<T, kAttnThreads>(p.k + tok0 * kHeadDim, min(T, len - jl * T),
                                        p.packed_out + tok0 * kPackedRowBytes, scale_row, red,
                                        red + kAttnWarps * kHeadDim, static_cast<int>(threadIdx.x), 2,
                                        new_k_row);
    }
    fence_proxy_async_global();
    __threadfence_block();
    named_barrier(2, kAttnThreads);
    if (threadIdx.x == 0) ctrl[4] = 1;
  }
  if (local_in_smem) {
    // Quantise the local block from K into scan stage 1 (the producer skips
    // that entry); scratch in the attention ring, idle until a block is kept,
    // which cannot happen before this entry has been scanned.
    const int jl = nb - 1;
    uint8_t *tile = scan_ring + 1 * SG::kStageBytes;
    float *red = reinterpret_cast<float *>(kv_ring);
    const uint16_t *k_rows = p.k + (row * static_cast<size_t>(p.capacity) + static_cast<size_t>(jl) * T) * kHeadDim;
    uint16_t *scale_row = reinterpret_cast<uint16_t *>(tile + T * SG::kRowBytes);
    if constexpr (kTR)
      quantize_block_tr<T, kAttnThreads>(k_rows, min(T, len - jl * T), tile, nullptr, scale_row, red,
                                         red + (kAttnThreads / 32) * kHeadDim,
                                         static_cast<int>(threadIdx.x), 2, new_k_row);
    else
      quantize_block<T, kAttnThreads>(k_rows, min(T, len - jl * T), tile, scale_row, red,
                                      red + (kAttnThreads / 32) * kHeadDim, static_cast<int>(threadIdx.x), 2,
                                      new_k_row);
    fence_proxy_async_smem();  // both regions are later written by async copies
    named_barrier(2, kAttnThreads);
    if (threadIdx.x == 0) {
      sh.scan_seq[1] = 1;
      mbar_arrive(&full_a[1]);
    }
  }
  float m_run[2] = {-INFINITY, -INFINITY};  // heads 2*t4, 2*t4 + 1
  float l_run[2] = {0.0f, 0.0f};
  float oacc[8][4];  // O^T: channel tile cm, rows 16cm + gid (+8), heads 2*t4 (+1)
#pragma unroll
  for (int cm = 0; cm < 8; ++cm) oacc[cm][0] = oacc[cm][1] = oacc[cm][2] = oacc[cm][3] = 0.0f;

  // Per-lane ldmatrix geometry.  K (A operand, non-transposed): row
  // 16mt + (lane & 7) + 8*((lane >> 3) & 1), 16-byte chunk 2ks + (lane >> 4).
  // V (A operand of O^T, transposed): row 16mt + (lane & 7) + 8*(lane >> 4),
  // chunk 2cm + ((lane >> 3) & 1).  Every row index is = lane & 7 (mod 8), so
  // the 128-byte swizzle XOR is a per-lane constant.
  const int r7 = lane & 7;
  const int k_row = r7 + 8 * ((lane >> 3) & 1);
  const int k_chi = lane >> 4;
  const int v_row = r7 + 8 * (lane >> 4);
  const int v_chi = (lane >> 3) & 1;
  const uint32_t kv_ring_addr = smem_addr(kv_ring);

  bool coop_wait = kCoop && !dense;  // until the scan warp says that this CTA does not help
  for (int it = warp;; it += kAttnWarps) {
    const int st = it % NKV;
    // Until item `it` is published, score scan entries whose tiles have
    // landed (the selector's work, decided in order by the scan warp).
    // (The scan warp publishes whether to help shortly after the start, so
    // the flag is read on every turn of the wait, one value for the warp.)
    if (coop_wait) {
      bool failed = false;
      uint64_t t0 = global_timer_ns();
      while (!__shfl_sync(kFull, lane == 0 ? seq[st] == it : 0, 0)) {
        const int flag = __shfl_sync(kFull, lane == 0 ? ctrl[7] : 0, 0);
        if (flag == 2) {  // no help in this call: wait plainly from now on
          coop_wait = false;
          break;
        }
        const int e = flag == 1 ? claim_scan_entry<NSA>(sh, full_a, nref + nbs, true, lane) : -2;
        if (e == -1) break;  // every entry is taken: wait for the item alone
        if (e >= 0) {
          const int jb = scan_block_index(e, nref, nb, j0);
          if (!score_scan_entry_helper<T, G, F>(sh, scan_ring, full_a, empty_a, e, min(T, len - jb * T), lane,
                                                p.wait_limit_ns)) {
            failed = true;
            break;
          }
          t0 = global_timer_ns();
        } else if (global_timer_ns() - t0 > p.wait_limit_ns) {
          failed = true;
          break;
        } else {
          __nanosleep(20);
        }
      }
      if (failed) {
        raise_timeout(p, ctrl);
        break;
      }
    }
    // Items go to the attention warps round-robin, so a warp can reach item
    // `it` before the stage's previous fill (another warp's item) has landed;
    // a parity wait could then match that older phase.  The producer writes
    // `it` into seq[st] only after the previous fill was consumed, so once it
    // is visible the parity below names exactly this fill.
    if (!wait_item_published(seq, st, it, p.wait_limit_ns)) {
      raise_timeout(p, ctrl);
      break;
    }
    constexpr int MT = kKvTok / 16;
    int tok = -1;
    float sc0 = kScaleLog2, sc1 = kScaleLog2;  // logit scale of heads 2*t4, 2*t4 + 1
    uint32_t qh[16];                           // thumbnail format: the folded query (f16 pairs)
    uint2 thumb[MT][2];                        // thumbnail format: rows 16mt + gid (+8), words 2*t4 (+1)
    if constexpr (kTrL2) {
      __threadfence_block();  // pairs with the producer's fence between meta and seq
      tok = meta[st];
      // While the stage's residuals and values are in flight, load its
      // thumbnail rows and its block's scale row from global memory (L2 after
      // the scan) and fold the scales into the query.  (Plain coherent loads:
      // the CTA that re-quantises the last block wrote these rows earlier in
      // this launch.)
      uint4 sv4[4] = {};
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) thumb[mt][0] = thumb[mt][1] = make_uint2(0u, 0u);
      if (tok >= 0 &&
          FFD_IN_BOUNDS(p, tok + kKvTok <= p.capacity && row < static_cast<size_t>(p.batch) * p.num_kv_heads)) {
        const uint8_t *trow = p.packed + (row * p.capacity + static_cast<size_t>(tok)) * kThumbRowBytes + 8 * t4;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          thumb[mt][0] = *reinterpret_cast<const uint2 *>(trow + (16 * mt + gid) * kThumbRowBytes);
          thumb[mt][1] = *reinterpret_cast<const uint2 *>(trow + (16 * mt + gid + 8) * kThumbRowBytes);
        }
        const uint4 *s4 =
            reinterpret_cast<const uint4 *>(
                p.scales + (row * static_cast<size_t>(p.capacity / T) + static_cast<size_t>(tok / T)) * kHeadDim) +
            4 * t4;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) sv4[w4] = s4[w4];
      }
      fold_query_tr(qb, t4, [&](int w4) { return sv4[w4]; }, qh, sc0, sc1);
    }
    if (!mbar_wait(&full_b[st], static_cast<uint32_t>(it / NKV) & 1u, p.wait_limit_ns)) {
      raise_timeout(p, ctrl);
      break;
    }
    if constexpr (!kTrL2) tok = meta[st];
    if (tok < 0) break;
    const uint32_t kbase = kv_ring_addr + st * KG::kStageBytes;
    const uint32_t vbase = kbase + KG::kVOffset;

    // S^T = K Q^T for kKvTok tokens: kKvTok/16 independent accumulator chains
    float sacc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) sacc[mt][0] = sacc[mt][1] = sacc[mt][2] = sacc[mt][3] = 0.0f;
    if constexpr (kTR) {
      // Lane (gid, t4) supplies channels 32*t4 + 16h + {2k, 2k+1} (a0/a1) and
      // {2k+8, 2k+9} (a2/a3) at k-step (h, k): thumbnail word 2*t4 + h and
      // residual chunk 2*t4 + h of rows gid and gid + 8 (both rows = gid mod
      // 8, so the swizzle XOR is gid).
      const uint8_t *stage = kv_ring + st * KG::kStageBytes;
      if constexpr (!kTrL2) {  // the block's scales from the stage
        const uint4 *s4 = reinterpret_cast<const uint4 *>(stage + KG::kScaleOffset) + 4 * t4;
        fold_query_tr(qb, t4, [&](int w4) { return s4[w4]; }, qh, sc0, sc1);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int r0 = 16 * mt + gid, r1 = r0 + 8;
        uint2 w0, w1;  // thumbnail words 2*t4 (+1) of rows r0, r1
        if constexpr (kTrL2) {
          w0 = thumb[mt][0];
          w1 = thumb[mt][1];
        } else {
          const uint8_t *thumb_s = stage + KG::kThumbOffset;
          w0 = *reinterpret_cast<const uint2 *>(thumb_s + r0 * kThumbRowBytes + 8 * t4);
          w1 = *reinterpret_cast<const uint2 *>(thumb_s + r1 * kThumbRowBytes + 8 * t4);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int chunk = ((2 * t4 + h) ^ gid) << 4;
          const uint4 e0 = *reinterpret_cast<const uint4 *>(stage + r0 * kResidRowBytes + chunk);
          const uint4 e1 = *reinterpret_cast<const uint4 *>(stage + r1 * kResidRowBytes + chunk);
          const uint32_t x0[4] = {e0.x, e0.y, e0.z, e0.w};
          const uint32_t x1[4] = {e1.x, e1.y, e1.z, e1.w};
          const uint32_t tw0 = h ? w0.y : w0.x, tw1 = h ? w1.y : w1.x;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t sel = (k & 1) ? 0x4342u : 0x4140u;
            const uint32_t a0 = key_pair(tw0 >> (2 * k), x0[k >> 1], sel);
            const uint32_t a1 = key_pair(tw1 >> (2 * k), x1[k >> 1], sel);
            const uint32_t a2 = key_pair(tw0 >> (2 * k + 8), x0[2 + (k >> 1)], sel);
            const uint32_t a3 = key_pair(tw1 >> (2 * k + 8), x1[2 + (k >> 1)], sel);
            mma_f16_16x8x16(sacc[mt], a0, a1, a2, a3, qh[8 * h + k], qh[8 * h + k + 4]);
          }
        }
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int chunk = 2 * ks + k_chi;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int r = 16 * mt + k_row;
          uint32_t a[4];
          ldmatrix_x4(a, kbase + (chunk >> 3) * kKvHalfBytes + r * 128 + (((chunk & 7) ^ r7) << 4));
          mma_bf16_16x8x16(sacc[mt], a[0], a[1], a[2], a[3], qb[ks][0], qb[ks][1]);
        }
      }
    }
    // online softmax (base 2); tokens at or past the length are masked
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int t_lo = tok + 16 * mt + gid;
      const bool v_lo = t_lo < len, v_hi = t_lo + 8 < len;
      sacc[mt][0] = v_lo ? sacc[mt][0] * sc0 : -INFINITY;
      sacc[mt][1] = v_lo ? sacc[mt][1] * sc1 : -INFINITY;
      sacc[mt][2] = v_hi ? sacc[mt][2] * sc0 : -INFINITY;
      sacc[mt][3] = v_hi ? sacc[mt][3] * sc1 : -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(sacc[mt][0], sacc[mt][2]));
      mx1 = fmaxf(mx1, fmaxf(sacc[mt][1], sacc[mt][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float corr0 = mn0 == -INFINITY ? 1.0f : exp2f(m_run[0] - mn0);
    const float corr1 = mn1 == -INFINITY ? 1.0f : exp2f(m_run[1] - mn1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    uint32_t pb[MT][2];
    float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const float e0 = mn0 == -INFINITY ? 0.0f : exp2f(sacc[mt][0] - mn0);
      const float e1 = mn1 == -INFINITY ? 0.0f : exp2f(sacc[mt][1] - mn1);
      const float e2 = mn0 == -INFINITY ? 0.0f : exp2f(sacc[mt][2] - mn0);
      const float e3 = mn1 == -INFINITY ? 0.0f : exp2f(sacc[mt][3] - mn1);
      // P rounded to bf16 once; the same weights feed P.V and the running sum
      const uint32_t lo = pack_bf16x2(e0, e1);  // token gid, heads 2*t4, 2*t4+1
      const uint32_t hi = pack_bf16x2(e2, e3);  // token gid + 8
      ps0 += bf16_lo(lo) + bf16_lo(hi);
      ps1 += bf16_hi(lo) + bf16_hi(hi);
      pb[mt][0] = movmatrix_trans(lo);  // head gid, tokens 16mt + 2*t4, +1
      pb[mt][1] = movmatrix_trans(hi);  // head gid, tokens 16mt + 8 + 2*t4, +1
    }
    l_run[0] = l_run[0] * corr0 + ps0;
    l_run[1] = l_run[1] * corr1 + ps1;
    // (the factor is exactly 1 whenever the running max stayed, which is most
    // stages once it has settled; skipping the multiply changes no bit)
    if (__any_sync(kFull, corr0 != 1.0f || corr1 != 1.0f)) {
#pragma unroll
      for (int cm = 0; cm < 8; ++cm) {
        oacc[cm][0] *= corr0;
        oacc[cm][1] *= corr1;
        oacc[cm][2] *= corr0;
        oacc[cm][3] *= corr1;
      }
    }
    // O^T += V^T P^T: 8 channel tiles x kKvTok/16 token steps
#pragma unroll
    for (int cm = 0; cm < 8; ++cm) {
      const int chunk = 2 * cm + v_chi;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int r = 16 * mt + v_row;
        uint32_t a[4];
        ldmatrix_x4_trans(a, vbase + (chunk >> 3) * kKvHalfBytes + r * 128 + (((chunk & 7) ^ r7) << 4));
        mma_bf16_16x8x16(oacc[cm], a[0], a[1], a[2], a[3], pb[mt][0], pb[mt][1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_b[st]);
  }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l_run[0] += __shfl_xor_sync(kFull, l_run[0], off);
    l_run[1] += __shfl_xor_sync(kFull, l_run[1], off);
  }

  // ------------------------------ split partial and the final merge
  named_barrier(1, kAttnThreads);  // every attention stage consumed; scan ring idle
  float *wm = reinterpret_cast<float *>(scan_ring);  // [warp][8]
  float *wl = wm + kAttnWarps * 8;                   // [warp][8]
  float *wacc = wl + kAttnWarps * 8;                 // [warp][8][128]
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * t4 + e;
    if (h < G) {
      if (gid == 0) {
        wm[warp * 8 + h] = m_run[e];
        wl[warp * 8 + h] = l_run[e];
      }
#pragma unroll
      for (int cm = 0; cm < 8; ++cm) {
        wacc[(warp * 8 + h) * kHeadDim + 16 * cm + gid] = oacc[cm][e];
        wacc[(warp * 8 + h) * kHeadDim + 16 * cm + gid + 8] = oacc[cm][2 + e];
      }
    }
  }
  named_barrier(1, kAttnThreads);
  const size_t unit = (row * p.nsplit_max + split) * R + part;
  float *part_out = p.partials + unit * G * kPartialStride;
  const bool unit_ok =
      FFD_IN_BOUNDS(p, unit < static_cast<size_t>(p.batch) * p.num_kv_heads * p.nsplit_max * R && split < p.nsplit_max);
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kAttnThreads) {
    const int h = idx >> 7, c = idx & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w * 8 + h]);
    float L = 0.0f, A = 0.0f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float mw = wm[w * 8 + h];
      if (mw != -INFINITY) {
        const float f = exp2f(mw - M);
        L += wl[w * 8 + h] * f;
        A += wacc[(w * 8 + h) * kHeadDim + c] * f;
      }
    }
    if (unit_ok) {
      part_out[h * kPartialStride + c] = A;
      if (c == 0) {
        part_out[h * kPartialStride + 128] = M;
        part_out[h * kPartialStride + 129] = L;
      }
    }
  }
  // (every part of a split holds the same selection: part 0 writes it)
  if (part == 0 && static_cast<int>(threadIdx.x) < p.split_words) {
    uint32_t bits = keepbits[threadIdx.x];
    if (dense) {  // every valid block of the split
      const int lo = 32 * threadIdx.x;
      bits = lo >= nbs ? 0u : (nbs - lo >= 32 ? kFull : ((1u << (nbs - lo)) - 1u));
    }
    if (unit_ok) p.split_bits[(row * p.nsplit_max + split) * p.split_words + threadIdx.x] = bits;
    // splits of a multiple of 32 blocks own whole mask words: write them here
    // rather than gather them in the final merge
    if (!p.partials_only && (p.split_blocks & 31) == 0 && (j0 >> 5) + static_cast<int>(threadIdx.x) < p.mask_words)
      p.mask[row * p.mask_words + (j0 >> 5) + threadIdx.x] = bits;
  }
  if (!p.partials_only && (p.split_blocks & 31) == 0 && split == nsplit - 1 && part == 0) {
    // the last split also clears the words past its range
    for (int w = ((j0 + p.split_blocks) >> 5) + static_cast<int>(threadIdx.x); w < p.mask_words; w += kAttnThreads)
      p.mask[row * p.mask_words + w] = 0u;
  }
  if (p.partials_only) return;  // context shard: the merge runs after the exchange
  // Split counter: the barrier, then one acquire-release add, publishes this
  // CTA's partial and mask words; the CTA that brings the count to nsplit
  // merges, its loads ordered after every other split's by the same add.
  named_barrier(1, kAttnThreads);
  if (threadIdx.x == 0)
    ctrl[2] = atomic_add_acq_rel_gpu(&p.counters[row], 1u) == static_cast<uint32_t>(nsplit * R - 1) ? 1 : 0;
  named_barrier(1, kAttnThreads);
  if (!ctrl[2]) return;

  // last CTA of (b, g): log-sum-exp merge over the splits.  Warp w merges
  // heads w, w + 4 (lane: output channels 4*lane .. 4*lane + 3).  Per chunk of
  // 16 splits every load (m, l and the lane's float4 of acc) is independent of
  // the others, so the merge costs about one L2 round trip per chunk; the
  // chunk is folded into a running (M, L, O) with the pairwise rule
  // (m1, l1, o1) + (m2, l2, o2) = (M, l1 2^(m1 - M) + l2 2^(m2 - M),
  // o1 2^(m1 - M) + o2 2^(m2 - M)), M = max(m1, m2).  A split that kept no
  // token has m = -inf and is skipped.
  const float *row_parts = p.partials + row * p.nsplit_max * R * G * kPartialStride;
  const int nunits = nsplit * R;  // the split partials, R per split
  constexpr int kChunk = 16;
  for (int h = warp; h < G; h += kAttnWarps) {
    float M = -INFINITY, L = 0.0f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < nunits; s0 += kChunk) {
      float ms[kChunk], ls[kChunk];
      float4 v[kChunk];
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        if (s0 + u < nunits) {
          const float *ps = row_parts + ((s0 + u) * G + h) * kPartialStride;
          ms[u] = __ldcg(ps + 128);
          ls[u] = __ldcg(ps + 129);
          v[u] = __ldcg(reinterpret_cast<const float4 *>(ps) + lane);
        } else {
          ms[u] = -INFINITY;
          ls[u] = 0.0f;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mc = M;
#pragma unroll
      for (int u = 0; u < kChunk; ++u) mc = fmaxf(mc, ms[u]);
      if (mc == -INFINITY) continue;
      const float f = M == -INFINITY ? 0.0f : exp2f(M - mc);
      L *= f;
      O.x *= f;
      O.y *= f;
      O.z *= f;
      O.w *= f;
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        if (ms[u] != -INFINITY) {
          const float wgt = exp2f(ms[u] - mc);
          L += ls[u] * wgt;
          O.x += wgt * v[u].x;
          O.y += wgt * v[u].y;
          O.z += wgt * v[u].z;
          O.w += wgt * v[u].w;
        }
      }
      M = mc;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    const uint32_t lo = pack_bf16x2(O.x * inv, O.y * inv), hi = pack_bf16x2(O.z * inv, O.w * inv);
    if (FFD_IN_BOUNDS(p, row < static_cast<size_t>(p.batch) * p.num_kv_heads))
      *reinterpret_cast<uint2 *>(out_rows + h * kHeadDim + 4 * lane) = make_uint2(lo, hi);
  }
  // mask row (splits not a multiple of 32 blocks): each word gathers 32
  // consecutive blocks' bits from the split bit rows
  if ((p.split_blocks & 31) != 0) {
    const uint32_t *row_bits = p.split_bits + row * p.nsplit_max * p.split_words;
    const int split_words = p.split_words;
    for (int w = threadIdx.x; w < p.mask_words; w += kAttnThreads)
      p.mask[row * p.mask_words + w] = gather_mask_word(
          w, nb, p.split_blocks, [&](int s, int wd) { return __ldcg(row_bits + s * split_words + wd); });
  }
  if (threadIdx.x == 0) p.counters[row] = 0u;
}

template <int T, int F, bool C>
constexpr size_t smem_bytes_tf(int split_blocks) {
  return 1024 + SmemLayout<T, F, C>::kKeep + 4 * static_cast<size_t>((((split_blocks + 31) / 32) + 3) & ~3) +
         2 * static_cast<size_t>((split_blocks + 7) & ~7);
}

// Two CTAs per SM (the launch bounds) need each CTA's dynamic shared memory
// within half of the SM's 228 KiB, less 1 KiB the hardware keeps per CTA.
constexpr size_t kSmemPerCta2 = (228 * 1024) / 2 - 1024;
static_assert(smem_bytes_tf<64, kFormatInt4, true>(FFD_MAX_SPLIT_BLOCKS) <= kSmemPerCta2, "two CTAs per SM");
static_assert(smem_bytes_tf<128, kFormatInt4, true>(FFD_MAX_SPLIT_BLOCKS) <= kSmemPerCta2, "two CTAs per SM");
static_assert(smem_bytes_tf<64, kFormatThumbResid, false>(FFD_MAX_SPLIT_BLOCKS) <= kSmemPerCta2, "two CTAs per SM");
static_assert(smem_bytes_tf<64, kFormatThumbResid, true>(FFD_MAX_SPLIT_BLOCKS) <= kSmemPerCta2, "two CTAs per SM");
static_assert(smem_bytes_tf<128, kFormatThumbResid, false>(FFD_MAX_SPLIT_BLOCKS) <= kSmemPerCta2, "two CTAs per SM");

// Raise the kernel's dynamic shared memory cap once per device, to the
// largest split this library accepts, so later launches (and graph captures)
// need no attribute call.
template <int T, int G, int F, bool C>
cudaError_t configure_tgfc() {
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit == 0 || (configured.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(decode_kernel<T, G, F, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes_tf<T, F, C>(FFD_MAX_SPLIT_BLOCKS)));
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  return cudaSuccess;
}

// The variants of one (T, G, F): the sparse-step variant (C) is built for
// 64-token blocks (at 128 tokens the cooperative selector's registers spill,
// and a thumbnail split of 64 blocks is too long for its rows to stay in L2).
template <int T, int F>
constexpr bool kHasSparseVariant = T == 64;

template <int T, int G, int F>
cudaError_t configure_tgf() {
  cudaError_t e = configure_tgfc<T, G, F, false>();
  if (e == cudaSuccess && kHasSparseVariant<T, F>) e = configure_tgfc<T, G, F, kHasSparseVariant<T, F>>();
  return e;
}

template <int T, int G, int F, bool C>
cudaError_t launch_tgfc(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, dim3 grid,
                        cudaStream_t stream) {
  cudaError_t e = configure_tgfc<T, G, F, C>();
  if (e != cudaSuccess) return e;
  const size_t smem = smem_bytes_tf<T, F, C>(p.split_blocks);
  decode_kernel<T, G, F, C><<<grid, kThreads, smem, stream>>>(p, tk, tv);
  return cudaGetLastError();
}

// Dense steps have no selector and no scan (so nothing puts thumbnail rows in
// L2 ahead of the computer); the thumbnail format's L2 loads pay only while a
// split's scan runs a short way ahead of its computer (at most 4096 tokens).
template <int T, int G, int F>
cudaError_t launch_tgf(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, dim3 grid,
                       cudaStream_t stream) {
  const bool sparse_variant =
      kHasSparseVariant<T, F> && !p.dense && (F == kFormatInt4 || p.split_blocks * T <= kTrL2MaxSplitTokens);
  if (sparse_variant) return launch_tgfc<T, G, F, kHasSparseVariant<T, F>>(p, tk, tv, grid, stream);
  return launch_tgfc<T, G, F, false>(p, tk, tv, grid, stream);
}

template <int T, int F>
cudaError_t configure_tf(int group) {
  switch (group) {
    case 1: return configure_tgf<T, 1, F>();
    case 2: return configure_tgf<T, 2, F>();
    case 4: return configure_tgf<T, 4, F>();
    case 8: return configure_tgf<T, 8, F>();
    default: return cudaErrorInvalidValue;
  }
}

template <int T, int F>
cudaError_t launch_tf(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int group,
                      dim3 grid, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_tgf<T, 1, F>(p, tk, tv, grid, stream);
    case 2: return launch_tgf<T, 2, F>(p, tk, tv, grid, stream);
    case 4: return launch_tgf<T, 4, F>(p, tk, tv, grid, stream);
    case 8: return launch_tgf<T, 8, F>(p, tk, tv, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int F>
cudaError_t launch_f(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int block_size,
                     int group, dim3 grid, cudaStream_t stream) {
  if (block_size == 64) return launch_tf<64, F>(p, tk, tv, group, grid, stream);
  if (block_size == 128) return launch_tf<128, F>(p, tk, tv, group, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

#ifdef FFD_DEBUG
namespace {
// Evaluates a failing bounds check, as a kernel index bug would.
__global__ void bounds_selftest_kernel(DecodeParams p) {
  if (threadIdx.x == 0 && FFD_IN_BOUNDS(p, p.batch < 0)) p.err[1] = 0u;
}
}  // namespace
#endif

size_t decode_smem_bytes(int block_size, int group, int split_blocks, int format) {
  (void)group;
  // the larger of a format's variants
  if (format == kFormatThumbResid)
    return block_size == 64 ? std::max(smem_bytes_tf<64, kFormatThumbResid, false>(split_blocks),
                                       smem_bytes_tf<64, kFormatThumbResid, true>(split_blocks))
                            : smem_bytes_tf<128, kFormatThumbResid, false>(split_blocks);
  return block_size == 64 ? smem_bytes_tf<64, kFormatInt4, true>(split_blocks)
                          : smem_bytes_tf<128, kFormatInt4, false>(split_blocks);
}

cudaError_t prepare_decode(int block_size, int group, int format) {
  const bool tr = format == kFormatThumbResid;
  if (block_size == 64) return tr ? configure_tf<64, kFormatThumbResid>(group) : configure_tf<64, kFormatInt4>(group);
  if (block_size == 128)
    return tr ? configure_tf<128, kFormatThumbResid>(group) : configure_tf<128, kFormatInt4>(group);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                          int block_size, int group, int format, dim3 grid, size_t smem_bytes,
                          cudaStream_t stream) {
  (void)smem_bytes;  // each variant's own size is used
  if (format == kFormatThumbResid)
    return launch_f<kFormatThumbResid>(p, tmap_k, tmap_v, block_size, group, grid, stream);
  if (format == kFormatInt4)
    return launch_f<kFormatInt4>(p, tmap_k, tmap_v, block_size, group, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ffd

#ifdef FFD_DEBUG
// Debug library only (not in the public header): sets FFD_DEVICE_FLAG_BOUNDS
// in the workspace's sticky word through the same check the kernel uses.
extern "C" ffd_status ffd_debug_bounds_selftest(void *workspace, void *cuda_stream) {
  if (workspace == nullptr) return FFD_ERR_INVALID_ARG;
  ffd::DecodeParams p{};
  p.err = static_cast<uint32_t *>(workspace);
  p.batch = 1;
  ffd::bounds_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(cuda_stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? FFD_OK : FFD_ERR_CUDA;
}
#endif
