// ffd_internal.h -- kernel parameter blocks and launchers shared between the
// host entry points (api.cu) and the kernels (quantize.cu, decode.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace ffd {

constexpr int kHeadDim = 128;
constexpr int kPackedRowBytes = kHeadDim / 2;  // 64 bytes of nibbles per token
constexpr int kThumbRowBytes = kHeadDim / 4;   // 32 bytes of 2-bit codes per token
constexpr int kResidRowBytes = kHeadDim;       // 128 residual bytes per token
constexpr int kScaleRowBytes = kHeadDim * 2;   // 128 bf16 scales per block

// Key formats: the int4 scan copy beside the bf16 cache, or the pages' split
// of K into 2-bit thumbnails and 8-bit residuals (no bf16 K on the read path).
constexpr int kFormatInt4 = 0;
constexpr int kFormatThumbResid = 1;

// Rows of one TMA box of K or V (tokens per attention pipeline stage); a box
// is 64 channels (128 bytes, the swizzle span) wide.
constexpr int kKvBoxRows = 32;
constexpr int kPartialStride = 132;  // floats per (split, head): acc[128], m, l
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded mbarrier waits (2 s)

constexpr uint32_t kFlagBadLength = 0x1u;
constexpr uint32_t kFlagTimeout = 0x2u;
constexpr uint32_t kFlagBounds = 0x4u;  // debug build only: an index left its extent

struct DecodeParams {
  const uint16_t *q;       // bf16 [B][Hq][D]
  const uint8_t *packed;   // scan copy: int4 [B][Hkv][cap][64] or thumbnails [B][Hkv][cap][32]
  const uint16_t *scales;  // bf16 [B][Hkv][nblk][D]
  const int32_t *lengths;  // [B]
  uint16_t *out;           // bf16 [B][Hq][D]
  uint32_t *mask;          // [B][Hkv][mask_words]
  uint32_t *err;           // sticky device flags
  uint32_t *counters;      // [B][Hkv]
  uint32_t *split_bits;    // [B][Hkv][nsplit_max][split_words]
  float *partials;         // [B][Hkv][nsplit_max][G][kPartialStride]
  int32_t batch, num_kv_heads, capacity, split_blocks, nsplit_max, mask_words, split_words;
  float delta;
  int32_t dense;
  // fused decode step: re-quantise each sequence's last key block first
  int32_t requant_last;
  // reference maximum: 0 = running max inside the split, 1 = running max
  // started at the pseudo-max of the sink (first) and local (last) blocks,
  // 2 = that pseudo-max as a fixed threshold
  int32_t reference;
  const uint16_t *k;         // bf16 [B][Hkv][cap][D] (read by the re-quantisation)
  uint8_t *packed_out;       // = packed, written for the last block
  uint16_t *scales_out;      // = scales, written for the last block
  uint8_t *resid_out;        // thumbnail format: residuals [B][Hkv][cap][128], last block
  // fused append: the new token's K and V rows (bf16 [B][Hkv][D]) are written
  // into the caches at position length - 1 by the CTA owning the last block
  const uint16_t *k_new;     // null: no append
  const uint16_t *v_new;
  uint16_t *k_out;           // = k (the bf16 K cache), written at the new token only
  uint16_t *v_out;           // = the bf16 V cache, written at the new token only
  // context sharding: write the split partials and bits only (no final merge;
  // out and mask unused)
  int32_t partials_only;
  // CTAs per split (grid.x = nsplit_max * parts): each scans the whole split
  // and attends over the kept blocks at kept-list positions = its index mod
  // parts, writing its own partial (partials [..][nsplit_max][parts][G][..])
  int32_t parts;
  // limit of the pipeline and queue waits (the drains of the kernel's own
  // copies always use kWaitLimitNs)
  uint64_t wait_limit_ns;
};

// Merge of split partials gathered from num_shards context shards.
struct MergeParams {
  const uint8_t *gathered;  // num_shards x region_bytes
  size_t region_bytes;      // one shard's workspace region: split bits, then partials
  size_t partials_offset;   // offset of the partials inside a region
  const int32_t *lengths;   // global lengths [B]
  uint16_t *out;            // bf16 [B][Hq][D]
  uint32_t *mask;           // [B][Hkv][mask_words] over the global capacity
  int32_t num_kv_heads, capacity, split_blocks, nsplit_max, split_words, mask_words, num_shards;
};

struct QuantizeParams {
  const uint16_t *k;
  const int32_t *lengths;
  uint8_t *packed;  // int4 rows, or thumbnail rows in the thumbnail format
  uint16_t *scales;
  uint8_t *resid;   // thumbnail format only
  int32_t batch, num_kv_heads, capacity, block_begin, format;
};

// Workspace carve-up (byte offsets), identical on host and device.
struct WorkspaceLayout {
  size_t err, counters, split_bits, partials, total;
  int32_t nsplit_max, split_words, parts;
};

// CTAs per split for a shape: the largest power of two up to 8 (and up to the
// split size) for which batch * kv-heads * splits * parts still fits in one
// wave of two CTAs on each of a B200's 148 SMs.
int32_t parts_per_split(int32_t batch, int32_t num_kv_heads, int32_t capacity, int32_t block_size,
                        int32_t split_blocks);

// parts: CTAs per split (the partials hold one slot per part).
WorkspaceLayout workspace_layout(int32_t batch, int32_t num_kv_heads, int32_t group,
                                 int32_t capacity, int32_t block_size, int32_t split_blocks,
                                 int32_t parts = 1);

size_t decode_smem_bytes(int block_size, int group, int split_blocks, int format);

size_t merge_smem_bytes(int num_shards, int nsplit_max);
cudaError_t launch_merge(const MergeParams &p, int block_size, int group, dim3 grid,
                         cudaStream_t stream);
cudaError_t launch_quantize(const QuantizeParams &p, int block_size, dim3 grid,
                            cudaStream_t stream);
// Kernel attributes for a (block size, group, format) variant, set once per
// device; launch_decode does it too, this lets a caller do it before a graph
// capture.
cudaError_t prepare_decode(int block_size, int group, int format);

// tmap_k maps the bf16 K cache (int4 format) or the residuals (thumbnail
// format); tmap_v the bf16 V cache.
cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmap_k,
                          const CUtensorMap &tmap_v, int block_size, int group, int format,
                          dim3 grid, size_t smem_bytes, cudaStream_t stream);

// ffd_decode on a scratch area shared between calls (the library's own
// device array of no_alloc.cu): every host check of ffd_decode runs first,
// then the error word and the arrival counters are cleared on the stream,
// then the kernel is launched.  Declared here with C++ linkage; the status
// type comes from ffd.h.
}  // namespace ffd
#include "ffd.h"
namespace ffd {
ffd_status decode_shared_scratch(const ffd_shape *s, const void *q_bf16, const void *k_bf16,
                                 const void *v_bf16, const void *k_packed, const void *k_scales,
                                 const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                                 void *scratch, size_t scratch_bytes, void *cuda_stream);
}  // namespace ffd
