// api.cu -- the C ABI declared in include/ffd.h: host-side validation,
// workspace layout, TMA descriptors and kernel launches.  No entry point
// allocates memory or synchronises, except ffd_check_device_status.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "ffd.h"
#include "ffd_internal.h"

namespace ffd {

namespace {

constexpr int32_t kAbiVersion = 2;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ffd_status check_shape(const ffd_shape *s) {
  if (s == nullptr) return FFD_ERR_INVALID_ARG;
  if (s->batch < 0 || s->num_q_heads <= 0 || s->num_kv_heads <= 0 || s->capacity < 0 ||
      s->head_dim <= 0 || s->block_size <= 0 || s->split_blocks <= 0)
    return FFD_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return FFD_ERR_INVALID_ARG;
  if (s->capacity % s->block_size != 0) return FFD_ERR_INVALID_ARG;
  if (s->head_dim != kHeadDim) return FFD_ERR_UNSUPPORTED;
  if (s->block_size != 64 && s->block_size != 128) return FFD_ERR_UNSUPPORTED;
  if (s->split_blocks > FFD_MAX_SPLIT_BLOCKS) return FFD_ERR_UNSUPPORTED;
  const int g = s->num_q_heads / s->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8) return FFD_ERR_UNSUPPORTED;
  if (s->num_kv_heads > 65535 || s->batch > 65535) return FFD_ERR_UNSUPPORTED;
  // token rows are addressed with 32-bit TMA coordinates
  if (static_cast<int64_t>(s->batch) * s->num_kv_heads * s->capacity >= (int64_t{1} << 31))
    return FFD_ERR_UNSUPPORTED;
  return FFD_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// K or V cache as a 3-D tensor {64 channels, token rows, 2 halves}: a row is
// 128 bf16 (256 bytes) and a half its low or high 128 bytes.  One box
// {64, kKvBoxRows, 2} is one attention stage's K (or V) tile; the 128-byte
// swizzle applies per 128-byte box row, and shared memory receives the tile
// as [half][row][64 channels].
bool make_kv_tensor_map(CUtensorMap *map, const void *base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[3] = {64, rows > 0 ? rows : 1, 2};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kKvBoxRows), 2};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                            strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Residuals of the thumbnail format as a 2-D u8 tensor {128 bytes, token
// rows}; one box {128, kKvBoxRows} is one attention stage's residual tile,
// 128-byte swizzled like the K/V tiles.
bool make_resid_tensor_map(CUtensorMap *map, const void *base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kResidRowBytes), rows > 0 ? rows : 1};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kResidRowBytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kResidRowBytes), static_cast<cuuint32_t>(kKvBoxRows)};
  const cuuint32_t elem_strides[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                            box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int32_t parts_per_split(int32_t batch, int32_t num_kv_heads, int32_t capacity, int32_t block_size,
                        int32_t split_blocks) {
  constexpr int64_t kSlots = 2 * 148;  // two CTAs per SM on a B200
  const int64_t nblk = capacity / block_size;
  const int64_t units = static_cast<int64_t>(batch) * num_kv_heads * ((nblk + split_blocks - 1) / split_blocks);
  int32_t r = 1;
  while (r < 8 && 2 * r <= split_blocks && units * 2 * r <= kSlots) r *= 2;
  return r;
}

WorkspaceLayout workspace_layout(int32_t batch, int32_t num_kv_heads, int32_t group, int32_t capacity,
                                 int32_t block_size, int32_t split_blocks, int32_t parts) {
  WorkspaceLayout L{};
  const int64_t nblk = capacity / block_size;
  L.nsplit_max = static_cast<int32_t>((nblk + split_blocks - 1) / split_blocks);
  L.split_words = (split_blocks + 31) / 32;
  L.parts = parts;
  const size_t rows = static_cast<size_t>(batch) * num_kv_heads;
  size_t off = 0;
  L.err = off;
  off += 256;
  L.counters = off;
  off += round_up(rows * 4, 256);
  L.split_bits = off;
  off += round_up(rows * L.nsplit_max * L.split_words * 4, 256);
  L.partials = off;
  off += rows * L.nsplit_max * parts * group * kPartialStride * 4;
  L.total = round_up(off, 256);
  return L;
}

}  // namespace ffd

using namespace ffd;

extern "C" {

int32_t ffd_abi_version(void) { return kAbiVersion; }

const char *ffd_status_string(ffd_status status) {
  switch (status) {
    case FFD_OK: return "ok";
    case FFD_ERR_INVALID_ARG: return "invalid argument";
    case FFD_ERR_UNSUPPORTED: return "unsupported shape";
    case FFD_ERR_WORKSPACE: return "workspace missing or too small";
    case FFD_ERR_CUDA: return "CUDA runtime error";
    case FFD_ERR_DEVICE_CHECK: return "device-side error flag set";
    case FFD_ERR_TIMEOUT: return "bounded device wait expired";
  }
  return "unknown status";
}

size_t ffd_packed_bytes(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  return static_cast<size_t>(s->batch) * s->num_kv_heads * s->capacity * (kHeadDim / 2);
}

size_t ffd_thumb_bytes(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  return static_cast<size_t>(s->batch) * s->num_kv_heads * s->capacity * kThumbRowBytes;
}

size_t ffd_residual_bytes(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  return static_cast<size_t>(s->batch) * s->num_kv_heads * s->capacity * kResidRowBytes;
}

size_t ffd_scale_bytes(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  return static_cast<size_t>(s->batch) * s->num_kv_heads * (s->capacity / s->block_size) * kHeadDim * 2;
}

size_t ffd_mask_words(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  const size_t nblk = s->capacity / s->block_size;
  return static_cast<size_t>(s->batch) * s->num_kv_heads * ((nblk + 31) / 32);
}

size_t ffd_decode_workspace_bytes(const ffd_shape *s) {
  if (check_shape(s) != FFD_OK) return 0;
  return workspace_layout(s->batch, s->num_kv_heads, s->num_q_heads / s->num_kv_heads, s->capacity,
                          s->block_size, s->split_blocks,
                          parts_per_split(s->batch, s->num_kv_heads, s->capacity, s->block_size, s->split_blocks))
      .total;
}

ffd_status ffd_workspace_init(const ffd_shape *s, void *workspace, size_t workspace_bytes,
                              void *cuda_stream) {
  ffd_status st = check_shape(s);
  if (st != FFD_OK) return st;
  const size_t need = ffd_decode_workspace_bytes(s);
  if (workspace == nullptr || workspace_bytes < need) return FFD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FFD_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, need, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FFD_ERR_CUDA;
  return FFD_OK;
}

}  // extern "C"

namespace {

ffd_status quantize_common(const ffd_shape *s, const void *k_bf16, const int32_t *d_lengths,
                           int32_t block_begin, void *packed, void *resid, void *k_scales, int format,
                           void *cuda_stream) {
  ffd_status st = check_shape(s);
  if (st != FFD_OK) return st;
  if (block_begin < FFD_LAST_BLOCK) return FFD_ERR_INVALID_ARG;
  const int nblk = s->capacity / s->block_size;
  if (s->batch == 0 || nblk == 0) return FFD_OK;
  const bool tr = format == kFormatThumbResid;
  if (k_bf16 == nullptr || d_lengths == nullptr || packed == nullptr || k_scales == nullptr ||
      (tr && resid == nullptr))
    return FFD_ERR_INVALID_ARG;
  if (!aligned16(k_bf16) || !aligned16(packed) || !aligned16(k_scales) || (tr && !aligned16(resid)) ||
      (reinterpret_cast<uintptr_t>(d_lengths) & 3u) != 0)
    return FFD_ERR_INVALID_ARG;
  const int blocks = block_begin < 0 ? 1 : nblk - block_begin;
  if (blocks <= 0) return FFD_OK;
  QuantizeParams p{};
  p.k = static_cast<const uint16_t *>(k_bf16);
  p.lengths = d_lengths;
  p.packed = static_cast<uint8_t *>(packed);
  p.scales = static_cast<uint16_t *>(k_scales);
  p.resid = tr ? static_cast<uint8_t *>(resid) : nullptr;
  p.batch = s->batch;
  p.num_kv_heads = s->num_kv_heads;
  p.capacity = s->capacity;
  p.block_begin = block_begin;
  p.format = format;
  const dim3 grid(static_cast<unsigned>(blocks), static_cast<unsigned>(s->num_kv_heads),
                  static_cast<unsigned>(s->batch));
  if (launch_quantize(p, s->block_size, grid, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FFD_ERR_CUDA;
  return FFD_OK;
}

}  // namespace

extern "C" {

ffd_status ffd_quantize_keys(const ffd_shape *s, const void *k_bf16, const int32_t *d_lengths,
                             int32_t block_begin, void *k_packed, void *k_scales, void *cuda_stream) {
  return quantize_common(s, k_bf16, d_lengths, block_begin, k_packed, nullptr, k_scales, kFormatInt4,
                         cuda_stream);
}

ffd_status ffd_quantize_keys_tr(const ffd_shape *s, const void *k_bf16, const int32_t *d_lengths,
                                int32_t block_begin, void *k_thumb, void *k_resid, void *k_scales,
                                void *cuda_stream) {
  return quantize_common(s, k_bf16, d_lengths, block_begin, k_thumb, k_resid, k_scales, kFormatThumbResid,
                         cuda_stream);
}

namespace {

// Where the keys come from: the int4 scan copy beside the bf16 cache, or the
// thumbnail + residual pair (bf16 K then read only by the re-quantisation).
struct KeyBuffers {
  int format;
  const void *k;       // bf16 K cache
  const void *packed;  // int4 codes or thumbnails
  const void *resid;   // residuals (thumbnail format)
  const void *scales;
};

// Shared body of every decode entry point.
// k_new / v_new (bf16 [B][Hkv][D], both or neither): the fused append writes
// them into the caches at position length - 1 (requant must be set).
ffd_status decode_common(const ffd_shape *s, const void *q_bf16, const KeyBuffers &kb, const void *v_bf16,
                         const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                         void *workspace, size_t workspace_bytes, void *cuda_stream, bool requant,
                         int32_t reference, bool partials_only = false, const void *k_new = nullptr,
                         const void *v_new = nullptr, uint64_t wait_limit_ns = kWaitLimitNs,
                         bool clear_counters = false) {
  ffd_status st = check_shape(s);
  if (st != FFD_OK) return st;
  if (reference != FFD_REFERENCE_RUNNING_MAX && reference != FFD_REFERENCE_SINK_LOCAL &&
      reference != FFD_REFERENCE_SINK_LOCAL_FIXED)
    return FFD_ERR_INVALID_ARG;
  if (partials_only) {
    // a context shard: splits must not straddle shards, and the pseudo-max
    // would need the sink and local blocks of other shards
    if (s->capacity % (s->block_size * s->split_blocks) != 0) return FFD_ERR_INVALID_ARG;
    if (reference != FFD_REFERENCE_RUNNING_MAX) return FFD_ERR_UNSUPPORTED;
  }
  if (std::isnan(delta) || delta < 0.0f) return FFD_ERR_INVALID_ARG;
  if (s->batch == 0) return FFD_OK;
  const bool dense = std::isinf(delta);
  const bool tr = kb.format == kFormatThumbResid;
  const int group = s->num_q_heads / s->num_kv_heads;
  // a context shard keeps one CTA per split: its exchanged region is the
  // one-part layout that ffd_partials_region names
  const int32_t parts = partials_only ? 1 : parts_per_split(s->batch, s->num_kv_heads, s->capacity,
                                                            s->block_size, s->split_blocks);
  const WorkspaceLayout L =
      workspace_layout(s->batch, s->num_kv_heads, group, s->capacity, s->block_size, s->split_blocks, parts);
  if (workspace == nullptr || workspace_bytes < L.total) return FFD_ERR_WORKSPACE;
  if (q_bf16 == nullptr || v_bf16 == nullptr || d_lengths == nullptr ||
      (!partials_only && (out_bf16 == nullptr || mask == nullptr)))
    return FFD_ERR_INVALID_ARG;
  // bf16 K: the int4 format's computer reads it; both formats re-quantise from it
  const bool need_k = !tr || requant;
  // scan copy: needed by the selector and written by the re-quantisation; the
  // thumbnail format's computer always reads thumbnails, residuals and scales
  const bool need_packed = tr || requant || !dense;
  if (need_k && kb.k == nullptr) return FFD_ERR_INVALID_ARG;
  if (need_packed && (kb.packed == nullptr || kb.scales == nullptr)) return FFD_ERR_INVALID_ARG;
  if (tr && kb.resid == nullptr) return FFD_ERR_INVALID_ARG;
  const bool append = k_new != nullptr || v_new != nullptr;
  if (append && (k_new == nullptr || v_new == nullptr || kb.k == nullptr || !requant ||
                 !aligned16(k_new) || !aligned16(v_new)))
    return FFD_ERR_INVALID_ARG;
  if (!aligned16(q_bf16) || !aligned16(kb.k) || !aligned16(v_bf16) || !aligned16(out_bf16) ||
      !aligned16(mask) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(d_lengths) & 3u) != 0)
    return FFD_ERR_INVALID_ARG;  // (null pointers pass: aligned16(nullptr) holds)
  if (!aligned16(kb.packed) || !aligned16(kb.scales) || !aligned16(kb.resid)) return FFD_ERR_INVALID_ARG;

  const uint64_t rows = static_cast<uint64_t>(s->batch) * s->num_kv_heads * s->capacity;
  CUtensorMap tmap_k, tmap_v;
  const bool kmap_ok = tr ? make_resid_tensor_map(&tmap_k, kb.resid, rows) : make_kv_tensor_map(&tmap_k, kb.k, rows);
  if (!kmap_ok || !make_kv_tensor_map(&tmap_v, v_bf16, rows)) return FFD_ERR_CUDA;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecodeParams p{};
  p.q = static_cast<const uint16_t *>(q_bf16);
  p.packed = static_cast<const uint8_t *>(kb.packed);
  p.scales = static_cast<const uint16_t *>(kb.scales);
  p.lengths = d_lengths;
  p.out = static_cast<uint16_t *>(out_bf16);
  p.mask = mask;
  p.err = reinterpret_cast<uint32_t *>(ws + L.err);
  p.counters = reinterpret_cast<uint32_t *>(ws + L.counters);
  p.split_bits = reinterpret_cast<uint32_t *>(ws + L.split_bits);
  p.partials = reinterpret_cast<float *>(ws + L.partials);
  p.batch = s->batch;
  p.num_kv_heads = s->num_kv_heads;
  p.capacity = s->capacity;
  p.split_blocks = s->split_blocks;
  p.nsplit_max = L.nsplit_max;
  p.mask_words = static_cast<int32_t>((s->capacity / s->block_size + 31) / 32);
  p.split_words = L.split_words;
  p.delta = delta;
  p.dense = dense ? 1 : 0;
  p.requant_last = requant ? 1 : 0;
  p.reference = reference;
  p.partials_only = partials_only ? 1 : 0;
  p.parts = L.parts;
  p.wait_limit_ns = wait_limit_ns;
  p.k = static_cast<const uint16_t *>(kb.k);
  p.packed_out = requant ? static_cast<uint8_t *>(const_cast<void *>(kb.packed)) : nullptr;
  p.scales_out = requant ? static_cast<uint16_t *>(const_cast<void *>(kb.scales)) : nullptr;
  p.resid_out = requant && tr ? static_cast<uint8_t *>(const_cast<void *>(kb.resid)) : nullptr;
  p.k_new = static_cast<const uint16_t *>(k_new);
  p.v_new = static_cast<const uint16_t *>(v_new);
  p.k_out = append ? static_cast<uint16_t *>(const_cast<void *>(kb.k)) : nullptr;
  p.v_out = append ? static_cast<uint16_t *>(const_cast<void *>(v_bf16)) : nullptr;

  const dim3 grid(static_cast<unsigned>(L.nsplit_max > 0 ? L.nsplit_max * L.parts : 1),
                  static_cast<unsigned>(s->num_kv_heads), static_cast<unsigned>(s->batch));
  const size_t smem = decode_smem_bytes(s->block_size, group, s->split_blocks, kb.format);
  if (clear_counters) {
    // a shared scratch area (decode_shared_scratch): the error word and the
    // arrival counters, which lie before the split bits, start at zero; only
    // now that the launch is certain
    if (L.err + 4 > L.split_bits || L.counters + static_cast<size_t>(s->batch) * s->num_kv_heads * 4 > L.split_bits)
      return FFD_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, L.split_bits, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
      return FFD_ERR_CUDA;
  }
  if (launch_decode(p, tmap_k, tmap_v, s->block_size, group, kb.format, grid, smem,
                    static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FFD_ERR_CUDA;
  return FFD_OK;
}

KeyBuffers int4_keys(const void *k, const void *packed, const void *scales) {
  return KeyBuffers{kFormatInt4, k, packed, nullptr, scales};
}

KeyBuffers tr_keys(const void *k, const void *thumb, const void *resid, const void *scales) {
  return KeyBuffers{kFormatThumbResid, k, thumb, resid, scales};
}

bool options_ok(const ffd_decode_options *opt) {
  return opt != nullptr && (opt->requant_last == 0 || opt->requant_last == 1) && opt->wait_limit_us >= 0;
}

uint64_t wait_limit(const ffd_decode_options *opt) {
  return opt->wait_limit_us > 0 ? static_cast<uint64_t>(opt->wait_limit_us) * 1000u : kWaitLimitNs;
}

}  // namespace

}  // extern "C"

namespace ffd {
ffd_status decode_shared_scratch(const ffd_shape *s, const void *q_bf16, const void *k_bf16,
                                 const void *v_bf16, const void *k_packed, const void *k_scales,
                                 const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                                 void *scratch, size_t scratch_bytes, void *cuda_stream) {
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_lengths, delta, out_bf16,
                       mask, scratch, scratch_bytes, cuda_stream, false, FFD_REFERENCE_RUNNING_MAX, false,
                       nullptr, nullptr, kWaitLimitNs, true);
}
}  // namespace ffd

extern "C" {

ffd_status ffd_decode(const ffd_shape *s, const void *q_bf16, const void *k_bf16, const void *v_bf16,
                      const void *k_packed, const void *k_scales, const int32_t *d_lengths, float delta,
                      void *out_bf16, uint32_t *mask, void *workspace, size_t workspace_bytes,
                      void *cuda_stream) {
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_lengths, delta, out_bf16,
                       mask, workspace, workspace_bytes, cuda_stream, false, FFD_REFERENCE_RUNNING_MAX);
}

ffd_status ffd_decode_step(const ffd_shape *s, const void *q_bf16, const void *k_bf16,
                           const void *v_bf16, void *k_packed, void *k_scales,
                           const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                           void *workspace, size_t workspace_bytes, void *cuda_stream) {
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_lengths, delta, out_bf16,
                       mask, workspace, workspace_bytes, cuda_stream, true, FFD_REFERENCE_RUNNING_MAX);
}

ffd_status ffd_decode_partials(const ffd_shape *s, const ffd_decode_options *opt, const void *q_bf16,
                               const void *k_bf16, const void *v_bf16, void *k_packed, void *k_scales,
                               const int32_t *d_local_lengths, float delta, void *workspace,
                               size_t workspace_bytes, void *cuda_stream) {
  if (!options_ok(opt)) return FFD_ERR_INVALID_ARG;
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_local_lengths, delta,
                       nullptr, nullptr, workspace, workspace_bytes, cuda_stream, opt->requant_last == 1,
                       opt->reference, true, nullptr, nullptr, wait_limit(opt));
}

ffd_status ffd_decode_partials_tr(const ffd_shape *s, const ffd_decode_options *opt, const void *q_bf16,
                                  const void *k_bf16, const void *v_bf16, void *k_thumb, void *k_resid,
                                  void *k_scales, const int32_t *d_local_lengths, float delta,
                                  void *workspace, size_t workspace_bytes, void *cuda_stream) {
  if (!options_ok(opt)) return FFD_ERR_INVALID_ARG;
  return decode_common(s, q_bf16, tr_keys(k_bf16, k_thumb, k_resid, k_scales), v_bf16, d_local_lengths,
                       delta, nullptr, nullptr, workspace, workspace_bytes, cuda_stream,
                       opt->requant_last == 1, opt->reference, true, nullptr, nullptr, wait_limit(opt));
}

ffd_status ffd_partials_region(const ffd_shape *s, size_t *offset, size_t *bytes) {
  ffd_status st = check_shape(s);
  if (st != FFD_OK) return st;
  if (offset == nullptr || bytes == nullptr) return FFD_ERR_INVALID_ARG;
  const WorkspaceLayout L = workspace_layout(s->batch, s->num_kv_heads, s->num_q_heads / s->num_kv_heads,
                                             s->capacity, s->block_size, s->split_blocks);
  *offset = L.split_bits;
  *bytes = L.total - L.split_bits;
  return FFD_OK;
}

ffd_status ffd_merge_partials(const ffd_shape *s, int32_t num_shards, const void *gathered,
                              size_t gathered_bytes, const int32_t *d_global_lengths, void *out_bf16,
                              uint32_t *mask, void *cuda_stream) {
  ffd_status st = check_shape(s);
  if (st != FFD_OK) return st;
  if (num_shards < 1 || s->capacity % (s->block_size * s->split_blocks) != 0) return FFD_ERR_INVALID_ARG;
  if (static_cast<int64_t>(num_shards) * s->capacity >= (int64_t{1} << 31)) return FFD_ERR_UNSUPPORTED;
  if (s->batch == 0) return FFD_OK;
  const int group = s->num_q_heads / s->num_kv_heads;
  const WorkspaceLayout L =
      workspace_layout(s->batch, s->num_kv_heads, group, s->capacity, s->block_size, s->split_blocks);
  const size_t region = L.total - L.split_bits;
  if (gathered == nullptr || d_global_lengths == nullptr || out_bf16 == nullptr || mask == nullptr)
    return FFD_ERR_INVALID_ARG;
  if (gathered_bytes < region * num_shards) return FFD_ERR_WORKSPACE;
  if (!aligned16(gathered) || !aligned16(out_bf16) || !aligned16(mask) ||
      (reinterpret_cast<uintptr_t>(d_global_lengths) & 3u) != 0)
    return FFD_ERR_INVALID_ARG;
  // every shard's split statistics live in shared memory (48 KiB without opt-in)
  if (merge_smem_bytes(num_shards, L.nsplit_max) > 48 * 1024) return FFD_ERR_UNSUPPORTED;
  MergeParams p{};
  p.gathered = static_cast<const uint8_t *>(gathered);
  p.region_bytes = region;
  p.partials_offset = L.partials - L.split_bits;
  p.lengths = d_global_lengths;
  p.out = static_cast<uint16_t *>(out_bf16);
  p.mask = mask;
  p.num_kv_heads = s->num_kv_heads;
  p.capacity = s->capacity;
  p.split_blocks = s->split_blocks;
  p.nsplit_max = L.nsplit_max;
  p.split_words = L.split_words;
  p.mask_words = static_cast<int32_t>((static_cast<int64_t>(num_shards) * (s->capacity / s->block_size) + 31) / 32);
  p.num_shards = num_shards;
  const dim3 grid(static_cast<unsigned>(s->num_kv_heads), static_cast<unsigned>(s->batch));
  if (launch_merge(p, s->block_size, group, grid, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess)
    return FFD_ERR_CUDA;
  return FFD_OK;
}

ffd_status ffd_decode_ex(const ffd_shape *s, const ffd_decode_options *opt, const void *q_bf16,
                         const void *k_bf16, const void *v_bf16, void *k_packed, void *k_scales,
                         const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                         void *workspace, size_t workspace_bytes, void *cuda_stream) {
  if (!options_ok(opt)) return FFD_ERR_INVALID_ARG;
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_lengths, delta, out_bf16,
                       mask, workspace, workspace_bytes, cuda_stream, opt->requant_last == 1,
                       opt->reference, false, nullptr, nullptr, wait_limit(opt));
}

ffd_status ffd_decode_append(const ffd_shape *s, int32_t reference, const void *q_bf16,
                             const void *k_new_bf16, const void *v_new_bf16, void *k_bf16, void *v_bf16,
                             void *k_packed, void *k_scales, const int32_t *d_lengths, float delta,
                             void *out_bf16, uint32_t *mask, void *workspace, size_t workspace_bytes,
                             void *cuda_stream) {
  return decode_common(s, q_bf16, int4_keys(k_bf16, k_packed, k_scales), v_bf16, d_lengths, delta, out_bf16,
                       mask, workspace, workspace_bytes, cuda_stream, true, reference, false, k_new_bf16,
                       v_new_bf16);
}

ffd_status ffd_decode_append_tr(const ffd_shape *s, int32_t reference, const void *q_bf16,
                                const void *k_new_bf16, const void *v_new_bf16, void *k_bf16, void *v_bf16,
                                void *k_thumb, void *k_resid, void *k_scales, const int32_t *d_lengths,
                                float delta, void *out_bf16, uint32_t *mask, void *workspace,
                                size_t workspace_bytes, void *cuda_stream) {
  return decode_common(s, q_bf16, tr_keys(k_bf16, k_thumb, k_resid, k_scales), v_bf16, d_lengths, delta,
                       out_bf16, mask, workspace, workspace_bytes, cuda_stream, true, reference, false,
                       k_new_bf16, v_new_bf16);
}

ffd_status ffd_decode_tr(const ffd_shape *s, const ffd_decode_options *opt, const void *q_bf16,
                         const void *k_bf16, const void *v_bf16, void *k_thumb, void *k_resid,
                         void *k_scales, const int32_t *d_lengths, float delta, void *out_bf16,
                         uint32_t *mask, void *workspace, size_t workspace_bytes, void *cuda_stream) {
  if (!options_ok(opt)) return FFD_ERR_INVALID_ARG;
  return decode_common(s, q_bf16, tr_keys(k_bf16, k_thumb, k_resid, k_scales), v_bf16, d_lengths, delta,
                       out_bf16, mask, workspace, workspace_bytes, cuda_stream, opt->requant_last == 1,
                       opt->reference, false, nullptr, nullptr, wait_limit(opt));
}

ffd_status ffd_check_device_status(void *workspace, uint32_t *flags_out, void *cuda_stream) {
  if (workspace == nullptr || !aligned16(workspace)) return FFD_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint32_t flags = 0;
  if (cudaMemcpyAsync(&flags, workspace, sizeof(flags), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return FFD_ERR_CUDA;
  if (flags != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(flags), stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return FFD_ERR_CUDA;
  }
  if (flags_out) *flags_out = flags;
  if (flags & FFD_DEVICE_FLAG_TIMEOUT) return FFD_ERR_TIMEOUT;
  return flags != 0 ? FFD_ERR_DEVICE_CHECK : FFD_OK;
}

}  // extern "C"
