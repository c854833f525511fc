/*
 * ffd.h -- C ABI of the B200 (sm_100a) Faster Flash Decoding decode path.
 *
 * Method: "Faster Than Flash: Exploiting Attention Sparsity for Efficient
 * Long-Context Decoding" (arXiv 2609.00097).  Single-token decode attention
 * over a long KV cache with a fused selector and computer: the selector scans
 * a low-bit copy of the keys (gist.science explainer, Methodology 1
 * "Content-Aware Scanning via Low-Bit Quantization"), keeps the blocks whose
 * tentative score lies within delta of a reference maximum (Methodology 2
 * "The Top-delta Selection Strategy"), and the computer runs exact attention
 * over the kept blocks only (Methodology 3, stage "Fine-Grained Refinement");
 * both live in one kernel (arXiv abstract: selector and computer "in a fully
 * fused kernel", scan results reused for computation).
 *
 * Conventions shared by every entry point
 *   - Pointers are caller-owned device memory unless stated otherwise; the
 *     library allocates nothing and keeps no state between calls.
 *   - Every device pointer must be 16-byte aligned; tensors are dense,
 *     row-major, in the layouts given below.
 *   - bf16 means IEEE bfloat16 bit patterns (uint16).
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = legacy
 *     default stream) and may be captured into a CUDA graph.  Per-sequence
 *     lengths live on the device, so no call reads device memory from the host.
 *   - Host-side argument checks fail before any launch and return a status;
 *     no entry point throws or aborts.  Length values are checked on the
 *     device (see ffd_decode).
 *
 * Shapes (symbols): B batch, Hq query heads, Hkv kv heads, G = Hq / Hkv,
 * D = 128 head dim, T block tokens, S split blocks, cap tokens per cache row,
 * nblk = cap / T, W = ceil(nblk / 32) mask words per (b, kv-head).
 *
 * Data layouts
 *   q        bf16 [B][Hq][D]                  query head h uses kv-head h / G
 *   k, v     bf16 [B][Hkv][cap][D]            the KV cache
 *   k_packed u8   [B][Hkv][cap][D/2]          int4 key copy: byte i of a token
 *            row holds channel 2i in the low nibble and channel 2i+1 in the high
 *            nibble, each as code + 8 with code in [-7, 7]
 *   k_scales bf16 [B][Hkv][nblk][D]           per-block-per-channel key scales
 *   lengths  int32 [B] (device)               valid tokens per sequence
 *   out      bf16 [B][Hq][D]
 *   mask     u32  [B][Hkv][W]                 bit (j % 32) of word j / 32 set iff
 *            block j was selected for that kv-head; bits >= ceil(len/T) are 0
 *   thumbnail + residual key format (ffd_quantize_keys_tr, ffd_decode_tr):
 *   k_thumb  u8   [B][Hkv][cap][D/4]          2-bit codes u in [0, 3]: channel
 *            16w + i of a token row sits in little-endian 32-bit word w at bit
 *            2 (i / 2) + 16 (i % 2) (even channels of the group in the low
 *            half-word, odd channels in the high half-word)
 *   k_resid  u8   [B][Hkv][cap][D]            8-bit residual e + 128, e in [-127, 127]
 *   k_scales bf16 [B][Hkv][nblk][D]           per-block-per-channel scales (as above)
 */
#ifndef FFD_H
#define FFD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FFD_OK = 0,
  FFD_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape, NaN or negative delta */
  FFD_ERR_UNSUPPORTED = 2,  /* a valid shape this library does not implement */
  FFD_ERR_WORKSPACE = 3,    /* workspace missing or smaller than ffd_decode_workspace_bytes */
  FFD_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, copy, tensor map) */
  FFD_ERR_DEVICE_CHECK = 5, /* ffd_check_device_status found a device-side error flag */
  FFD_ERR_TIMEOUT = 6       /* a bounded device wait gave up (ffd_check_device_status) */
} ffd_status;

/* Device-side error flags, reported by ffd_check_device_status. */
#define FFD_DEVICE_FLAG_BAD_LENGTH 0x1u /* some lengths[b] outside [0, cap] */
#define FFD_DEVICE_FLAG_TIMEOUT 0x2u    /* a bounded barrier wait expired */
/* Debug library only (libffd_b200_debug.so, built with FFD_DEBUG): a computed
 * global index left the extent the shape implies; that access was skipped. */
#define FFD_DEVICE_FLAG_BOUNDS 0x4u

/* block_begin value for ffd_quantize_keys: each sequence's last block only. */
#define FFD_LAST_BLOCK (-1)

/* Largest split size (blocks) this library accepts. */
#define FFD_MAX_SPLIT_BLOCKS 512

typedef struct {
  int32_t batch;        /* B >= 0 */
  int32_t num_q_heads;  /* Hq > 0, multiple of num_kv_heads */
  int32_t num_kv_heads; /* Hkv in [1, 65535] */
  int32_t head_dim;     /* D, must be 128 */
  int32_t capacity;     /* cap >= 0, multiple of block_size */
  int32_t block_size;   /* T: 64 or 128 */
  int32_t split_blocks; /* S in [1, FFD_MAX_SPLIT_BLOCKS] */
} ffd_shape;

/* Bytes of k_packed, k_scales; words of mask (all for the whole batch).
 * Return 0 for an invalid shape. */
size_t ffd_packed_bytes(const ffd_shape *shape);
size_t ffd_scale_bytes(const ffd_shape *shape);
size_t ffd_mask_words(const ffd_shape *shape);

/* Device workspace ffd_decode needs: split partials (running max, sum and
 * unnormalised output per head), per-split selection bits, one arrival
 * counter per (b, kv-head) and the sticky device error word.  When the
 * splits alone would leave SMs idle, R CTAs share each split (R the largest
 * power of two up to 8 and up to S with B * Hkv * ceil(nblk / S) * R <= 296,
 * two CTAs on each of a B200's 148 SMs): each scans the whole split, so all
 * take the same selection with no exchange, and attends over every R-th kept
 * block; the partials then hold R slots per split.  The selection bits a call
 * leaves in the workspace also steer how the next call on it spreads the
 * selector's work over its warps (never what it computes).  0 for an invalid
 * shape. */
size_t ffd_decode_workspace_bytes(const ffd_shape *shape);

/* Zero a workspace (cudaMemsetAsync on the stream).  Call once after
 * allocating it; ffd_decode leaves it ready for the next call. */
ffd_status ffd_workspace_init(const ffd_shape *shape, void *workspace,
                              size_t workspace_bytes, void *cuda_stream);

/* Low-bit key copy (gist.science explainer, Methodology 1: keys are kept as a
 * low-bit "thumbnail" used only for scanning; here int4 with per-block-per-
 * channel bf16 scales).  For every (b, kv-head) and every block j with
 * block_begin <= j < ceil(lengths[b] / T) -- or only j = ceil(lengths[b]/T) - 1
 * when block_begin == FFD_LAST_BLOCK -- over the block's valid tokens t:
 *   amax_c  = max_t |k[t][c]|,  s_c = bf16_rne(amax_c / 7)   (IEEE fp32 division)
 *   code    = s_c == 0 ? 0 : clamp(rint_even(k[t][c] / s_c), -7, 7)
 * Tokens at or beyond lengths[b] in the last block get code 0 and do not
 * enter amax.  Blocks outside that range are not written.  Sequences whose
 * length is outside [0, cap] are skipped (ffd_decode reports them).
 * Run it once over the whole cache after prefill (block_begin = 0) and with
 * FFD_LAST_BLOCK after each appended token. */
ffd_status ffd_quantize_keys(const ffd_shape *shape, const void *k_bf16,
                             const int32_t *d_lengths, int32_t block_begin,
                             void *k_packed, void *k_scales, void *cuda_stream);

/* One fused decode step (selector + computer + split merge, one launch).
 *
 * Selector (skipped when delta == +INFINITY):
 *   per (b, query head h, block j): p_c = q_c * s_{j,c} (fp32),
 *   a = max_c |p_c|, qi_c = clamp(rint_even(p_c * (127 / a)), -127, 127) (int8),
 *   cf = (a / 127) * (1 / sqrt(128)); I_t = sum_c qi_c * code_{t,c} (exact int),
 *   score_j = float(max over valid t of I_t) * cf   (a == 0 gives score 0).
 *   Blocks are cut into splits of S consecutive blocks (split s holds blocks
 *   [sS, min((s+1)S, nb))); inside a split, in ascending order,
 *   m = max(m, score_j) and block j is kept for head h iff score_j >= m - delta
 *   (Methodology 2, Mechanism, with the running maximum of the split as the
 *   reference: no synchronisation across splits).  A kv-head keeps the union
 *   over its G query heads; delta is in natural-log logit units (after
 *   1/sqrt(D)), delta = 0 keeps running-maximum records only, and the first
 *   block of every split is always kept.
 * Computer: every query head of the group attends (softmax(q.K/sqrt(D)) V,
 *   fp32 accumulation, bf16 output) over the valid tokens of the kept blocks;
 *   splits are merged with log-sum-exp.  delta == +INFINITY is dense
 *   flash-decoding over all valid tokens (k_packed, k_scales may be NULL).
 *
 * A sequence with lengths[b] == 0 yields zero output rows and an empty mask.
 * lengths[b] outside [0, cap] sets FFD_DEVICE_FLAG_BAD_LENGTH in the
 * workspace and yields zero rows and an empty mask for that sequence.
 * Steps that share a workspace must not overlap on the GPU. */
ffd_status ffd_decode(const ffd_shape *shape, const void *q_bf16, const void *k_bf16,
                      const void *v_bf16, const void *k_packed, const void *k_scales,
                      const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                      void *workspace, size_t workspace_bytes, void *cuda_stream);

/* The whole decode step in one launch: re-quantise each sequence's last key
 * block (exactly ffd_quantize_keys with FFD_LAST_BLOCK: the caller has just
 * appended the current token's K/V at position lengths[b] - 1), then run
 * ffd_decode.  The CTA that owns a sequence's last split does the
 * re-quantisation while its scan streams the split's other blocks; only its
 * own copies of that block wait for it, and no other CTA waits at all.
 * k_packed and k_scales are read and (for the last block) written; they are
 * required even when delta == +INFINITY.  Results are bit-identical to the
 * two calls in sequence. */
ffd_status ffd_decode_step(const ffd_shape *shape, const void *q_bf16, const void *k_bf16,
                           const void *v_bf16, void *k_packed, void *k_scales,
                           const int32_t *d_lengths, float delta, void *out_bf16, uint32_t *mask,
                           void *workspace, size_t workspace_bytes, void *cuda_stream);

/* Reference maximum of the Top-delta filter. */
#define FFD_REFERENCE_RUNNING_MAX 0       /* running max inside each split (default) */
#define FFD_REFERENCE_SINK_LOCAL 1        /* running max started at the sink/local pseudo-max */
#define FFD_REFERENCE_SINK_LOCAL_FIXED 2  /* the sink/local pseudo-max as a fixed threshold */

typedef struct {
  /* FFD_REFERENCE_RUNNING_MAX: each split's running maximum starts at -inf
   *   (the first block of every split is kept).
   * FFD_REFERENCE_SINK_LOCAL_FIXED: the rule of gist.science explainer,
   *   Methodology 2 "Mechanism" with the pseudo-max of "Pseudo-Max
   *   Approximation" (estimated from the sink tokens and the local tokens
   *   only).  Per query head, mt = max(score of block 0, score of block
   *   nb - 1), and block j is kept iff score_j >= mt - delta: one threshold
   *   for the whole sequence, so the split size does not change the mask.
   *   Every block at or above mt is kept; a split may keep nothing.
   * FFD_REFERENCE_SINK_LOCAL: a seeded variant -- each split's running
   *   maximum starts at mt and keeps rising inside the split as under
   *   FFD_REFERENCE_RUNNING_MAX; it keeps a subset of the fixed rule's
   *   blocks and the head's highest-scoring block is always kept.
   * In both pseudo-max modes every split still decides on its own (each CTA
   * scores the sink and local blocks itself); a split may keep nothing. */
  int32_t reference;
  /* 1: re-quantise each sequence's last block first, as ffd_decode_step. */
  int32_t requant_last;
  /* Longest wait, in microseconds, of any pipeline barrier or selection-queue
   * wait inside the kernel; a wait that runs out sets FFD_DEVICE_FLAG_TIMEOUT
   * and the kernel finishes without a valid result (ffd_check_device_status
   * then returns FFD_ERR_TIMEOUT).  0: the default of 2 s; negative values
   * are rejected.  The kernel's waits for its own copies still in flight use
   * the default in every case. */
  int32_t wait_limit_us;
} ffd_decode_options;

/* ffd_decode / ffd_decode_step with options (NULL is rejected).  k_packed
 * and k_scales are written only when requant_last == 1. */
ffd_status ffd_decode_ex(const ffd_shape *shape, const ffd_decode_options *options,
                         const void *q_bf16, const void *k_bf16, const void *v_bf16, void *k_packed,
                         void *k_scales, const int32_t *d_lengths, float delta, void *out_bf16,
                         uint32_t *mask, void *workspace, size_t workspace_bytes, void *cuda_stream);

/* ---- The pages' own key format: 2-bit thumbnails + 8-bit residuals ----
 * gist.science explainer, Methodology 1: the K cache is split into 2-bit
 * quantised thumbnails, scanned to estimate scores, and 8-bit residuals that
 * with the thumbnails reconstruct the keys to near-16-bit precision for the
 * exact computation (Methodology 3, "Fine-Grained Refinement": kept blocks
 * load residuals and values).  The computer then never reads bf16 K: per
 * token it reads 32 thumbnail + 128 residual + 256 V bytes instead of 64
 * int4 + 256 K + 256 V bytes. */

/* Bytes of k_thumb and k_resid for the whole batch (k_scales: ffd_scale_bytes).
 * 0 for an invalid shape. */
size_t ffd_thumb_bytes(const ffd_shape *shape);
size_t ffd_residual_bytes(const ffd_shape *shape);

/* Thumbnail + residual copy of the keys, for the same blocks as
 * ffd_quantize_keys (block_begin, FFD_LAST_BLOCK).  Per (block, channel) over
 * the block's valid tokens t:
 *   amax_c = max_t |k[t][c]|,  s_c = bf16_rne(amax_c / 1.5)   (IEEE fp32 division)
 *   y = k / s_c,  u = clamp(floor(y) + 2, 0, 3)   (level (u - 1.5) s_c)
 *   e = clamp(rint_even((y - (u - 1.5)) * 254), -127, 127)   (fp32, one rounding per step)
 *   s_c == 0 gives u = 2, e = 0; tokens at or past lengths[b] in the last
 *   block are zero bytes (thumbnail and residual) and do not enter amax.
 * The computer's key is k_hat = s_c (254 u - 381 + e) / 254, within s_c / 508
 * of k (a 10-bit grid over the block's range). */
ffd_status ffd_quantize_keys_tr(const ffd_shape *shape, const void *k_bf16,
                                const int32_t *d_lengths, int32_t block_begin, void *k_thumb,
                                void *k_resid, void *k_scales, void *cuda_stream);

/* One fused decode step on the thumbnail + residual format.
 * Selector (skipped when delta == +INFINITY): the int8 query fold of
 *   ffd_decode, then I_t = sum_c qi_c (2 u_{t,c} - 3) (exact int; the level of
 *   code u is (2u - 3) s / 2) and score_j = float(max over valid t of I_t) *
 *   ((a / 254) * (1 / sqrt(128))); Top-delta and the group union exactly as
 *   ffd_decode_ex (options->reference).
 * Computer: every query head of the group attends over the kept blocks' valid
 *   tokens with the reconstructed keys k_hat (f16 tensor-core products of the
 *   integer codes z = 254 u - 381 + e with the query folded by s / 254, fp32
 *   accumulation) and bf16 V; splits merged with log-sum-exp; bf16 output.
 * options: NULL is rejected; requant_last == 1 first re-quantises each
 *   sequence's last block from k_bf16 (bit-identical to ffd_quantize_keys_tr
 *   with FFD_LAST_BLOCK), writing k_thumb, k_resid, k_scales.  k_bf16 is read
 *   only then and may be NULL when requant_last == 0.
 * Length handling, workspace and errors as ffd_decode. */
ffd_status ffd_decode_tr(const ffd_shape *shape, const ffd_decode_options *options,
                         const void *q_bf16, const void *k_bf16, const void *v_bf16, void *k_thumb,
                         void *k_resid, void *k_scales, const int32_t *d_lengths, float delta,
                         void *out_bf16, uint32_t *mask, void *workspace, size_t workspace_bytes,
                         void *cuda_stream);

/* ---- The decode step with the KV append fused in ----
 * One launch per decode step for callers that hold the new token's K and V
 * rows (k_new, v_new: bf16 [B][Hkv][D]) rather than an already appended
 * cache: the CTA that owns each sequence's last block writes the two rows
 * into k and v at position lengths[b] - 1 (lengths[b] counts the new token),
 * re-quantises that block and runs the decode; every CTA that reads the new
 * token takes it from k_new, so nothing waits on another CTA.  Equivalent to
 * storing the rows, then ffd_decode_step (or ffd_decode_ex with requant_last
 * and `reference`; ffd_decode_tr for the _tr form); the results are
 * bit-identical.  The step of the pages' system part (gist.science explainer,
 * Methodology 3: the decoding step captured whole in a CUDA graph) keeps one
 * kernel per layer this way.  reference: FFD_REFERENCE_*.  A sequence of
 * length 0 appends nothing.  Other arguments and errors as ffd_decode_ex and
 * ffd_decode_tr. */
ffd_status ffd_decode_append(const ffd_shape *shape, int32_t reference, const void *q_bf16,
                             const void *k_new_bf16, const void *v_new_bf16, void *k_bf16,
                             void *v_bf16, void *k_packed, void *k_scales,
                             const int32_t *d_lengths, float delta, void *out_bf16,
                             uint32_t *mask, void *workspace, size_t workspace_bytes,
                             void *cuda_stream);
ffd_status ffd_decode_append_tr(const ffd_shape *shape, int32_t reference, const void *q_bf16,
                                const void *k_new_bf16, const void *v_new_bf16, void *k_bf16,
                                void *v_bf16, void *k_thumb, void *k_resid, void *k_scales,
                                const int32_t *d_lengths, float delta, void *out_bf16,
                                uint32_t *mask, void *workspace, size_t workspace_bytes,
                                void *cuda_stream);

/* ---- One layer's whole decode step as a native CUDA graph ----
 * gist.science explainer, Methodology 3: the decoding step is captured whole in
 * a CUDA graph, so a small batch pays no CPU launch overhead.  The graph
 * (captured here on a private stream, nothing is executed at creation) holds:
 *   1. the H2D copy of host_in -> dev_in, both laid out as
 *      q bf16 [B][Hq][D] | k_new bf16 [B][Hkv][D] | v_new bf16 [B][Hkv][D]
 *      (host_in must be pinned host memory);
 *   2. when advance == 1, lengths[b] += 1 for every sequence;
 *   3. ffd_decode_append (format 0: k_copy = k_packed, k_resid unused) or
 *      ffd_decode_append_tr (format 1: k_copy = k_thumb), writing the output
 *      rows at dev_result and the mask at dev_result + mask_offset (a
 *      multiple of 16, at least B*Hq*D*2 bytes);
 *   4. the D2H copy of dev_result (mask_offset + 4 * ffd_mask_words bytes) to
 *      host_result (pinned).  With dev_result == NULL the kernel writes the
 *      results straight into host_result, which must then be pinned host
 *      memory mapped into the device address space (the default for pinned
 *      memory under unified addressing), and the graph has no D2H node.
 * ffd_step_graph_run launches it and waits for it on the graph's stream: a
 * decode step from host inputs to host outputs in one call.  All buffers stay
 * caller-owned and must outlive the graph; the caller orders its own earlier
 * device work (cache prefill, quantisation) before the first run, e.g. with a
 * device synchronisation.  This object is the one place the library keeps
 * state: a stream, a graph and its executable, released by
 * ffd_step_graph_destroy.  Argument checks as ffd_decode_append; a failure
 * returns a status and no graph. */
typedef struct ffd_step_graph ffd_step_graph;
ffd_status ffd_step_graph_create(const ffd_shape *shape, int32_t format, int32_t reference,
                                 float delta, int32_t advance, const void *host_in, void *dev_in,
                                 void *k_bf16, void *v_bf16, void *k_copy, void *k_resid,
                                 void *k_scales, int32_t *d_lengths, void *dev_result,
                                 void *host_result, size_t mask_offset, void *workspace,
                                 size_t workspace_bytes, ffd_step_graph **graph_out);
ffd_status ffd_step_graph_run(ffd_step_graph *graph);
void ffd_step_graph_destroy(ffd_step_graph *graph);

/* Context (sequence) sharding across GPUs.  Each rank holds a contiguous
 * shard of every sequence's cache: rank r holds global tokens
 * [r * cap_local, (r + 1) * cap_local) in a cache of capacity cap_local, with
 * cap_local a multiple of block_size * split_blocks so that every split lies
 * in one shard and its Top-delta selection is exactly the unsharded one
 * (running-max reference only: the pseudo-max needs the sink and local blocks
 * of other shards).  Steps per decode step:
 *   1. ffd_decode_partials on every rank with the LOCAL shape and the local
 *      lengths clip(len - r * cap_local, 0, cap_local): writes the shard's
 *      split partials and selection bits into its workspace (no merge, no
 *      output);
 *   2. all-gather the workspace region named by ffd_partials_region (same
 *      offset and size on every rank) into num_shards consecutive regions;
 *   3. ffd_merge_partials with the global lengths: the log-sum-exp merge over
 *      every split of every shard, writing out [B][Hq][D] and the mask over the
 *      global capacity num_shards * cap_local ([B][Hkv][ceil(nblk_global/32)]).
 * Both kernels are the flash-decoding split merge stretched across GPUs; the
 * exchange moves B * Hkv * nsplit * G * 528 bytes plus the bits per rank. */
ffd_status ffd_decode_partials(const ffd_shape *local_shape, const ffd_decode_options *options,
                               const void *q_bf16, const void *k_bf16, const void *v_bf16,
                               void *k_packed, void *k_scales, const int32_t *d_local_lengths,
                               float delta, void *workspace, size_t workspace_bytes,
                               void *cuda_stream);
/* ffd_decode_partials on the thumbnail + residual format (arguments as
 * ffd_decode_tr); the exchange and ffd_merge_partials are unchanged. */
ffd_status ffd_decode_partials_tr(const ffd_shape *local_shape, const ffd_decode_options *options,
                                  const void *q_bf16, const void *k_bf16, const void *v_bf16,
                                  void *k_thumb, void *k_resid, void *k_scales,
                                  const int32_t *d_local_lengths, float delta, void *workspace,
                                  size_t workspace_bytes, void *cuda_stream);
ffd_status ffd_partials_region(const ffd_shape *local_shape, size_t *offset, size_t *bytes);
ffd_status ffd_merge_partials(const ffd_shape *local_shape, int32_t num_shards, const void *gathered,
                              size_t gathered_bytes, const int32_t *d_global_lengths,
                              void *out_bf16, uint32_t *mask, void *cuda_stream);

/* ffd_decode without a caller workspace, for callers that cannot allocate
 * device memory: e.g. a plug-in inside an inference engine that is given only
 * its input and output buffers, or a serving loop that must not call
 * cudaMalloc once running (an allocation can synchronise the whole device).
 * The paper has no counterpart to this entry point; it is a deployment aid.
 *
 * Same arguments and results as ffd_decode, minus the workspace.  The kernel's
 * scratch lives in a fixed 16 MiB device array inside this library, held on
 * every GPU that loads the library until the process exits; this call
 * allocates nothing.  Shapes whose ffd_decode_workspace_bytes exceeds
 * 16 MiB (16777216 bytes) return FFD_ERR_WORKSPACE before any launch.
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it, so make that first call before any stream
 * capture.  Every call that passes its host checks clears the array's
 * counters and error word on the stream just before its launch (a rejected
 * call writes nothing); the array is shared by all calls on a device and
 * keeps the last call's contents, so calls that overlap on the GPU race and
 * must be serialised by the caller.  Device-side errors are reported by
 * ffd_no_alloc_device_status: a length outside [0, cap] (zero rows and an
 * empty mask for that sequence), or a bounded wait that ran out (the output
 * is then not valid).  Outside a stream capture each call looks the array's
 * address up again, so it stays right after a device reset; inside a capture
 * the address from the last call outside it is used. */
ffd_status ffd_decode_no_alloc(const ffd_shape *shape, const void *q_bf16, const void *k_bf16,
                               const void *v_bf16, const void *k_packed, const void *k_scales,
                               const int32_t *d_lengths, float delta, void *out_bf16,
                               uint32_t *mask, void *cuda_stream);

/* The error word of ffd_decode_no_alloc's built-in array on the current
 * device, as ffd_check_device_status reads a workspace's: synchronise the
 * stream, read the flags the last ffd_decode_no_alloc call on this device
 * left and clear them.  Call it after that call and before the next one.
 * Returns FFD_ERR_TIMEOUT if FFD_DEVICE_FLAG_TIMEOUT was set (that call's
 * output is not valid), FFD_ERR_DEVICE_CHECK for any other flag,
 * FFD_ERR_INVALID_ARG while the stream is being captured.  Allocates
 * nothing; the paper has no counterpart. */
ffd_status ffd_no_alloc_device_status(uint32_t *flags_out, void *cuda_stream);

/* Synchronise the stream, read and clear the workspace's sticky device error
 * word.  *flags_out (may be NULL) receives FFD_DEVICE_FLAG_* bits.  Returns
 * FFD_ERR_TIMEOUT if FFD_DEVICE_FLAG_TIMEOUT was set, else
 * FFD_ERR_DEVICE_CHECK if any other flag was, FFD_ERR_CUDA on a CUDA error. */
ffd_status ffd_check_device_status(void *workspace, uint32_t *flags_out, void *cuda_stream);

/* Static description of a status code. */
const char *ffd_status_string(ffd_status status);

/* ABI version of this library (bumped on any incompatible change). */
int32_t ffd_abi_version(void);

/* Streaming-read bandwidth probe (not part of the method; a reference point
 * for the decode kernel's roofline, which is a one-pass read of HBM).  Reads
 * `bytes` of device memory at `buf` once with 16-byte loads that do not
 * allocate in L1, on `cuda_stream`; time it with events around the call.
 * `sink` (device, one uint32) is written only if the data fold to a fixed
 * constant, so that no load can be elided.  buf must be 16-byte aligned and
 * bytes a non-zero multiple of 16 (else FFD_ERR_INVALID_ARG, nothing
 * launched).  Use a buffer well above the 126 MB L2 to measure HBM. */
ffd_status ffd_read_probe(const void *buf, size_t bytes, uint32_t *sink, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* FFD_H */
