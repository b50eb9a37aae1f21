/*
 * fa.h -- C ABI of the B200 (sm_100a) exact tiled attention library (libfa_sm100.so).
 *
 * What it computes.  O = softmax(scale * Q K^T + mask) V for every (batch, head), together with the
 * per-row natural log-sum-exp LSE_i = ln sum_j exp(scale * q_i . k_j) over the visible keys j.  The
 * three steps of standard attention (scores, row softmax, product with V) are those of the Ascend
 * CANN ops-transformer FlashAttention article (zskr.cn), section "背景"; the tiled evaluation with a
 * running row max m and running row sum l is its section "原理" (steps 1-4).  The result is exact
 * attention, not an approximation ("Was FlashAttention bei Transformer-Inference verändert"): the
 * N x N matrices S and P never leave the chip and are never returned (output_attentions has no
 * counterpart, as in the parameter table of "如何为 Hugging Face Transformers 更多架构添加 Flash
 * Attention 2 支持？").
 *
 * Conventions shared by every entry point:
 *   - Pointers named q, k, v, o, k_cache, v_cache, lse, cu_seqlens and workspace are DEVICE
 *     pointers of the current CUDA device.  The caller owns every buffer; the library never
 *     allocates, frees or synchronises.  All work is enqueued on `stream` (0 = legacy default
 *     stream) and runs asynchronously.
 *   - Q/K/V/O layout is [B, N, H, D], row-major and contiguous (the layout of the tiling sketch in
 *     the Ascend article, section "代码讲解").  Element types: FA_BF16 or FA_FP16 inputs; the
 *     output O is either the input type or FA_FP32.  LSE is always fp32.
 *   - Head dimension D must be 64 or 128 (the Hugging Face page asks for a head_dim of at least 64
 *     that is a multiple of 64 / a power of two; these are the two sizes the kernels implement).
 *   - fp32/fp64 inputs are rejected with FA_ERR_DTYPE (Hugging Face page, "常见错误排查", error 1).
 *   - Only sm_100 devices (B200) are accepted; anything else returns FA_ERR_DEVICE (same page,
 *     error 3, states the GPU-generation gate).
 *   - Every argument is validated before anything is launched; on error nothing is enqueued and the
 *     status code is returned.  No entry point aborts, throws or prints.
 *   - Device-side failures (a bounded wait inside a kernel that ran out) are recorded in a device
 *     status word that fa_device_status() reads.
 *   - Per-device set-up (the status word's address, raised shared-memory limits) is done once per
 *     CUDA context and redone when the device's context changes (for example after cudaDeviceReset).
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                     /* the same type as cudaStream_t */
typedef struct CUstream_st* fa_stream_t;

typedef enum { FA_BF16 = 0, FA_FP16 = 1, FA_FP32 = 2 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = 1,        /* a required pointer is NULL                                      */
  FA_ERR_DTYPE = 2,       /* input not bf16/fp16, or output type not (input type | fp32)      */
  FA_ERR_HEADDIM = 3,     /* D not in {64, 128}                                               */
  FA_ERR_SHAPE = 4,       /* B, H, Nq, Nk, num_splits out of range, or scale not finite > 0   */
  FA_ERR_ALIGN = 5,       /* a tensor pointer is not 16-byte aligned (lse: 4-byte)            */
  FA_ERR_CU_SEQLENS = 6,  /* cu_seqlens / seqlens_k out of range (device-detected)              */
  FA_ERR_WORKSPACE = 7,   /* decode workspace missing or smaller than required                */
  FA_ERR_DEVICE = 8,      /* no CUDA device, or the current device is not sm_100             */
  FA_ERR_LAUNCH = 9,      /* a CUDA launch or driver call failed                              */
  FA_ERR_TIMEOUT = 10,    /* a bounded wait inside a kernel ran out (device-detected)         */
  FA_ERR_BOUNDS = 11,     /* debug builds only: an index check caught an access outside its
                             buffer (device-detected; the access was skipped)                  */
  FA_ERR_PAGE_TABLE = 12  /* a paged-cache block-table entry names no pool page
                             (device-detected; see fa_decode_splitkv_paged)                     */
} fa_status;

/*
 * fa_fwd -- attention forward pass over many queries (prefill / encoder).
 *
 * Passage: Ascend article sections "原理" (tiling, online softmax with m and l) and "代码讲解"
 * (outer loop over query blocks, inner loop over key/value blocks); the mask kinds of the Hugging
 * Face page ("原因分析" item 1: causal and bidirectional; "常见错误排查" error 4: the 2-D key
 * padding mask) and its varlen variant (FAQ 4, flash_attn_varlen).
 *
 * Dense mode (cu_seqlens == NULL):
 *   q [B, Nq, H, D], k and v [B, Nk, H, D], o [B, Nq, H, D] of type o_dtype, lse [B, H, Nq].
 * Varlen mode (cu_seqlens != NULL): B sequences packed back to back,
 *   q, k, v, o [total, H, D] with total = Nq = Nk (the packed row extent of the buffers);
 *   cu_seqlens: device int32[B + 1], cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = total;
 *   sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 and its queries see exactly its own
 *   keys (self-attention: one cu_seqlens for Q and K); lse [H, total].  The kernels never touch a
 *   row outside [0, total).  A cu_seqlens that is not non-decreasing or ends above total is
 *   detected on the device: its tiles are skipped and the device status becomes FA_ERR_CU_SEQLENS.
 * causal != 0: query i (0-based within its sequence) sees key j iff j <= i + (Nk_b - Nq_b),
 *   i.e. the lower triangle aligned at the bottom-right corner; with Nq_b = Nk_b this is j <= i.
 *   A query that sees no key gets O = 0 and LSE = -inf.
 * scale: the softmax scale, finite and > 0 (callers wanting the default pass 1/sqrt(D)).
 * in_dtype: FA_BF16 or FA_FP16; o_dtype: in_dtype or FA_FP32.
 * Limits: 1 <= B, 1 <= H, 1 <= Nq, Nk <= 2^24 rows per batch item (dense) or packed (varlen);
 *   B * Nq and B * Nk below 2^31.
 * Returns FA_OK or an fa_status error code; see the conventions above.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int Nq, int Nk, int D, float scale, int causal,
           const int* cu_seqlens, fa_stream_t stream, int in_dtype, int o_dtype);

/*
 * fa_fwd_prefix -- fa_fwd with the prefix mask: causal, except that the first prefix_len keys of each
 * sequence are visible to every query of it (bidirectional attention over a prefix, causal after).
 *
 * Passage: the Hugging Face page, "原因分析" item 1, names the prefix mask (前缀掩码) next to the causal
 * and bidirectional masks without defining it; the reading implemented is the prefix-LM mask:
 * query i sees key j iff j < prefix_len or j <= i + (Nk_b - Nq_b).  prefix_len = 0 gives exactly
 * fa_fwd(..., causal = 1, ...); prefix_len >= Nk gives the unmasked result.
 *
 * Arguments, layouts, ownership, limits and errors as fa_fwd (causal is implied), plus
 * prefix_len >= 0 (negative -> FA_ERR_SHAPE).  In varlen mode the prefix is counted from the first
 * key of every sequence.
 */
int fa_fwd_prefix(const void* q, const void* k, const void* v, void* o, float* lse,
                  int B, int H, int Nq, int Nk, int D, float scale, int prefix_len,
                  const int* cu_seqlens, fa_stream_t stream, int in_dtype, int o_dtype);

/*
 * fa_bwd_workspace_bytes -- size of the scratch buffer fa_bwd needs: B * H * Nq * 4 bytes (one fp32
 * row term per query), rounded up to 256 bytes.  Returns 0 for invalid arguments.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int Nq);

/*
 * fa_bwd -- gradients dQ, dK, dV of the attention forward pass (dense layout).
 *
 * Passage: "轻松读懂FlashAttention 上", end of section "Softmax求解重构": keeping O and the softmax
 * statistics lets the backward pass recompute S and P instead of storing them; the Hugging Face
 * page's parameter table (row training) ties training mode to gradient computation.  The gradients
 * are the derivative of fa_fwd's definition for an upstream gradient dO of L = sum(dO * O):
 * dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)), dQ = scale dS K, dK = scale dS^T Q, with P
 * recomputed from Q, K and the forward LSE.
 *
 * q, o, dout [B, Nq, H, D] and k, v [B, Nk, H, D] of in_dtype (FA_BF16 / FA_FP16); lse [B, H, Nq]
 * fp32 as written by fa_fwd with the same q, k, v, scale and causal; dq [B, Nq, H, D] and dk, dv
 * [B, Nk, H, D] of grad_dtype (in_dtype or FA_FP32), fully overwritten.  causal as fa_fwd
 * (bottom-right aligned).  workspace: device buffer of at least fa_bwd_workspace_bytes(B, H, Nq)
 * bytes, owned by the caller, 16-byte aligned.  The prefix-mask and varlen forms are
 * fa_bwd_masked.  Limits and errors as fa_fwd (FA_ERR_WORKSPACE for a missing or short workspace).
 * A query row with LSE = -inf (no visible key) contributes nothing.  Three kernels run in order on
 * `stream`; nothing is allocated.  Same as fa_bwd_masked with prefix_len = 0, cu_seqlens = NULL.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int D, float scale, int causal,
           void* workspace, size_t workspace_bytes, fa_stream_t stream, int in_dtype, int grad_dtype);

/*
 * fa_bwd_masked -- gradients of every forward form: the backward of fa_fwd (dense or packed
 * varlen, causal or not) and of fa_fwd_prefix.
 *
 * Passages: those of fa_bwd for the gradients; the masks are the forward's (causal, bottom-right
 * aligned; the prefix-LM mask of fa_fwd_prefix, where prefix_len > 0 makes the first prefix_len keys
 * of each sequence visible to all its queries and implies causal); the varlen layout is that of
 * fa_fwd with cu_seqlens (Hugging Face page, FAQ 4 and "常见错误排查", error 4).
 *
 * Dense (cu_seqlens == NULL): layouts and lse as fa_bwd.  Varlen (cu_seqlens != NULL, int32[B + 1]
 * on the device, as given to fa_fwd): q, k, v, o, dout, dq, dk, dv are packed [total, H, D] with
 * Nq = Nk = total, lse is [H, total] as fa_fwd wrote it, and the workspace needs
 * fa_bwd_workspace_bytes(1, H, total) bytes.  lse must come from the forward call with the same
 * inputs, scale and mask.  Errors as fa_bwd, plus FA_ERR_SHAPE for prefix_len < 0 or Nq != Nk with
 * cu_seqlens, FA_ERR_ALIGN for a misaligned cu_seqlens; an inconsistent cu_seqlens is reported on
 * the device as FA_ERR_CU_SEQLENS (fa_device_status) and its tiles are skipped.
 */
int fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int D, float scale, int causal,
                  int prefix_len, const int* cu_seqlens, void* workspace, size_t workspace_bytes,
                  fa_stream_t stream, int in_dtype, int grad_dtype);

/*
 * fa_decode_workspace_bytes -- size of the scratch buffer fa_decode_splitkv needs:
 * num_splits * B * H * (D + 1) * 4 bytes (one fp32 partial output row and one fp32 partial LSE per
 * split), rounded up to 256 bytes.  Returns 0 for invalid arguments.
 */
size_t fa_decode_workspace_bytes(int B, int H, int D, int num_splits);

/*
 * fa_decode_splitkv -- single-token decode over a KV cache with split-KV and an LSE combine.
 *
 * Passage: "Was FlashAttention bei Transformer-Inference verändert" (prefill versus decode of a
 * single token differ in the parallel work available; the cache layout question), and the merge of
 * per-group softmax statistics of "轻松读懂FlashAttention 上", section "Softmax求解重构", which is
 * exactly how the per-split partial results are combined.
 *
 * q [B, 1, H, D]; k_cache, v_cache [B, Nk, H, D]; o [B, 1, H, D] of type o_dtype; lse [B, H].
 * The query attends to all Nk cached keys (no mask).  The keys are cut into ranges of
 * max(ceil(Nk / num_splits), 512) keys (at most num_splits of them; fewer when the cache is short);
 * a first kernel writes each range's normalised partial output and partial LSE to `workspace`, a
 * second kernel merges them.  1 <= num_splits <= 128.
 * workspace: device buffer of at least fa_decode_workspace_bytes(B, H, D, num_splits) bytes, owned
 * by the caller, 16-byte aligned; its contents on entry are irrelevant.
 * Returns FA_OK or an fa_status error code.
 */
int fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                      int B, int H, int Nk, int D, float scale, int num_splits,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream,
                      int in_dtype, int o_dtype);

/*
 * fa_decode_splitkv_gqa -- fa_decode_splitkv with grouped KV heads and per-sequence cache lengths.
 *
 * Passage: as fa_decode_splitkv.  "Was FlashAttention bei Transformer-Inference verändert" asks
 * whether a backend supports the cache layout without fixing one; this entry point takes the
 * common layout with fewer KV heads than query heads and a valid length per sequence.
 *
 * q [B, 1, Hq, D]; k_cache, v_cache [B, Nk, Hkv, D] (Nk = cache capacity); o [B, 1, Hq, D] of type
 * o_dtype; lse [B, Hq].  Hq must be a multiple of Hkv (else FA_ERR_SHAPE); query head h reads KV
 * head h / (Hq / Hkv).  seqlens_k: device int32[B] (4-byte aligned) or NULL; the query of batch
 * item b attends to cached keys [0, seqlens_k[b]) (all Nk when NULL).  A length of 0 gives O = 0 and
 * LSE = -inf; a length outside [0, Nk] is detected on the device, treated as 0, and sets the device
 * status to FA_ERR_CU_SEQLENS.  Each KV row is read once for all query heads of its group (up to 16
 * per CTA; groups of 2 or more heads run on the tensor cores).  workspace: at least
 * fa_decode_workspace_bytes(B, Hq, D, num_splits) bytes.  Other
 * arguments, ownership and errors as fa_decode_splitkv; with Hkv = Hq and seqlens_k = NULL the
 * result equals fa_decode_splitkv's.
 */
int fa_decode_splitkv_gqa(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                          int B, int Hq, int Hkv, int Nk, int D, float scale, int num_splits,
                          const int* seqlens_k, void* workspace, size_t workspace_bytes,
                          fa_stream_t stream, int in_dtype, int o_dtype);

/*
 * fa_decode_splitkv_paged -- fa_decode_splitkv_gqa over a paged cache: a pool of fixed-size pages
 * of cache rows and a per-sequence table of page indices.
 *
 * Passage: as fa_decode_splitkv_gqa ("Was FlashAttention bei Transformer-Inference verändert":
 * whether a backend supports the cache layout).  A page pool read through a block table is the
 * layout a serving runtime gets when it grows each sequence's cache by whole pages; it changes
 * where each key row is read from, not what is computed.
 *
 * k_pages, v_pages [num_pages, page_size, Hkv, D] (16-byte aligned); row r of page p is one key.
 * block_table: device int32 [B, pages_per_seq] (4-byte aligned), row-major; entry (b, i) is the page
 * holding keys [i * page_size, (i + 1) * page_size) of batch item b.  seqlens_k: device int32[B] or
 * NULL: batch item b sees its first seqlens_k[b] keys (all pages_per_seq * page_size when NULL);
 * only the first ceil(seqlens_k[b] / page_size) entries of its table row are read, and nothing of a
 * page beyond the valid keys reaches the result (it may hold anything, NaN included).
 * page_size: a power of two, 16 <= page_size <= 65536; num_pages * page_size, pages_per_seq *
 * page_size and B * pages_per_seq below 2^31 (else FA_ERR_SHAPE).  q, o, lse, workspace, num_splits,
 * dtypes: as fa_decode_splitkv_gqa, with Nk = pages_per_seq * page_size (split ranges are rounded to
 * whole 64-key tiles).  Errors as fa_decode_splitkv_gqa, plus FA_ERR_NULL for a NULL block_table and
 * FA_ERR_ALIGN for a misaligned one.  A table entry outside [0, num_pages) that a batch item needs is
 * detected on the device: nothing outside the pool is read, the split-KV range holding it
 * contributes nothing (so that item's O and LSE are not meaningful) and the device status becomes
 * FA_ERR_PAGE_TABLE.  The function computed is fa_decode_splitkv_gqa's over the rows gathered in
 * table order.
 */
int fa_decode_splitkv_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                            void* o, float* lse, int B, int Hq, int Hkv, int num_pages, int page_size,
                            int pages_per_seq, int D, float scale, int num_splits, const int* seqlens_k,
                            void* workspace, size_t workspace_bytes, fa_stream_t stream, int in_dtype,
                            int o_dtype);

/*
 * fa_decode_part_bytes -- size of one key shard's partial decode result (see
 * fa_decode_splitkv_shard): O [B, H, D] fp32 followed by LSE [B, H] fp32, padded to a multiple of
 * 16 bytes.  R shards' results laid end to end at this stride form the input of fa_decode_merge.
 * Returns 0 for invalid arguments.
 */
size_t fa_decode_part_bytes(int B, int H, int D);

/*
 * fa_decode_splitkv_shard -- single-token decode over ONE key shard of a cache cut along the key
 * axis (one shard per GPU), leaving the shard's partial result for fa_decode_merge.
 *
 * Passage: "轻松读懂FlashAttention 上", section "内存卡点" (contexts of 64k to 128k tokens and more,
 * far beyond on-chip memory), and the merge of per-group softmax statistics of its section
 * "Softmax求解重构": a shard's normalised output and LSE are the statistics of one key group, so
 * the merge of all shards' results is the softmax over the whole cache.
 *
 * The shard holds keys [key_offset, key_offset + Nk_shard) of a cache of Nk_total keys:
 * k_shard, v_shard [B, Nk_shard, Hkv, D] (row j is key key_offset + j).  q [B, 1, Hq, D].
 * seqlens_k: device int32[B] or NULL, valid lengths of the WHOLE cache (NULL: Nk_total); the shard
 * attends to its keys below seqlens_k[b].  A length outside [0, Nk_total] is detected on the device,
 * treated as 0, and sets the device status to FA_ERR_CU_SEQLENS.  Requires 0 <= key_offset and
 * key_offset + Nk_shard <= Nk_total (else FA_ERR_SHAPE).
 * part: device buffer of fa_decode_part_bytes(B, Hq, D) bytes, 16-byte aligned, owned by the
 * caller; receives the shard's fp32 O (normalised over the shard's keys; 0 where it has none) and
 * natural-log LSE (-inf where it has none).  The split-KV kernels of fa_decode_splitkv_gqa run on
 * the shard with `workspace` (at least fa_decode_workspace_bytes(B, Hq, D, num_splits) bytes).
 * Other arguments, limits and errors as fa_decode_splitkv_gqa.
 */
int fa_decode_splitkv_shard(const void* q, const void* k_shard, const void* v_shard, float* part, int B,
                            int Hq, int Hkv, int Nk_shard, int key_offset, int Nk_total, int D, float scale,
                            int num_splits, const int* seqlens_k, void* workspace, size_t workspace_bytes,
                            fa_stream_t stream, int in_dtype);

/*
 * fa_decode_merge -- merge R key shards' partial decode results into the output of the whole cache.
 *
 * Passage: "轻松读懂FlashAttention 上", section "Softmax求解重构" (merge of group statistics),
 * applied to R groups at once: with M = max_r LSE_r and w_r = exp(LSE_r - M),
 * O = sum_r w_r O_r / sum_r w_r and LSE = M + ln sum_r w_r; a row with LSE_r = -inf in every shard
 * gets O = 0, LSE = -inf.
 *
 * parts: device fp32, R blocks of fa_decode_part_bytes(B, H, D) bytes each (block r as written by
 * fa_decode_splitkv_shard for shard r, e.g. gathered from R ranks), 16-byte aligned.  The order of
 * the blocks does not matter.  o [B, 1, H, D] of o_dtype (FA_BF16, FA_FP16 or FA_FP32), 16-byte
 * aligned; lse [B, H] fp32.  1 <= R <= 65536.  One kernel on `stream`; nothing is allocated.
 * Errors: FA_ERR_NULL, FA_ERR_DTYPE (o_dtype), FA_ERR_HEADDIM, FA_ERR_SHAPE, FA_ERR_ALIGN,
 * FA_ERR_DEVICE, FA_ERR_LAUNCH.
 */
int fa_decode_merge(const float* parts, int R, int B, int H, int D, void* o, float* lse, fa_stream_t stream,
                    int o_dtype);

/*
 * fa_decode_splitkv_noalloc -- fa_decode_splitkv without a caller-provided workspace.
 *
 * The pages describe nothing like this; it exists for callers that cannot allocate device memory
 * when they call: an engine that reserves all of its memory at start-up and forbids allocation
 * afterwards, a plugin whose host framework owns the allocator, or latency-critical code that must
 * not pay for cudaMalloc (which can synchronise the device).  Arguments, layouts and results are
 * those of fa_decode_splitkv minus workspace/workspace_bytes.  The per-split partials go to a fixed
 * array of FA_NOALLOC_SCRATCH_BYTES inside the library, reserved on each GPU where the library's
 * code is first used and kept until the process exits.
 *   - Returns FA_ERR_WORKSPACE, without launching, when fa_decode_workspace_bytes(B, H, D,
 *     num_splits) exceeds FA_NOALLOC_SCRATCH_BYTES.
 *   - The first call on a device looks up the array's device address (with that device current)
 *     and caches it for that device's CUDA context; make that first call before any stream
 *     capture.  After the context is destroyed and recreated (cudaDeviceReset), the next call looks
 *     the address up again.
 *   - Its argument checks are those of fa_decode_splitkv, in the same order, with the fixed array's
 *     capacity in place of workspace_bytes.
 *   - Every call on a device shares the one array.  Nothing in it needs clearing between calls, but
 *     calls whose kernels may overlap on the GPU (unordered streams) race on it: order them.
 *   - Calls no allocating routine (no cudaMalloc / cudaFree).
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                              int B, int H, int Nk, int D, float scale, int num_splits,
                              fa_stream_t stream, int in_dtype, int o_dtype);

/*
 * fa_selftest_wait_timeout -- run the kernels' bounded wait on a barrier that nothing arrives on.
 *
 * The pages describe nothing like this; it lets a caller check, on its own GPU, that a stalled wait
 * inside this library ends with an error instead of a hang: a one-thread kernel waits with the
 * library's bounded mbarrier wait (one second without progress), which then records FA_ERR_TIMEOUT
 * in the device status word (see fa_device_status) and returns.  Takes about one second; the CUDA
 * context stays usable.  *waited_ms receives the time the wait took (milliseconds), or -1 if the
 * wait unexpectedly completed.  Synchronises `stream`; uses a mapped host word (allocates and frees
 * it).  Returns FA_OK when the kernel ran to completion (the timeout itself is reported through the
 * status word), FA_ERR_NULL, FA_ERR_DEVICE or FA_ERR_LAUNCH.
 */
int fa_selftest_wait_timeout(int* waited_ms, fa_stream_t stream);

/* fa_status_string -- static English text for a status code (never NULL). */
const char* fa_status_string(int status);

/*
 * fa_device_status -- read the device status word of the current device into *status_out
 * (FA_OK if no kernel recorded a failure) and, if clear != 0, reset it to FA_OK.  This call
 * synchronises with the device (it copies one int).  Returns FA_OK, FA_ERR_NULL, FA_ERR_DEVICE or
 * FA_ERR_LAUNCH.
 */
int fa_device_status(int* status_out, int clear);

/*
 * fa_build_flags -- how this library was built.  Bit 0 (FA_BUILD_DEBUG): a debug build
 * (libfa_sm100_debug.so): every plain global load and store of the kernels (those no TMA descriptor
 * bounds) checks its index against its buffer and, when it would leave it, skips the access and
 * records FA_ERR_BOUNDS in the device status word; the prefill kernel also walks every key block of
 * a causal or prefix-masked row instead of stopping after the last visible one, masking the rest
 * (the results are the same bit for bit).  The pages have no counterpart: this is test equipment
 * standing in for a memory checker.  Never fails.
 */
#define FA_BUILD_DEBUG 1
int fa_build_flags(void);

/* fa_abi_version -- version of this interface (incremented on any signature change). */
int fa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
