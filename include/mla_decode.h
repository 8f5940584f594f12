/*
 * mla_decode.h -- C ABI of the Blackwell (sm_100a) MLA decoding library.
 *
 * Multi-head latent attention (MLA) decoding over a paged latent KV cache, in
 * the "MQA mode" of the upstream FlashMLA documentation ("MLA Mode" footnote to
 * the support matrix): every query head attends one shared latent KV head whose
 * cached rows are d_qk = 576 wide (512 latent columns, then 64 RoPE columns) or
 * d_qk = 512 wide (no RoPE part); V is the leading d_v = 512 columns of the same
 * rows.  Cached tokens sit in 64-token pages found through a block table.
 *
 * The call sequence is the one the "FlashMLA" usage page (deepep.org) shows:
 * mla_get_metadata once per decoding step (its result is reused by every
 * layer), then mla_decode_with_kvcache once per layer, which returns (o, lse).
 *
 * Conventions for every entry point:
 *   - Pointers named "device" are CUDA device pointers; "host" ones are host memory.
 *   - The caller allocates and owns every buffer.  The library allocates no
 *     memory and keeps no state between calls (apart from a per-process cache
 *     of one CUDA driver entry point and per-device kernel attributes set on
 *     first use).
 *   - Calls taking a stream enqueue work on it and return without
 *     synchronising; results are ready when the stream reaches that point.
 *     A stream of NULL means the legacy default stream.
 *   - Invalid arguments are rejected on the host before anything is enqueued;
 *     the return value says why (mla_status_string gives a message).
 *   - Errors that only the device can see (a block-table entry outside the
 *     cache, a pipeline wait that ran out of time) are recorded in a status
 *     word at the start of the workspace; mla_read_device_status reads it.
 *     The outputs of a call that recorded one are unspecified: rows may hold
 *     anything, including what they held before (a cluster that gave up, or a
 *     combine that stopped waiting once the status word was set, writes nothing).
 *
 * Array layouts (all row-major / C order):
 *   q             [batch, s_q, h_q, d_qk]             bf16 or fp16
 *   kvcache       [num_blocks, 64, h_kv, d_qk]        same dtype as q, or, with
 *                 [num_blocks, 64, h_kv, 656] bytes   dtype MLA_BF16_FP8KV, "FP8 with scale"
 *                                                     rows (see mla_dtype)
 *   block_table   [batch, max_blocks_per_seq] int32   physical page ids; only the
 *                                                     first ceil(L_b / 64) entries
 *                                                     of row b are read
 *   cache_seqlens [batch] int32                       L_b >= 0
 *   o             [batch, s_q, h_q, 512]              same dtype as q
 *   lse           [batch, s_q, h_q] float32           natural log
 *   tile_md       [num_parts, 8] int32                scheduler output (opaque)
 *   num_splits    [batch * row_groups + 1] int32      scheduler output, prefix sums
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_PAGE_SIZE 64       /* tokens per KV-cache page ("block size of 64") */
#define MLA_HEAD_DIM_V 512     /* d_v: the latent width */
#define MLA_MD_INTS 8          /* int32 entries per row of tile_md */
#define MLA_ROWS_PER_GROUP 128 /* query rows (s_q * h_q) handled per row group */

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned buffer, ... */
    MLA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    MLA_ERR_WORKSPACE = 3,    /* workspace smaller than mla_decode_workspace_bytes */
    MLA_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
    MLA_ERR_TIMEOUT = 5,      /* device: a pipeline wait gave up (kernel returned early) */
    MLA_ERR_DEVICE_CHECK = 6  /* device: a needed block-table entry was outside [0, num_blocks),
                                 or a sequence needs more than max_blocks_per_seq pages */
} mla_status;

/*
 * Data types of a call.  MLA_BF16 / MLA_FP16: q, kvcache and o all of that type.
 * MLA_BF16_FP8KV: q and o bfloat16, kvcache in the "FP8 with scale" format of the
 * upstream FlashMLA documentation ("FP8 KV Cache" section): each token row is 656
 * bytes, 512 float8_e4m3 latent values, then 4 little-endian float32 scales (the
 * k-th for latent values [128k, 128k + 128)), then the 64 bfloat16 RoPE values
 * (not quantized); d_qk must be 576.  The kernel dequantizes each latent value to
 * bfloat16 as bf16(e4m3 * scale), the product in float32 rounded to nearest even,
 * and computes in bfloat16 as for a bfloat16 cache.
 */
typedef enum { MLA_BF16 = 0, MLA_FP16 = 1, MLA_BF16_FP8KV = 2 } mla_dtype;

/* Message for a status code; never NULL. */
MLA_API const char* mla_status_string(int status);

/*
 * Number of scheduler partitions for a device: one per pair of SMs (the
 * decode kernel runs one two-CTA cluster per partition).  On success writes
 * *num_parts (> 0).  Errors: MLA_ERR_INVALID_ARG (null), MLA_ERR_CUDA (no such
 * device).
 */
MLA_API mla_status mla_num_sm_parts(int device, int* num_parts);

/*
 * Sizes of the scheduler outputs for a problem: *tile_md_ints = num_parts * 8,
 * *num_splits_ints = batch * ceil(heads_per_kv / 128) + 1.
 * heads_per_kv = s_q * h_q / h_kv, as in get_mla_metadata's second argument.
 */
MLA_API mla_status mla_metadata_sizes(int batch, int heads_per_kv, int h_kv, int num_parts,
                              size_t* tile_md_ints, size_t* num_splits_ints);

/*
 * Tile scheduler ("FlashMLA" usage page: get_mla_metadata(cache_seqlens,
 * s_q * h_q // h_kv, h_kv) returns tile_scheduler_metadata and num_splits; the
 * page's Tile Scheduler "distributes work across GPU resources"; the upstream
 * FlashMLA documentation's "Usage / MLA Decoding" call also takes is_fp8).
 *
 * Splits the work -- for each request b and row group of 128 query rows, the
 * ceil(L_b / 64) pages of its cache plus a fixed per-chunk overhead -- into
 * num_parts contiguous ranges of nearly equal cost.  A (request, row group)
 * whose pages fall into more than one range is split; num_splits holds the
 * prefix sums of the split counts, and the decode call merges split results.
 *
 *   cache_seqlens    device [batch] int32
 *   heads_per_kv     s_q * h_q / h_kv (> 0)
 *   h_kv             number of KV heads (must be 1: MQA mode)
 *   num_parts        from mla_num_sm_parts (the same value must be passed to decode)
 *   is_fp8_kvcache   nonzero when the decode calls read an "FP8 with scale" cache:
 *                    its pages take longer, so a chunk's fixed overhead counts for
 *                    fewer pages (any schedule is valid for either cache; this one
 *                    balances the work better)
 *   tile_md          device [num_parts, 8] int32, written
 *   num_splits       device [batch * row_groups + 1] int32, written
 * Runs one small kernel on `stream`; no host synchronisation.
 */
MLA_API mla_status mla_get_metadata(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                                    int num_parts, int is_fp8_kvcache, int32_t* tile_md, int32_t* num_splits,
                                    void* stream);

/* Same schedule computed on the host: every pointer is host memory. */
MLA_API mla_status mla_get_metadata_host(const int32_t* cache_seqlens, int batch, int heads_per_kv, int h_kv,
                                         int num_parts, int is_fp8_kvcache, int32_t* tile_md, int32_t* num_splits);

/*
 * Bytes of device workspace mla_decode_with_kvcache needs: a control block of
 * fixed size (the status word and two int32 counters for each of up to
 * MLA_MAX_VIRTUAL_BATCHES (request, row group) pairs), then float32 partial
 * outputs and LSEs for up to batch * row_groups + num_parts splits of 128 rows
 * each.  Returns 0 for invalid sizes, and for batch * row_groups above
 * MLA_MAX_VIRTUAL_BATCHES.
 *
 * mla_decode_workspace_zero_bytes returns the size of the control block (the
 * same for every problem).  It must be zero before a workspace is first used;
 * every call that completes without a device error leaves it zero again, for
 * every later call of any size: the control block does not depend on the
 * problem, so the partial results of one call never land on the counters of
 * another.  After a device error (see mla_read_device_status, whose clear flag
 * zeroes the whole control block) zero it before reusing the workspace.
 */
#define MLA_MAX_VIRTUAL_BATCHES 16384
MLA_API size_t mla_decode_workspace_bytes(int batch, int s_q, int h_q, int h_kv, int num_parts);
MLA_API size_t mla_decode_workspace_zero_bytes(int batch, int s_q, int h_q, int h_kv);

/*
 * Dense MLA decoding with a paged KV cache ("FlashMLA" usage page:
 * flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens, dv,
 * tile_scheduler_metadata, num_splits, causal) -> (o, lse); upstream FlashMLA
 * documentation, "Usage / MLA Decoding": lse is the log-sum-exp of the
 * attention scores per query head).
 *
 * For request b, query token s and head h (kv head 0):
 *   n      = causal ? clamp(L_b - s_q + 1 + s, 0, L_b) : L_b   (bottom-right mask)
 *   x_j    = softmax_scale * <q[b,s,h,:], k_j>,  k_j = cached row j (j < n)
 *   lse    = log(sum_j exp(x_j))                 (-inf when n = 0)
 *   o      = sum_j exp(x_j - lse) * k_j[0:512]   (0 when n = 0)
 *
 *   q, kvcache      device, dtype `dtype` (see mla_dtype), 16-byte aligned
 *   d_qk            576 or 512 (576 for MLA_BF16_FP8KV);  dv must be 512;  h_kv must be 1;
 *                   page_size must be 64
 *   block_table     device int32 [batch, max_blocks_per_seq]
 *   cache_seqlens   device int32 [batch]  (the same array given to mla_get_metadata)
 *   tile_md, num_splits, num_parts   from mla_get_metadata for this batch
 *   causal          0 or 1
 *   softmax_scale   > 0, or <= 0 for 1/sqrt(d_qk)
 *   active_heads    heads [0, active_heads) are real, heads [active_heads, h_q) are
 *                   padding ("FlashMLA vLLM Optimization" page, active-head switch: a
 *                   tensor-parallel rank's query is padded to h_q heads of which it
 *                   consumes only a few).  Padding heads are still computed inside the
 *                   MMA tiles, but their o and lse are left as they were and the
 *                   combine skips them.  A value that is not a multiple of 8 in
 *                   (0, h_q] (0 included), or an h_q that is not a multiple of 8,
 *                   means every head is real.
 *   o               device [batch, s_q, h_q, 512], dtype of q, 16-byte aligned, written
 *                   (real heads)
 *   lse             device float32 [batch, s_q, h_q], written (real heads)
 *   workspace       device, >= mla_decode_workspace_bytes(...), 256-byte aligned
 * Enqueues the split-KV kernel and the combine kernel on `stream`.  Calls
 * sharing one workspace must not run concurrently.
 */
MLA_API mla_status mla_decode_with_kvcache(const void* q, int batch, int s_q, int h_q, int d_qk,
                                   const void* kvcache, int num_blocks, int page_size, int h_kv,
                                   const int32_t* block_table, int max_blocks_per_seq,
                                   const int32_t* cache_seqlens, int dv, int dtype,
                                   const int32_t* tile_md, int num_parts,
                                   const int32_t* num_splits, int causal, float softmax_scale,
                                   int active_heads, void* o, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * The two stages of mla_decode_with_kvcache, for callers that schedule or time
 * them separately (the split-KV / combine kernel pair named on the "FlashMLA
 * vLLM Optimization" page, background section).  Calling mla_decode_splitkv
 * and then mla_decode_combine on one stream with the same arguments is exactly
 * mla_decode_with_kvcache.
 *
 * mla_decode_splitkv: same arguments and checks as mla_decode_with_kvcache.
 *   Each (request, row group) processed by one partition is written to o / lse
 *   directly; one spread over several partitions leaves float32 partial results
 *   in the workspace.
 * mla_decode_combine: merges those partial results into o / lse
 *   (lse = log sum_k exp(lse_k), o = sum_k exp(lse_k - lse) o_k); batch, s_q,
 *   h_q, h_kv, dv, dtype, num_splits, num_parts, active_heads, o, lse and
 *   workspace must be the ones given to mla_decode_splitkv.
 */
MLA_API mla_status mla_decode_splitkv(const void* q, int batch, int s_q, int h_q, int d_qk,
                                      const void* kvcache, int num_blocks, int page_size, int h_kv,
                                      const int32_t* block_table, int max_blocks_per_seq,
                                      const int32_t* cache_seqlens, int dv, int dtype,
                                      const int32_t* tile_md, int num_parts,
                                      const int32_t* num_splits, int causal, float softmax_scale,
                                      int active_heads, void* o, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream);

MLA_API mla_status mla_decode_combine(int batch, int s_q, int h_q, int h_kv, int dv, int dtype,
                                      const int32_t* num_splits, int num_parts, int active_heads,
                                      void* o, float* lse, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * Token-level sparse decoding over an "FP8 with scale" cache (upstream FlashMLA
 * documentation, "Sparse Attention (indices tensor)": indices [batch, s_q, topk],
 * indices[i][j][k] = page * page_size + offset of the k-th row query token j of
 * request i attends, -1 invalid, no block table; the support matrix lists sparse
 * decoding with the FP8 cache only).
 *
 * For request b, query token s and head h (kv head 0):
 *   E      = { k < topk : 0 <= indices[b][s][k] < num_blocks * 64 }   (other entries are invalid)
 *   x_k    = softmax_scale * <q[b,s,h,:], row(indices[b][s][k])>,  k in E   (a row listed twice
 *            counts twice)
 *   lse    = log(sum_{k in E} exp(x_k))                   (-inf when E is empty)
 *   o      = sum_{k in E} exp(x_k - lse) * row(...)[0:512] (0 when E is empty)
 * with rows dequantized as for MLA_BF16_FP8KV.  No causal mask (the list is what the
 * token sees).
 *
 * mla_get_metadata_sparse: the tile scheduler for num_tokens = batch * s_q query tokens of
 *   topk entries each, h_q heads (h_q / h_kv rows per token); tile_md as for
 *   mla_get_metadata with num_parts rows, num_splits [num_tokens * ceil(h_q / h_kv / 128) + 1].
 * mla_decode_sparse:
 *   q            device [batch, s_q, h_q, 576] bfloat16, 16-byte aligned
 *   kvcache      device [num_blocks, 64, 1, 656] bytes ("FP8 with scale" rows) for MLA_BF16_FP8KV,
 *                or [num_blocks, 64, 1, 576] bf16 / fp16 rows for MLA_BF16 / MLA_FP16 (a
 *                16-bit cache: not on the pages, whose sparse decode reads FP8; same definition);
 *                16-byte aligned
 *   indices      device int32 [batch, s_q, topk]
 *   dtype        MLA_BF16_FP8KV, MLA_BF16 or MLA_FP16; d_qk 576 (MLA_ERR_UNSUPPORTED otherwise), dv 512,
 *                h_kv 1, page_size 64
 *   tile_md, num_splits, num_parts   from mla_get_metadata_sparse for this batch * s_q and topk
 *   active_heads, softmax_scale, o, lse  as for mla_decode_with_kvcache
 *   workspace    >= mla_decode_workspace_bytes(batch * s_q, 1, h_q, 1, num_parts)
 * Enqueues the split-KV kernel and the combine kernel on `stream`.
 * mla_decode_sparse_splitkv: its first stage alone; mla_decode_combine with batch * s_q,
 *   s_q = 1 is the second (as for mla_decode_splitkv).
 */
MLA_API mla_status mla_get_metadata_sparse(int num_tokens, int topk, int h_q, int h_kv, int num_parts,
                                           int32_t* tile_md, int32_t* num_splits, void* stream);
/* The same schedule computed on the host into host arrays (synchronous; for tests and tools). */
MLA_API mla_status mla_get_metadata_sparse_host(int num_tokens, int topk, int h_q, int h_kv, int num_parts,
                                                int32_t* tile_md, int32_t* num_splits);
MLA_API mla_status mla_decode_sparse(const void* q, int batch, int s_q, int h_q, int d_qk, const void* kvcache,
                                     int num_blocks, int page_size, int h_kv, const int32_t* indices, int topk,
                                     int dv, int dtype, const int32_t* tile_md, int num_parts,
                                     const int32_t* num_splits, float softmax_scale, int active_heads, void* o,
                                     float* lse, void* workspace, size_t workspace_bytes, void* stream);
MLA_API mla_status mla_decode_sparse_splitkv(const void* q, int batch, int s_q, int h_q, int d_qk,
                                             const void* kvcache, int num_blocks, int page_size, int h_kv,
                                             const int32_t* indices, int topk, int dv, int dtype,
                                             const int32_t* tile_md, int num_parts, const int32_t* num_splits,
                                             float softmax_scale, int active_heads, void* o, float* lse,
                                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse MLA prefill (upstream FlashMLA documentation, "Sparse MLA Prefill": flash_mla_sparse_fwd(q,
 * kv, indices, sm_scale) returns (out, max_logits, lse), equivalent to the documentation's PyTorch
 * code).  No batch dimension and no pages: query token i attends the rows indices[i][0][k] of kv.
 *
 * For query token i and head h (kv head 0), over the valid entries E = { k < topk :
 * 0 <= indices[i][0][k] < s_kv } (-1 or any index >= s_kv is invalid):
 *   P_k        = <q[i,h,:], kv[idx_k,0,:]> * sm_scale * log2(e)
 *   max_logits = max_{k in E} P_k                      (-inf when E is empty)
 *   lse        = log2(sum_{k in E} 2^{P_k})             (base 2; -inf when E is empty)
 *   out        = sum_{k in E} 2^{P_k - lse} kv[idx_k,0,0:512]   (0 when E is empty)
 * (The documentation's equivalent code multiplies by the whole focused row; as everywhere in
 * the MQA mode, V is the leading dv = 512 columns.)
 *
 *   q            device [s_q, h_q, 576] bf16 or fp16, 16-byte aligned
 *   kv           device [s_kv, 1, 576], the dtype of q, 16-byte aligned
 *   indices      device int32 [s_q, 1, topk]
 *   dtype        MLA_BF16 or MLA_FP16;  dv 512;  h_kv 1
 *   sm_scale     > 0, or <= 0 for 1/sqrt(576)
 *   tile_md, num_splits, num_parts   from mla_get_metadata_sparse(s_q, topk, h_q, 1, num_parts, ...)
 *   out          device [s_q, h_q, 512], the dtype of q, written
 *   max_logits   device float32 [s_q, h_q], written
 *   lse          device float32 [s_q, h_q], written (base 2)
 *   workspace    >= mla_decode_workspace_bytes(s_q, 1, h_q, 1, num_parts), zero control block
 * Enqueues the split-KV kernel and the combine kernel on `stream`.  Errors: as for
 * mla_decode_with_kvcache; MLA_ERR_UNSUPPORTED for an FP8 dtype.
 */
MLA_API mla_status mla_sparse_prefill(const void* q, int s_q, int h_q, int d_qk, const void* kv, int s_kv, int h_kv,
                                      const int32_t* indices, int topk, int dv, int dtype, float sm_scale,
                                      const int32_t* tile_md, int num_parts, const int32_t* num_splits, void* out,
                                      float* max_logits, float* lse, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * Reads the device status word of a workspace (synchronises `stream`).
 * *device_status receives MLA_OK or the first device-side error recorded by a
 * decode call that used this workspace; clear != 0 then zeroes the workspace's
 * whole control block (the status word back to MLA_OK, and the split / combine
 * counters a call that met a device error may have left nonzero), so the
 * workspace can be used again.
 */
MLA_API mla_status mla_read_device_status(void* workspace, int clear, int* device_status, void* stream);

/*
 * Allocation-free variant of mla_decode_with_kvcache (the pages describe no
 * counterpart: it exists for callers that cannot allocate device memory).
 *
 * Some callers cannot call cudaMalloc or any allocator at decode time: runtimes
 * that plan all device memory ahead and forbid later allocations, plugins that
 * are handed only tensor pointers by a host framework that owns every buffer,
 * and latency-critical paths where an allocation could block.  This entry point
 * takes the same arguments as mla_decode_with_kvcache minus the workspace; it
 * uses instead a fixed scratch array of MLA_NOALLOC_SCRATCH_BYTES compiled into
 * the library, which every GPU that loads the library holds until the process
 * exits.  The caller still provides q, kvcache, block_table, cache_seqlens, the
 * scheduler outputs, o and lse.
 *
 *   - Problems needing more than MLA_NOALLOC_SCRATCH_BYTES of workspace
 *     (mla_decode_workspace_bytes) are rejected with MLA_ERR_WORKSPACE.
 *   - The first call on a device looks up the device address of the scratch
 *     array (once per device, with that device current); make that first call
 *     before capturing any stream on that device.
 *   - No memory is allocated or freed; each call clears the scratch's status
 *     word and its own split / combine counters with an asynchronous memset on
 *     `stream` and then enqueues the same kernels as mla_decode_with_kvcache.
 *     Device-side errors of a call are read with mla_read_noalloc_status.
 *   - All calls on a device share one scratch array, which keeps the last
 *     call's contents: calls whose execution overlaps on the GPU (different
 *     streams without ordering between them) race on it and give wrong results.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

MLA_API mla_status mla_decode_with_kvcache_noalloc(const void* q, int batch, int s_q, int h_q, int d_qk,
                                                   const void* kvcache, int num_blocks, int page_size,
                                                   int h_kv, const int32_t* block_table,
                                                   int max_blocks_per_seq, const int32_t* cache_seqlens,
                                                   int dv, int dtype, const int32_t* tile_md,
                                                   int num_parts, const int32_t* num_splits, int causal,
                                                   float softmax_scale, int active_heads, void* o, float* lse,
                                                   void* stream);

/*
 * Device status of the allocation-free entry point's scratch on the current
 * device (synchronises `stream`): MLA_OK, or the device-side error
 * (MLA_ERR_DEVICE_CHECK, MLA_ERR_TIMEOUT) recorded by the last
 * mla_decode_with_kvcache_noalloc call on this device, whose o / lse are then
 * not to be trusted.  Read it after a call and before the next one: every
 * call clears it when it starts.  clear != 0 resets it to MLA_OK.  Errors:
 * MLA_ERR_INVALID_ARG (null), MLA_ERR_CUDA.
 */
MLA_API mla_status mla_read_noalloc_status(int clear, int* device_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
