/*
 * pagedmla.h -- C ABI of libpagedmla.so: FlashMLA-style decode attention for
 * Multi-head Latent Attention over a paged latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (absorbed-query MLA decode):
 *   Each cached token stores ONE latent row c of d = 576 bf16 values (512 latent + 64
 *   rope) per latent head; there is no per-head K or V.  With the query absorbed into
 *   latent space (q' = W^UK^T q, "DeepSeek FlashMLA practitioner notes", dpshk.com,
 *   section 2.1) a query head's score against token j is scale * (q' . c_j) over all 576
 *   columns, and its output is the softmax-weighted sum of the first dv = 512 columns of
 *   the same rows.  Tokens live in fixed 64-token pages addressed through a block table
 *   ("OpenSourceWeek Day 1 - FlashMLA", section II.1, and its params-struct listing with
 *   page_block_size = 64).  Query heads are grouped consecutively per latent head: with
 *   g = h_q / h_kv, head h reads latent head h / g, and the s_q * g query rows of one
 *   latent head form one tile (same page, q.view(b, s_q, h_kv, g, d) listing).
 *
 *   For row (b, s, h): n = causal ? L_b - (s_q - 1 - s) : L_b keys are visible (the s_q
 *   new tokens are the last s_q cache entries), and
 *     out[b, s, h, :] = sum_j softmax_j(scale * q'.c_j) * c_j[0:dv]      (bf16)
 *     lse[b, h, s]    = ln sum_j exp(scale * q'.c_j)                      (fp32)
 *   A row with no visible key gets out = 0 and lse = -inf.
 *
 * Call sequence (same page, section V.2: get_mla_metadata, then flash_mla_with_kvcache):
 *   mla_device_sm_count -> mla_num_parts -> mla_get_metadata (device, once per step)
 *   -> mla_workspace_size -> mla_decode_paged (runs the combine unless told not to).
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" must be device memory of the current CUDA device; the
 *     caller owns all memory.  The library allocates no device memory.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Nothing synchronises the host except mla_query_status.
 *   - Return MLA_OK (0) or a negative MLA_ERR_* code; on error nothing was enqueued and
 *     mla_last_error_string() (thread-local) says why.
 *   - bf16 tensors are passed as void* holding IEEE bfloat16 bit patterns.
 */
#ifndef PAGEDMLA_H_
#define PAGEDMLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#define MLA_OK 0
#define MLA_ERR_ARG (-1)          /* bad shape, stride, pointer or value */
#define MLA_ERR_UNSUPPORTED (-2)  /* d != 576, dv != 512, page != 64, device not sm_100 */
#define MLA_ERR_WORKSPACE (-3)    /* workspace missing, misaligned or too small */
#define MLA_ERR_TIMEOUT (-4)      /* a device-side wait hit its time limit */
#define MLA_ERR_CUDA (-5)         /* a CUDA runtime/driver call failed */

#define MLA_PAGE_SIZE 64          /* tokens per cache page */
#define MLA_D_QK 576              /* latent row width: 512 latent + 64 rope */
#define MLA_D_V 512               /* value width: first 512 latent columns */
#define MLA_TILE_FIELDS 8         /* int32 fields per tile_metadata entry */
#define MLA_SPLIT_OVERHEAD_ROWS 32 /* a split costs max(1, ceil(R / 32)) pages in the plan */
#define MLA_ROWS_PER_SM 64        /* query rows one SM serves; sets the part count */
#define MLA_MAX_BATCH 16384       /* largest batch mla_get_metadata accepts */

#define MLA_FLAG_SKIP_COMBINE 1u  /* mla_decode_paged: leave split partials unmerged */
#define MLA_FLAG_WARP_MMA 2u      /* mla_decode_paged: force the warp-MMA (mma.sync) kernels */
#define MLA_FLAG_TCGEN05 4u       /* mla_decode_paged: force the tcgen05 kernels (up to 16
                                     rows per latent head the 16-row tcgen05 kernel; above 16
                                     rows the default is a tcgen05 kernel already) */
#define MLA_FLAG_ONE_SM 8u        /* mla_decode_paged: above 16 rows, the 1-SM 64-row tcgen05
                                     kernel even where the CTA-pair kernel applies */

typedef struct CUstream_st *mla_stream_t; /* identical to cudaStream_t */

/*
 * mla_device_sm_count -- number of SMs of CUDA device `device` (148 on B200).
 * Host only.  Errors: MLA_ERR_ARG (null out pointer), MLA_ERR_CUDA.
 */
MLA_API int mla_device_sm_count(int device, int *num_sms);

/*
 * mla_num_parts -- how many split-KV parts the scheduler plans for a device with
 * `num_sms` SMs:  max(1, num_sms / (h_kv * ceil(rows_per_kv_head / MLA_ROWS_PER_SM))).
 * rows_per_kv_head = s_q * h_q / h_kv (the second argument of the pages'
 * get_mla_metadata call).  Host only, pure arithmetic.  Errors: MLA_ERR_ARG.
 */
MLA_API int mla_num_parts(int num_sms, int rows_per_kv_head, int h_kv, int *num_parts);

/*
 * mla_metadata_size -- the part count mla_get_metadata needs on the calling thread's current
 * CUDA device: mla_num_parts with that device's SM count.  tile_metadata then takes
 * num_parts * 8 int32 and num_splits batch + 1.  Host only (no kernel, no allocation).
 * Errors: MLA_ERR_ARG (null out pointer, batch < 1 or > MLA_MAX_BATCH, rows_per_kv_head
 * outside [1, 2^20] as in mla_get_metadata, h_kv < 1), MLA_ERR_CUDA (no current device).
 */
MLA_API int mla_metadata_size(int batch, int rows_per_kv_head, int h_kv, int *num_parts);

/*
 * mla_get_metadata -- the split-KV tile scheduler ("OpenSourceWeek Day 1 - FlashMLA",
 * section V.2: get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) -> tile_metadata,
 * num_splits; the pages print its call only, the plan is this library's specification).
 *
 * Plan ("balanced cuts"): with R = rows_per_kv_head and OVH = max(1, ceil(R / 32)) pages
 * (the cost of one split: its fp32 partial of R rows, the query tile, the epilogue),
 * sequence b occupies OVH + ceil(L_b / 64) units of a cost axis (its OVH units first, then
 * one unit per page).  With T the axis length and payload = ceil(T / num_parts), part p
 * covers [p*payload, (p+1)*payload) clipped to T.  A cut at position x inside sequence i
 * becomes the cursor (i, max(0, x - start_i - OVH)) in pages, so a cut inside a
 * sequence's overhead units moves the whole sequence to the next part.  Each part does at
 * most payload + OVH units of work.
 *
 *   cache_seqlens  device int32 [batch], each >= 0
 *   tile_metadata  device int32 [num_parts][8], written:
 *                  {begin_seq, begin_token, end_seq, end_token, begin_split_ordinal, 0,0,0}
 *                  the part covers tokens from (begin_seq, begin_token) up to but
 *                  excluding (end_seq, end_token); tokens are multiples of 64
 *   num_splits     device int32 [batch + 1], written: prefix sums of the number of parts
 *                  touching each sequence (num_splits[0] = 0)
 *   rows_per_kv_head  s_q * h_q / h_kv (sets OVH); num_parts from mla_num_parts.
 * Launches one small kernel on `stream`, as a programmatic dependent launch: it reads
 * cache_seqlens and computes the plan while the kernel before it in the stream is still
 * finishing, and writes tile_metadata and num_splits only after that kernel has completed.
 * So a kernel that writes cache_seqlens and signals programmatic dependents
 * (griddepcontrol.launch_dependents) must do so after those writes; ordinary launches and
 * copies are always waited for.  Errors: MLA_ERR_ARG (null pointer, batch < 1
 * or > MLA_MAX_BATCH, rows_per_kv_head < 1, num_parts < 1), MLA_ERR_CUDA.  Negative lengths are not detected
 * on the device; mla_decode_paged's callers must pass lengths >= 0.
 */
MLA_API int mla_get_metadata(const int32_t *cache_seqlens, int batch, int rows_per_kv_head,
                             int num_parts, int32_t *tile_metadata, int32_t *num_splits,
                             mla_stream_t stream);

/*
 * mla_workspace_size -- bytes of scratch mla_decode_paged needs: a 256-byte status
 * block, then fp32 LSE and fp32 normalised outputs of up to (batch + num_parts) split
 * partials per latent head.  Host only.  Errors: MLA_ERR_ARG.
 * The workspace must be 256-byte aligned and its first 256 bytes zero before first
 * use (the library sets a status word there only when a device wait times out, and
 * mla_query_status clears it again).
 */
MLA_API int mla_workspace_size(int batch, int s_q, int h_q, int h_kv, int num_parts, size_t *bytes);

/*
 * mla_decode_paged -- fused paged MLA decode (see the operation above), following the
 * pages' flash_mla_with_kvcache(q, k_cache, block_table, cache_seqlens, dv,
 * tile_metadata, num_splits, causal=True) (same page, section V.2), with softmax_scale
 * made explicit (the pages' scale is 1/sqrt(d) = 576^-0.5).
 *
 *   q              device bf16 [batch][s_q][h_q][d]; q_strides = element strides of its
 *                  first three dims (the last dim must be contiguous, rows 16-byte
 *                  aligned)
 *   k_cache        device bf16 [num_pages][page_size][h_kv][d], contiguous, 16-byte
 *                  aligned.  Tail slots of a sequence's last page must hold finite values
 *                  (they are loaded and multiplied by zero weights).
 *   block_table    device int32 [batch][>= ceil(L_b/64)] with row stride
 *                  block_table_stride elements; entries used must be in [0, num_pages)
 *                  (not checked on the device)
 *   cache_seqlens  device int32 [batch]; L_b >= 0
 *   dv             must be 512; d must be 576; page_size must be 64
 *   tile_metadata, num_parts, num_splits: from mla_get_metadata on the same lengths
 *   softmax_scale  score scale (> 0, finite)
 *   causal         nonzero: row s sees keys j < L_b - (s_q - 1 - s)
 *   out            device bf16 [batch][s_q][h_q][dv], contiguous (written)
 *   lse            device fp32 [batch][h_q][s_q], contiguous (written; natural log)
 *   workspace      device scratch of mla_workspace_size bytes (see there)
 *   flags          0, or an OR of MLA_FLAG_SKIP_COMBINE (leave the split partials in
 *                  the workspace for a later mla_combine) and at most one kernel choice:
 *                  MLA_FLAG_WARP_MMA, MLA_FLAG_TCGEN05 or MLA_FLAG_ONE_SM.  By default
 *                  the kernel follows the measured costs on B200: up to 16 rows per latent
 *                  head the 16-row warp-MMA kernel; for whole 128-row blocks with
 *                  h_q / h_kv a multiple or a divisor of 64 the CTA-pair tcgen05 kernel
 *                  (two SMs share each MMA, 64 rows each, at the full tensor rate); other
 *                  shapes above 16 rows the 1-SM 64-row tcgen05 kernel.
 *                  MLA_FLAG_WARP_MMA selects the 64-row warp-MMA kernel above 16 rows,
 *                  MLA_FLAG_TCGEN05 the 16-row tcgen05 kernel up to 16 rows and
 *                  MLA_FLAG_ONE_SM the 1-SM 64-row tcgen05 kernel above 16 rows; all are
 *                  kept as measured alternatives and parity-tested like the defaults.
 * Errors: MLA_ERR_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE, MLA_ERR_CUDA.  A device
 * wait that times out (never in correct use) sets the workspace status word; read it
 * with mla_query_status.
 */
MLA_API int mla_decode_paged(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q,
                     int d, const void *k_cache, int64_t num_pages, int page_size, int h_kv,
                     const int32_t *block_table, int64_t block_table_stride,
                     const int32_t *cache_seqlens, int dv, const int32_t *tile_metadata,
                     int num_parts, const int32_t *num_splits, float softmax_scale,
                     int causal, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, unsigned flags, mla_stream_t stream);

/*
 * mla_decode_paged_fp8 -- mla_decode_paged over an FP8 latent cache, for up to 16 query rows
 * per latent head (s_q * h_q / h_kv <= 16: the memory-bound decode shape; the cache bytes
 * halve).  The Baidu page on Flash MLA ("Flash MLA：面向可变长度序列的高效MLA解码内核库解析",
 * section 三.2 and section 四, step 3) names FP8 storage of the cache without a format; this
 * library's format:
 *   k8        device uint8 [num_pages][page_size][h_kv][d]: every token's latent row as OCP
 *             E4M3 ("e4m3fn") codes, contiguous, 16-byte aligned
 *   k_scale   device fp32 [h_kv][num_pages][page_size]: one scale per token and latent head,
 *             contiguous, 16-byte aligned
 * and the latent row a token contributes (to the score and, first dv columns, to the
 * value) is k_scale * e4m3(k8).  Codes are widened exactly in the kernel (every E4M3 value
 * is an f16 value) and both products run on f16 tensor-core MMAs with fp32 accumulation, the
 * query and the probabilities carried in f16 after power-of-two scalings.  The slots of a
 * sequence's last page past its length are not keys: their scales are never read, their
 * codes are read and must not be NaN (any finite code).  All other arguments, layouts,
 * results and errors as in mla_decode_paged (flags: 0 or MLA_FLAG_SKIP_COMBINE; the same
 * workspace size and the same mla_combine).  Errors also: MLA_ERR_UNSUPPORTED for more than
 * 16 rows per latent head.
 */
MLA_API int mla_decode_paged_fp8(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q,
                                 int d, const void *k8, const float *k_scale, int64_t num_pages,
                                 int page_size, int h_kv, const int32_t *block_table,
                                 int64_t block_table_stride, const int32_t *cache_seqlens, int dv,
                                 const int32_t *tile_metadata, int num_parts, const int32_t *num_splits,
                                 float softmax_scale, int causal, void *out, float *lse, void *workspace,
                                 size_t workspace_bytes, unsigned flags, mla_stream_t stream);

/*
 * mla_get_metadata_csr -- split plan for the token-level sparse decode.  The same balanced
 * cuts as mla_get_metadata, over n_lists key lists (one per query token, n_lists = batch *
 * s_q) whose lengths are row_ptr[i + 1] - row_ptr[i] (row_ptr: device int32 [n_lists + 1]).
 * rows_per_kv_head = h_q / h_kv (one query token per tile); num_parts from
 * mla_metadata_size(n_lists, rows_per_kv_head, h_kv, ...).  tile_metadata [num_parts][8] and
 * num_splits [n_lists + 1] as for mla_get_metadata, positions counted in list entries.
 * Errors: MLA_ERR_ARG, MLA_ERR_CUDA.
 */
MLA_API int mla_get_metadata_csr(const int32_t *row_ptr, int n_lists, int rows_per_kv_head, int num_parts,
                                 int32_t *tile_metadata, int32_t *num_splits, mla_stream_t stream);

/*
 * mla_decode_sparse -- token-level sparse decode (the Baidu page on Flash MLA, section 三.3:
 * only the Top-K key connections of a query are kept, the pattern stored in CSR form).
 * Query token (b, s) attends, with all its heads, to the key positions
 * col_idx[row_ptr[b * s_q + s] .. row_ptr[b * s_q + s + 1]) of sequence b that it may see
 * (0 <= position < L_b, and with causal the bottom-right rule: position < L_b - (s_q - 1 -
 * s)); other entries (padding such as -1, positions past the sequence) are pruned, and a
 * position listed twice counts twice.  A query token whose list has no visible entry gets
 * out = 0 and lse = -inf.
 *   row_ptr   device int32 [batch * s_q + 1], non-decreasing, row_ptr[0] = 0 not required
 *   col_idx   device int32 [row_ptr[batch * s_q]] key positions within the sequence
 *   tile_metadata / num_parts / num_splits: from mla_get_metadata_csr over the same row_ptr
 * Other arguments, layouts and results as mla_decode_paged; the workspace size of
 * mla_workspace_size(batch, s_q, h_q, h_kv, num_parts) suffices.  h_q / h_kv <= 16 (one
 * query token's heads form a 16-row warp-MMA tile), batch * s_q <= MLA_MAX_BATCH.  flags:
 * 0 or MLA_FLAG_SKIP_COMBINE; the partials left in the workspace are those of batch * s_q
 * lists of one position each: mla_combine(num_splits, batch * s_q, 1, h_q, ...) merges them
 * into out (same memory order) and writes lse in [batch, s_q, h_q] order.
 * Key rows are fetched one token row at a time (1,152 bytes per latent head).
 * Errors: MLA_ERR_ARG, MLA_ERR_UNSUPPORTED (d, dv, page size, more than 16 heads per latent
 * head, not sm_100), MLA_ERR_WORKSPACE, MLA_ERR_CUDA.
 */
MLA_API int mla_decode_sparse(const void *q, const int64_t q_strides[3], int batch, int s_q, int h_q, int d,
                              const void *k_cache, int64_t num_pages, int page_size, int h_kv,
                              const int32_t *block_table, int64_t block_table_stride, const int32_t *cache_seqlens,
                              const int32_t *row_ptr, const int32_t *col_idx, int dv,
                              const int32_t *tile_metadata, int num_parts, const int32_t *num_splits,
                              float softmax_scale, int causal, void *out, float *lse, void *workspace,
                              size_t workspace_bytes, unsigned flags, mla_stream_t stream);

/*
 * mla_combine -- log-sum-exp merge of split-KV partials: for every sequence with more
 * than one split and every query row, lse = ln sum_k exp(lse_k) and
 * out = sum_k exp(lse_k - lse) * o_k (partials with lse_k = -inf weigh nothing).
 * Reads the partials mla_decode_paged(..., MLA_FLAG_SKIP_COMBINE) left in `workspace`;
 * writes out/lse rows of split sequences only.  Arguments as in mla_decode_paged.
 * Errors: MLA_ERR_ARG, MLA_ERR_WORKSPACE, MLA_ERR_CUDA.
 */
MLA_API int mla_combine(const int32_t *num_splits, int batch, int s_q, int h_q, int h_kv, int dv,
                int num_parts, const void *workspace, size_t workspace_bytes, void *out,
                float *lse, mla_stream_t stream);

/*
 * mla_merge_partials -- log-sum-exp merge of n_parts partial decodes of the same query rows,
 * each over a disjoint part of the keys (a sequence sharded over GPUs: every GPU decodes its
 * shard of the pages with mla_decode_paged, the (out, lse) of all shards are gathered, then
 * merged here).  The merge is mla_combine's log-sum-exp merge, applied across GPUs instead of
 * across the splits of one GPU: lse = ln sum_k exp(lse_k), out = sum_k exp(lse_k - lse) out_k;
 * partials with lse_k = -inf weigh nothing; rows with no key in any part get out = 0 and
 * lse = -inf.
 *   o_parts    device bf16 [n_parts][batch][s_q][h_q][dv], contiguous, 16-byte aligned
 *   lse_parts  device fp32 [n_parts][batch][h_q][s_q] (natural log), contiguous
 *   out, lse   device bf16 [batch][s_q][h_q][dv] and fp32 [batch][h_q][s_q], written
 * dv must be 512.  One kernel on `stream`.  Errors: MLA_ERR_ARG, MLA_ERR_UNSUPPORTED,
 * MLA_ERR_CUDA.
 */
MLA_API int mla_merge_partials(const void *o_parts, const float *lse_parts, int n_parts, int batch, int s_q,
                               int h_q, int dv, void *out, float *lse, mla_stream_t stream);

/*
 * mla_absorb_query / mla_absorb_output -- the dense GEMMs either side of the latent decode
 * ("DeepSeek FlashMLA ... practitioner notes", dpshk.com, section 2.1: with the per-head key
 * k_h = W^UK_h c of latent row c, the score q_h . k_h = (W^UK_h^T q_h) . c, so the query is
 * carried into latent space once instead of expanding the cache per head; the value
 * W^UV_h c likewise leaves latent space after the weighted sum).  Head sizes are fixed to
 * those of the call shape: 128 non-positional query columns per head, 64 positional (rope)
 * columns, latent width 512, 128 output columns per head.  tokens = batch * s_q.
 *
 * mla_absorb_query:  q_out[t][h][0:512] = sum_d q_nope[t][h][d] * w_uk[h][d][0:512];
 *                    q_out[t][h][512:576] = q_rope[t][h][0:64]
 *   q_nope   device bf16, element (t, h, d) at t * nope_strides[0] + h * nope_strides[1] + d
 *   q_rope   device bf16, element (t, h, c) at t * rope_strides[0] + h * rope_strides[1] + c
 *   w_uk     device bf16 [heads][128][512], contiguous
 *   q_out    device bf16 [tokens][heads][576], contiguous (the decode's q)
 * mla_absorb_output: out[t][h][d] = sum_c o_latent[t][h][c] * w_uv[h][d][c]
 *   o_latent device bf16, element (t, h, c) at t * latent_strides[0] + h * latent_strides[1]
 *            + c (the decode's out)
 *   w_uv     device bf16 [heads][128][512], contiguous
 *   out      device bf16 [tokens][heads][128], contiguous
 * bf16 inputs, fp32 accumulation (warp MMA), bf16 results; strides in elements, multiples of
 * 8; q_nope, q_rope, o_latent, the weights and q_out 16-byte aligned, out 4-byte aligned.
 * Each call launches one kernel on `stream` as a programmatic dependent launch: it starts
 * reading w_uk / w_uv while the kernel before it in the stream is still finishing, and reads
 * the activations (q_nope, q_rope, o_latent) only after that kernel has completed.  So the
 * weights must not be written by that kernel (a kernel that writes them and signals
 * programmatic dependents must do so after those writes); ordinary launches and copies are
 * always waited for.  Errors: MLA_ERR_ARG, MLA_ERR_CUDA.
 */
MLA_API int mla_absorb_query(const void *q_nope, const int64_t nope_strides[2], const void *q_rope,
                             const int64_t rope_strides[2], const void *w_uk, int tokens, int heads, void *q_out,
                             mla_stream_t stream);
MLA_API int mla_absorb_output(const void *o_latent, const int64_t latent_strides[2], const void *w_uv, int tokens,
                              int heads, void *out, mla_stream_t stream);

/*
 * mla_query_status -- synchronise `stream`, read and clear the workspace status block.
 * Returns MLA_OK, MLA_ERR_TIMEOUT (a device wait gave up; its results are invalid) or
 * MLA_ERR_CUDA (the stream reported an error).
 */
MLA_API int mla_query_status(void *workspace, mla_stream_t stream);

/*
 * mla_watchdog_selftest -- launches one CTA that waits on a shared-memory barrier that
 * nothing ever completes, with the same bounded wait the decode kernel uses and a
 * limit of `timeout_ns`; the wait gives up, sets the workspace status word and the
 * kernel returns.  Lets a test check the time-out path without hanging a GPU.
 * Errors: MLA_ERR_ARG, MLA_ERR_CUDA.
 */
MLA_API int mla_watchdog_selftest(void *workspace, uint64_t timeout_ns, mla_stream_t stream);

/*
 * mla_decode_paged_static -- mla_decode_paged for callers that cannot allocate device
 * memory (a framework that owns the whole memory budget, a server that reserves all
 * memory at start-up, a real-time loop where an allocation could block or fail).  It
 * allocates nothing: instead of a caller-provided workspace it uses one fixed device
 * array of 8 MiB (MLA_STATIC_SCRATCH_BYTES) that the library carries and that every
 * device which loads the library holds until the process exits.  Arguments, layouts and
 * errors are those of mla_decode_paged without workspace/workspace_bytes; the caller
 * still provides all inputs and outputs.  The pages describe no such variant; it exists
 * for deployment only.
 *   - A shape whose split scratch (mla_workspace_size) exceeds 8 MiB is rejected with
 *     MLA_ERR_WORKSPACE before anything is enqueued.
 *   - MLA_FLAG_SKIP_COMBINE is rejected with MLA_ERR_ARG: the split partials stay in the
 *     library's own array, which cannot be passed to mla_combine, so the combine always
 *     runs.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, host only); the first call on a device may load the library's
 *     device code there, so make it before any stream capture.
 *   - Each call clears the array's 256-byte status block on `stream`, then runs the
 *     decode; the partial results in the array are overwritten by every call.
 *   - All calls share the one array: calls that can overlap on the GPU (different
 *     streams without ordering between them) race and corrupt each other's results.
 *   - A device-side wait that times out is recorded in the array's status block; read it
 *     with mla_query_status_static before the next static call clears it.
 */
#define MLA_STATIC_SCRATCH_BYTES (8u << 20)
MLA_API int mla_decode_paged_static(const void *q, const int64_t q_strides[3], int batch, int s_q,
                                    int h_q, int d, const void *k_cache, int64_t num_pages,
                                    int page_size, int h_kv, const int32_t *block_table,
                                    int64_t block_table_stride, const int32_t *cache_seqlens,
                                    int dv, const int32_t *tile_metadata, int num_parts,
                                    const int32_t *num_splits, float softmax_scale, int causal,
                                    void *out, float *lse, unsigned flags, mla_stream_t stream);

/*
 * mla_query_status_static -- mla_query_status for the static array of
 * mla_decode_paged_static on the current device: synchronise `stream`, read and clear its
 * status block.  Returns MLA_OK, MLA_ERR_TIMEOUT (the last static call's device waits gave
 * up; its out/lse are invalid) or MLA_ERR_CUDA.  Allocates nothing.
 */
MLA_API int mla_query_status_static(mla_stream_t stream);

/* Thread-local description of this thread's last error ("" when none). */
MLA_API const char *mla_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDMLA_H_ */
