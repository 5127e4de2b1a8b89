/*
 * pagedmla.h - C ABI of the B200 (sm_100a) paged MLA decode library.
 *
 * The library decodes Multi-head Latent Attention over a paged KV cache, the
 * operation that the DeepSeek FlashMLA pages describe:
 *
 *   - FlashMLA overview (deepseek.csdn.net), section 2.2 "DeepSeek-V3 MLA",
 *     attention equation: o_{t,i} = sum_{j<=t} softmax_j(q_{t,i}.k_{j,i} /
 *     sqrt(d_h + d_h^R)) v^C_{j,i}; only c^KV (512) and k^R (64) are cached,
 *     the other projections are absorbed, so one cached 576-wide row is the
 *     key of every query head and its first 512 entries are the value.
 *   - same article, section 4.2(1): 64-token pages mapped through block_table;
 *     a split-KV forward kernel plus a kernel that merges the splits.
 *   - FlashMLA usage (blog.soe.dolphin-ai.jp), steps 3-4: the two calls
 *     get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) and
 *     flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens, dv,
 *     tile_scheduler_metadata, num_splits, causal).
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers to contiguous row-major buffers
 *     owned by the caller; the library keeps no reference after returning.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No entry point synchronises the host with the device and none
 *     allocates device memory.
 *   - The return value is PMLA_OK (0) or a negative PMLA_ERR_* code; nothing
 *     is launched when an error is returned.  No C++ exception crosses the ABI.
 *     pmla_last_error() gives a message for the last failing call of the
 *     calling host thread.
 *   - bf16 tensors are passed as pointers to 16-bit storage (uint16_t).
 */
#ifndef PAGEDMLA_H_
#define PAGEDMLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PMLA_API __attribute__((visibility("default")))
#else
#define PMLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define PMLA_OK 0
#define PMLA_ERR_INVALID_ARG (-1)  /* null pointer, negative or inconsistent size      */
#define PMLA_ERR_UNSUPPORTED (-2)  /* d != 576, dv != 512, no sm_100 device, ...      */
#define PMLA_ERR_ALIGNMENT (-3)    /* a pointer is not aligned as its argument requires */
#define PMLA_ERR_CUDA (-4)         /* a CUDA runtime / driver call or launch failed    */
#define PMLA_ERR_WORKSPACE (-5)    /* workspace pointer missing or too small           */
#define PMLA_ERR_DEVICE (-6)       /* a kernel reported an error (see below)           */
#define PMLA_ERR_EXHAUSTED (-7)    /* the page pool has fewer free pages than asked    */

/* The same status codes under the mla_ prefix of the decode calls. */
#define MLA_OK PMLA_OK
#define MLA_ERR_INVALID_ARG PMLA_ERR_INVALID_ARG
#define MLA_ERR_UNSUPPORTED PMLA_ERR_UNSUPPORTED
#define MLA_ERR_ALIGNMENT PMLA_ERR_ALIGNMENT
#define MLA_ERR_CUDA PMLA_ERR_CUDA
#define MLA_ERR_WORKSPACE PMLA_ERR_WORKSPACE
#define MLA_ERR_DEVICE PMLA_ERR_DEVICE
#define MLA_ERR_EXHAUSTED PMLA_ERR_EXHAUSTED

/* Codes the kernels record in the device error word (pmla_device_error()). */
#define PMLA_DEVERR_BAD_PAGE 2    /* a block_table entry outside [0, num_pages): read as zeros  */
#define PMLA_DEVERR_BAD_APPEND 3  /* an appended row lies past its sequence's block table        */
#define PMLA_DEVERR_BAD_SEQLEN 4  /* cache_seqlens[b] > 64 * max_pages_per_seq: decoded as empty */
#define PMLA_DEVERR_WAIT_BASE 100 /* + id of a bounded device wait that gave up                  */

#define PMLA_PAGE_SIZE 64     /* tokens per KV page                                  */
#define PMLA_HEAD_DIM 576     /* q / k width: 512 latent (c^KV) + 64 RoPE (k^R)      */
#define PMLA_HEAD_DIM_V 512   /* value width: the latent part of the same row        */
#define PMLA_METADATA_INTS 8  /* int32 entries per part in tile_scheduler_metadata   */

/*
 * Sizes for one batch shape, computed on the host from device properties.
 *
 *   batch, num_heads_per_head_k (= s_q * h_q / h_kv), num_heads_k (= h_kv):
 *       the shape the metadata is for.
 *   num_parts (out): number of scheduler parts; tile_scheduler_metadata has
 *       num_parts * PMLA_METADATA_INTS int32 entries, num_splits has batch+1.
 *       One part per decode cluster the device holds at once: with one
 *       128-row group per KV head a 2-CTA cluster per (part, KV head); with
 *       more, a 4-CTA cluster per (part, KV head, two row groups), plus the
 *       parts that 2-CTA clusters (one per row group) run on the SMs the 4-CTA
 *       clusters leave free (on B200 and num_heads_per_head_k = 256: 33 + 4).
 *   workspace_bytes (out): device workspace mla_decode_with_kvcache needs for
 *       split partial results of this shape (an upper bound over all lengths).
 * Uses the current CUDA device.  Errors: INVALID_ARG, UNSUPPORTED (more than
 * 2^20 rows per KV head, or (batch + 2048) * num_heads_k * num_heads_per_head_k
 * above 2^32), CUDA.
 */
PMLA_API int mla_get_metadata_sizes(int batch, int num_heads_per_head_k, int num_heads_k, int* num_parts,
                           size_t* workspace_bytes);

/*
 * Length-balanced split-KV schedule (step 3 of the FlashMLA usage).
 *
 * Splits the pages of all sequences (ceil(cache_seqlens[b] / 64) each) into
 * num_parts contiguous ranges of roughly equal cost, charging each piece of a
 * sequence a fixed overhead, so that one long sequence is shared by many SMs
 * and many short ones are packed together.  Runs as one small kernel on
 * `stream`; the host never reads the lengths.
 *
 *   cache_seqlens          int32 [batch], device, lengths in tokens (>= 0).
 *   tile_scheduler_metadata int32 [num_parts][8], device, out.  Part p covers,
 *       in (sequence, page) order, from (m[0], m[1]) up to but excluding
 *       (m[2], m[3]); m[4] is the ordinal of its first piece among the pieces
 *       of sequence m[0]; m[5] is the part's share weight w_p (128, or 107
 *       for a part run by the 2-CTA clusters on the free SMs, which cover a
 *       part at about 0.84 of the 4-CTA clusters' rate per SM); m[6..7] are 0.
 *   num_splits             int32 [batch+1], device, out: exclusive prefix sum
 *       of pieces per sequence (0 pieces: empty sequence, 1: unsplit).
 *   num_parts              from mla_get_metadata_sizes for the same shape
 *                          (any value in [1, 2048] is accepted; only exactly
 *                          that value gives parts of weight 107, otherwise all
 *                          parts weigh 128 and run as 4-CTA clusters).
 * Part boundaries are spaced in cost in proportion to the weights, assuming
 * every part but the first starts inside a sequence, and snapped so no piece
 * is shorter than two pages; no part costs more than
 * ceil(w_p (total + (num_parts-1)*3) / W) + 5, where total sums pages + 3 over
 * the non-empty sequences and W sums the weights (with equal weights,
 * ceil((total + (num_parts-1)*3) / num_parts) + 5).
 * Errors: INVALID_ARG (num_parts outside [1, 2048], null pointers), CUDA.
 */
PMLA_API int mla_get_metadata(const int32_t* cache_seqlens, int batch, int num_heads_per_head_k,
                     int num_heads_k, int32_t* tile_scheduler_metadata, int num_parts,
                     int32_t* num_splits, void* stream);

/*
 * Paged MLA decode (step 4 of the FlashMLA usage): for every sequence b,
 * query token i < s_q and query head h, with g = h / (h_q / h_kv):
 *
 *   S_j   = softmax_scale * dot(q[b][i][h][0:576], K_j)   for visible j
 *   lse   = log(sum_j exp(S_j))                           (natural log)
 *   o     = sum_j exp(S_j - lse) * K_j[0:512]
 *
 * where K_j = kvcache[block_table[b][j / 64]][j % 64][g][0:576] and token j
 * is visible when j < cache_seqlens[b] and, if causal, j <= cache_seqlens[b]
 * - s_q + i.  A row that sees no token gets o = 0 and lse = -inf.
 *
 *   q             bf16 [batch][s_q][h_q][576]
 *   kvcache       bf16 [num_pages][64][h_kv][576]
 *   block_table   int32 [batch][max_pages_per_seq]; entries for pages a
 *                 sequence uses must lie in [0, num_pages)
 *   cache_seqlens int32 [batch], each <= 64 * max_pages_per_seq; a longer
 *                 sequence is not read at all: its rows are written as empty
 *                 (o = 0, lse = -inf) and the device error word records
 *                 PMLA_DEVERR_BAD_SEQLEN
 *   tile_scheduler_metadata, num_parts, num_splits: from mla_get_metadata on
 *                 the same cache_seqlens and shape (must not be modified
 *                 before this call has run on the device)
 *   o             bf16 [batch][s_q][h_q][512], out
 *   lse           fp32 [batch][h_q][s_q], out
 *   workspace     device scratch of >= workspace_bytes from
 *                 mla_get_metadata_sizes; contents need not be initialised;
 *                 must not be shared by calls that may run concurrently.
 * Alignment: q and kvcache 16-byte aligned; o and workspace 32-byte aligned.
 * batch = 0 returns PMLA_OK once the shape arguments are valid, without looking
 * at any pointer (empty tensors may be null) and without launching anything.
 * Errors: INVALID_ARG, UNSUPPORTED (d != 576, dv != 512, h_q % h_kv != 0,
 *         h_q/h_kv neither a divisor of 128 that is >= 8 nor a multiple of 128,
 *         or a shape mla_get_metadata_sizes rejects), ALIGNMENT, WORKSPACE, CUDA.
 * Device-side waits are bounded; a kernel that gives up records an error that
 * pmla_device_error() returns.
 * Launches: a counter-clear kernel, the decode kernel and the merge kernel, the
 * last three as a programmatic launch chain (each may start its setup while the
 * one before runs, and waits for it before reading its results).  The schedule
 * kernel of mla_get_metadata lets the next kernel start early the same way;
 * kernels of the caller that are not launched as programmatic dependents are
 * ordered as usual.
 */
PMLA_API int mla_decode_with_kvcache(const uint16_t* q, const uint16_t* kvcache, const int32_t* block_table,
                            const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                            int d, int dv, int num_pages, int max_pages_per_seq,
                            const int32_t* tile_scheduler_metadata, int num_parts,
                            const int32_t* num_splits, int causal, float softmax_scale,
                            uint16_t* o, float* lse, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * The two kernels of mla_decode_with_kvcache as separate calls, with the same
 * arguments, rules and errors; calling mla_decode_splits then mla_merge_splits
 * on one stream equals one mla_decode_with_kvcache (the FlashMLA overview's
 * split-KV kernel followed by its combine step, section 4.2(1)).
 *
 *   mla_decode_splits: the split-KV decode kernel only.  Sequences cut into
 *       one piece get their final o and lse; pieces of split sequences leave
 *       normalised fp32 partials and their lse in `workspace`.
 *   mla_merge_splits: the merge kernel only.  Reads those partials from
 *       `workspace` and writes o and lse of split and of empty sequences.
 * Useful to time the decode kernel on its own; no state is kept between the
 * calls other than the caller's workspace, which must not change in between.
 */
PMLA_API int mla_decode_splits(const uint16_t* q, const uint16_t* kvcache, const int32_t* block_table,
                               const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                               int d, int dv, int num_pages, int max_pages_per_seq,
                               const int32_t* tile_scheduler_metadata, int num_parts,
                               const int32_t* num_splits, int causal, float softmax_scale,
                               uint16_t* o, float* lse, void* workspace, size_t workspace_bytes,
                               void* stream);
PMLA_API int mla_merge_splits(const uint16_t* q, const uint16_t* kvcache, const int32_t* block_table,
                              const int32_t* cache_seqlens, int batch, int s_q, int h_q, int h_kv,
                              int d, int dv, int num_pages, int max_pages_per_seq,
                              const int32_t* tile_scheduler_metadata, int num_parts,
                              const int32_t* num_splits, int causal, float softmax_scale,
                              uint16_t* o, float* lse, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * Allocation-free variant of mla_decode_with_kvcache (the FlashMLA pages have
 * no counterpart: this entry point exists for callers that cannot allocate
 * device memory, such as code inside a CUDA stream capture, runtimes that own
 * all device memory up front, or plugins whose host forbids other allocations).
 *
 * Same arguments, meaning, layouts and errors as mla_decode_with_kvcache,
 * without workspace/workspace_bytes: the split scratch comes from a 32 MiB
 * array the library keeps in device memory (held on every GPU that loads the
 * library, until the process exits).  Shapes whose scratch bound, as reported
 * by mla_get_metadata_sizes, exceeds 32 MiB are rejected with
 * PMLA_ERR_WORKSPACE and a message in pmla_last_error().
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * All calls share the array: calls whose work may overlap on the GPU race and
 * must be serialised by the caller.  Allocates nothing.
 */
PMLA_API int mla_decode_with_kvcache_noalloc(const uint16_t* q, const uint16_t* kvcache,
                                             const int32_t* block_table, const int32_t* cache_seqlens,
                                             int batch, int s_q, int h_q, int h_kv, int d, int dv,
                                             int num_pages, int max_pages_per_seq,
                                             const int32_t* tile_scheduler_metadata, int num_parts,
                                             const int32_t* num_splits, int causal,
                                             float softmax_scale, uint16_t* o, float* lse,
                                             void* stream);

/*
 * Append of new tokens to the paged cache (the write side of the paged layout
 * of the FlashMLA overview, section 4.2(1); the pages describe the cache but
 * give no call for this, so the signature is ours).  For every sequence b and
 * new token t < s_new, row t of new_kv is copied to position
 * cache_seqlens[b] + t of the sequence: page block_table[b][pos / 64], slot
 * pos % 64, for every KV head.  Decode with cache_seqlens[b] + s_new afterwards.
 *
 *   new_kv        bf16 [batch][s_new][h_kv][576], device, 16-byte aligned.
 *   block_table   int32 [batch][max_pages_per_seq], device: must already hold
 *                 pages for positions up to cache_seqlens[b] + s_new - 1.
 *   cache_seqlens int32 [batch], device: lengths before the append (not changed).
 *   kvcache       bf16 [num_pages][64][h_kv][576], device, written in place.
 *   new_seqlens   int32 [batch], device, out, optional (NULL): cache_seqlens + s_new.
 * Runs as one kernel on `stream` (one warp per row, HBM-bound).  A row past the
 * block table or with a page id outside [0, num_pages) is skipped and recorded
 * in the device error word (pmla_device_error()).
 * Errors: INVALID_ARG, UNSUPPORTED (d != 576), ALIGNMENT, CUDA.
 */
PMLA_API int mla_append_kvcache(const uint16_t* new_kv, const int32_t* block_table,
                                const int32_t* cache_seqlens, int batch, int s_new, int h_kv,
                                int d, uint16_t* kvcache, int num_pages, int max_pages_per_seq,
                                int32_t* new_seqlens, void* stream);

/*
 * Page pool for the paged cache (host memory only, no GPU work).  The FlashMLA
 * overview (section 4.2(1)) describes fixed 64-token physical pages handed to
 * sequences through block_table; it gives no allocator, so this API is ours.
 * Page ids are 0..num_pages-1, i.e. indices into the kvcache's first dimension.
 * Every call is all-or-nothing (on an error the pool is unchanged) and calls on
 * one pool are serialised internally.
 *
 *   pmla_page_pool_create(num_pages, &pool)        -> OK, INVALID_ARG
 *   pmla_page_pool_destroy(pool)                   frees the pool object
 *   pmla_page_pool_num_free(pool)                  -> free pages (>= 0) or INVALID_ARG
 *   pmla_page_pool_alloc(pool, n, pages_out[n])    -> OK, EXHAUSTED (fewer than n free)
 *   pmla_page_pool_free(pool, n, pages[n])         -> OK, INVALID_ARG (an id out of range,
 *                                                     not allocated, or repeated)
 *   pmla_page_pool_grow_sequence(pool, row, max_pages, cur_len, new_len)
 *       allocates pages for a sequence growing from cur_len to new_len tokens
 *       into block-table row entries ceil(cur_len/64) .. ceil(new_len/64)-1
 *       -> OK, EXHAUSTED, INVALID_ARG (new_len < cur_len or past max_pages)
 *   pmla_page_pool_release_sequence(pool, row, len) frees the ceil(len/64)
 *       pages of a sequence of len tokens -> OK, INVALID_ARG
 * `row`, `pages` and `pages_out` are host int32 arrays owned by the caller;
 * copy block tables to the device for mla_decode_with_kvcache.
 */
typedef struct pmla_page_pool pmla_page_pool;
PMLA_API int pmla_page_pool_create(int num_pages, pmla_page_pool** out);
PMLA_API void pmla_page_pool_destroy(pmla_page_pool* pool);
PMLA_API int pmla_page_pool_num_free(pmla_page_pool* pool);
PMLA_API int pmla_page_pool_alloc(pmla_page_pool* pool, int n, int32_t* pages_out);
PMLA_API int pmla_page_pool_free(pmla_page_pool* pool, int n, const int32_t* pages);
PMLA_API int pmla_page_pool_grow_sequence(pmla_page_pool* pool, int32_t* block_table_row,
                                          int max_pages, int cur_len, int new_len);
PMLA_API int pmla_page_pool_release_sequence(pmla_page_pool* pool, const int32_t* block_table_row,
                                             int len);

/*
 * Absorbed MLA projections around the latent decode (FlashMLA overview,
 * section 2.2, "matrix absorption"): per query head h, with W^UK_h and W^UV_h
 * the key and value up-projections (128 x 512 each, stored [h][128][512], bf16),
 *   mla_absorb_query:   q[t][h] = [ W^UK_h^T q_nope[t][h] (512) ; q_rope[t][h] (64) ]
 *   mla_project_output: o[t][h] = W^UV_h o_latent[t][h]           (128)
 * so that decoding q against the latent cache and projecting its output equals
 * attention with the up-projected per-head keys and values.  t runs over the
 * `tokens` query tokens (batch * s_q); one KV head.  Tensor-core GEMMs with
 * fp32 accumulation, bf16 results; the pages give no call for these steps, so
 * the signatures are ours.
 *   q_nope [tokens][heads][128], q_rope [tokens][heads][64], q_out [tokens][heads][576]
 *   o_latent [tokens][heads][512], o_out [tokens][heads][128]
 * Inputs 16-byte aligned, outputs 32-byte aligned, all device memory.
 * Each runs as one kernel launched as a programmatic dependent of the kernel
 * before it on `stream`: it may start, and prefetch the weight matrix into L2,
 * before that kernel has completed; it reads nothing into the computation and
 * writes nothing until that kernel has completed, so stream order holds as for
 * a plain launch.
 * Errors: INVALID_ARG, ALIGNMENT, CUDA.
 */
PMLA_API int mla_absorb_query(const uint16_t* q_nope, const uint16_t* q_rope, const uint16_t* w_uk,
                              int tokens, int heads, uint16_t* q_out, void* stream);
PMLA_API int mla_project_output(const uint16_t* o_latent, const uint16_t* w_uv, int tokens, int heads,
                                uint16_t* o_out, void* stream);

/*
 * Reads and clears the device error word of the current device (synchronises
 * the device).  Returns 0 if no kernel reported an error since the last call,
 * else the first code a kernel recorded (PMLA_DEVERR_*; PMLA_DEVERR_WAIT_BASE
 * plus an id names a bounded wait that gave up).
 */
PMLA_API int pmla_device_error(void);

/* Message for the last failing call of this host thread ("" if none). */
PMLA_API const char* pmla_last_error(void);

/* The same message under the mla_ prefix of the decode calls. */
PMLA_API const char* mla_get_last_error(void);

/* Library version string. */
PMLA_API const char* pmla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDMLA_H_ */
