/*
 * dsa.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention decode library.
 *
 * The decode step has three stages, named on "GLM-52 Runs on RTX 4090" (kernel list:
 * 1. lightning-indexer GEMM, 2. top-k + page-mapping transforms, 3. MLA sparse decode)
 * and in the renning22/glm-5.2-4090 README ("how it works": indexer, top-k + page
 * mapping, MLA sparse decode; "usage": SGLANG_NSA_FUSE_TOPK=1 fuses the page-mapping
 * transform into top-k):
 *
 *   score[q,s] = sum_h w[q,h] * ReLU(q_idx[q,h] . k_idx[s])            (64 heads x 128)
 *   sel[q]     = the min(top_k, vis(q)) highest-scoring logical tokens s < vis(q)
 *   slot       = block_table[b, s / 64] * 64 + s % 64                  (page size 64)
 *   out[q,h,:] = sum_j softmax_j(scale * q_mla[q,h] . KV[slot_j, 0:576]) * KV[slot_j, 0:512]
 *
 * The latent cache row is 576 wide: 512 latent ("nope") columns plus 64 RoPE columns;
 * keys use all 576, values the first 512 ("Show HN: colibri", features: compressed
 * KV-cache of 576 floats per token, 64 heads, no GQA).
 *
 * Conventions shared by every entry point
 *  - Pointers named as device pointers are caller-owned device memory on the current
 *    device; the library never allocates or frees device memory.
 *  - Every call is asynchronous on `stream` (a cudaStream_t, 0 = legacy default).
 *  - Argument errors return synchronously, before any launch, with no side effect.
 *  - Problems only the device can see (a block-table entry outside [0, num_pages),
 *    a sequence longer than its block-table row, a slot index outside the cache)
 *    are clamped so no access leaves its buffer, and are recorded in a sticky error
 *    word inside the workspace; read it with dsa_get_error(). Kernels never trap.
 *    Every wait inside a kernel is bounded (4e9 SM clock cycles, about two seconds); a
 *    wait that runs out records DSA_ERR_TIMEOUT and the kernel returns.
 *  - The workspace must be zero-filled once before its first use (cudaMemset); the
 *    library leaves it reusable. Calls sharing one workspace must be stream-ordered.
 *  - Layouts are row-major and contiguous as annotated. "fp8" is OCP FP8 E4M3, the
 *    "fn" variant (no infinities, largest finite value 448).
 *  - Index lists hold -1 in unused entries. Within a query the order of selected
 *    indices is unspecified.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* bad pointer, size, dtype or alignment (synchronous)        */
  DSA_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement (synchronous)  */
  DSA_ERR_CUDA = 3,          /* a CUDA runtime call failed (synchronous)                   */
  DSA_ERR_WORKSPACE = 4,     /* workspace NULL, too small or misaligned (synchronous)      */
  DSA_ERR_DEVICE_BOUNDS = 5, /* device-side: an index or length was out of range, clamped  */
  DSA_ERR_TIMEOUT = 6        /* device-side: a bounded wait ran out                        */
} dsa_status;

typedef enum {
  DSA_BF16 = 0,
  DSA_FP8_E4M3 = 1,
  DSA_FP32 = 2,
  /* MLA latent caches only: packed 656-byte rows. Bytes [0, 512) the E4M3 codes of the
   * 512 latent columns; [512, 528) four little-endian fp32 scales, scale g for columns
   * [128g, 128g+128); [528, 656) the 64 rope columns as bf16. No scale plane. */
  DSA_FP8_E4M3_ROPE_BF16 = 3
} dsa_dtype;

/* Which call a workspace is sized for (dsa_workspace_size). */
typedef enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_PAGEMAP = 2,
  DSA_OP_LAYER = 3,
  DSA_OP_SHARD_LOCAL = 4,    /* dsa_shard_local_topk  */
  DSA_OP_SHARD_SELECT = 5    /* dsa_shard_select      */
} dsa_op;

/*
 * Paged cache description shared by the indexer, top-k, page-map and layer calls
 * (the "page-mapping transforms" of "GLM-52 Runs on RTX 4090", kernel list item 2).
 * One block table and one physical slot numbering serve both the indexer-key cache
 * and the latent cache. Query q (0 <= q < B*n_q) belongs to sequence b = q / n_q.
 */
typedef struct {
  int32_t B;                  /* sequences (block-table rows), >= 1                        */
  int32_t n_q;                /* queries per sequence: 1 for decode, >1 for chunked prefill */
  const int32_t* seq_lens;    /* device [B]: tokens in each sequence's cache               */
  const int32_t* q_pos;       /* device [B*n_q] causal position (vis = q_pos+1) or NULL
                                 (vis = seq_len)                                            */
  const int32_t* block_table; /* device [B, max_pages_per_seq]: physical page of each
                                 logical page; entries past a sequence's length unused      */
  int32_t max_pages_per_seq;  /* block-table row width, >= 1                               */
  int32_t page_size;          /* tokens per page; must be 64                               */
  int32_t num_pages;          /* physical pages in the caches (bounds for the table)       */
} dsa_paging;

/*
 * Stage 1 - lightning indexer ("GLM-52 Runs on RTX 4090", kernel list item 1).
 *   score[q, s] = k_scale[slot(s)] * sum_h (head_w[q,h] * q_scale[q,h]) * ReLU(<q8[q,h], k8[slot(s)]>)
 * which equals sum_h w * ReLU(q_idx . k_idx) on the dequantised values (scales > 0).
 *  q_idx    device [B*n_q, 64, 128] in q_dtype (DSA_BF16 or DSA_FP8_E4M3)
 *  q_scale  device [B*n_q, 64] fp32 per (query, head) scale; required for fp8, NULL for bf16
 *  head_w   device [B*n_q, 64] fp32 head weights
 *  k_cache  device [num_pages, 64, 128] in k_dtype (must equal q_dtype)
 *  k_scale  device [num_pages, 64] fp32 per-token scale; required for fp8, NULL for bf16
 *  scores   device [B*n_q, L_max] fp32 output; entries s < vis(q) are written, the rest
 *           are left untouched. L_max >= max_pages_per_seq*64 is not required, but
 *           vis(q) is clamped to L_max.
 *  Alignment: q_idx, k_cache and k_scale 16-byte aligned; L_max >= 1.
 */
dsa_status dsa_indexer_scores(const dsa_paging* paging,
                              const void* q_idx, dsa_dtype q_dtype, const float* q_scale,
                              const float* head_w,
                              const void* k_cache, dsa_dtype k_dtype, const float* k_scale,
                              float* scores, int64_t L_max,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Stage 2 - top-k selection with the fused page-mapping transform ("GLM-52 Runs on
 * RTX 4090", kernel list item 2; glm-5.2-4090 README, usage: SGLANG_NSA_FUSE_TOPK=1).
 * For each query picks the k = min(top_k, vis(q)) largest scores among s < vis(q)
 * (all of them when vis(q) <= top_k: the dense path) and writes
 *  logical_out  device [B*n_q, top_k] int32 logical token indices, or NULL
 *  physical_out device [B*n_q, top_k] int32 physical slots block_table[b,s/64]*64+s%64
 * Entries k..top_k-1 are -1. Equal scores at the boundary are broken arbitrarily.
 * Scores are ranked by the IEEE-754 total order of their bit patterns
 * (-NaN < -inf < ... < -0 < +0 < ... < +inf < +NaN); dsa_indexer_scores writes no NaN
 * when its inputs are finite.
 *  scores  device [B*n_q, L_max] fp32 (as written by dsa_indexer_scores)
 *  1 <= top_k <= 16384.
 */
dsa_status dsa_topk_pagemap(const dsa_paging* paging, const float* scores, int64_t L_max,
                            int32_t top_k, int32_t* logical_out, int32_t* physical_out,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * The page-mapping transform alone (the second half of stage 2), exposed so a caller
 * can map an index list it chose itself:
 *  physical[q, i] = block_table[b, logical[q,i] / 64] * 64 + logical[q,i] % 64, -1 -> -1.
 *  logical, physical  device [B*n_q, top_k] int32. Bit-exact integer transform.
 */
dsa_status dsa_pagemap(const dsa_paging* paging, const int32_t* logical, int32_t top_k,
                       int32_t* physical, void* workspace, size_t ws_bytes, void* stream);

/*
 * Stage 3 - MLA sparse decode ("GLM-52 Runs on RTX 4090", kernel list item 3):
 * 64-head attention of each query over only its selected latent rows, split across
 * SMs along the index list and merged with an online-softmax (log-sum-exp) combine.
 *  q         device [Bq, 64, 576] bf16 (absorbed, post-RoPE query)
 *  kv_cache  device [num_slots, 576] in kv_dtype: DSA_BF16, or DSA_FP8_E4M3 with
 *  kv_scale  device [num_slots, 5] fp32: scale g covers columns [128g, 128g+128) for
 *            g < 4 and the 64 rope columns [512, 576) for g = 4; NULL for bf16;
 *            or kv_cache device [num_slots, 656] bytes in DSA_FP8_E4M3_ROPE_BF16 (the
 *            packed layout above) with kv_scale NULL. In the packed layout each row's
 *            values are scaled by 2^-E, E the exponent of its largest group scale, into
 *            fp16: rope values must stay below 2^16 x 2^E in magnitude
 *  physical  device [Bq, top_k] int32 slots, -1 = unused
 *  out       device [Bq, 64, 512] in out_dtype (DSA_BF16 or DSA_FP32)
 *  lse       device [Bq, 64] fp32 natural-log sum of exp(logits), or NULL
 * A query with no valid slot gets out = 0 and lse = -inf.
 * Workspace: mla_workspace_size(Bq, top_k).
 */
dsa_status mla_sparse_decode(int32_t Bq, const void* q, const void* kv_cache, dsa_dtype kv_dtype,
                             const float* kv_scale, int64_t num_slots,
                             const int32_t* physical, int32_t top_k, float softmax_scale,
                             void* out, dsa_dtype out_dtype, float* lse,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * mla_sparse_decode without a workspace argument, for callers that cannot allocate
 * device memory themselves: a plugin running inside an engine that reserves and owns all
 * of the GPU's memory and hands out none of it, or a decode loop that must not call
 * cudaMalloc and cudaFree, which can synchronise the whole device. The source pages
 * have no counterpart to this entry point; it is a packaging of stage 3 only. Arguments and results are those of mla_sparse_decode, except:
 *  status  optional device [2] uint32 (8-byte aligned), or NULL: receives this call's
 *          device-side error words; read and clear it with dsa_get_error(status, stream).
 *          With NULL, device-side range and timeout errors are not reported.
 * The split partials live in a 20 MiB array that the library defines in device memory;
 * every GPU that loads the library holds it until the process exits. That covers every
 * (Bq, top_k) on a 148-SM B200; a call whose partials would not fit (a GPU with more SMs)
 * returns DSA_ERR_WORKSPACE. The first call on each device looks up the array's device
 * address (with that device current), so make that call before any stream capture.
 * All calls on a device share the array and it keeps the last call's contents: calls that
 * may overlap on the GPU (different streams, no ordering between them) race and corrupt
 * each other's results. Allocates nothing (no cudaMalloc, cudaFree or allocating library
 * routine); each call enqueues one 8-byte memset, the kernels of mla_sparse_decode and,
 * with a status pointer, one 8-byte device-to-device copy.
 */
dsa_status mla_sparse_decode_noalloc(int32_t Bq, const void* q, const void* kv_cache, dsa_dtype kv_dtype,
                                     const float* kv_scale, int64_t num_slots,
                                     const int32_t* physical, int32_t top_k, float softmax_scale,
                                     void* out, dsa_dtype out_dtype, float* lse,
                                     unsigned int* status, void* stream);

/*
 * The fused decode layer: indexer -> top-k + page map -> MLA sparse decode on one
 * stream, intermediate scores and index lists kept in the workspace. Arguments as
 * in the three stages above (q_idx and k_cache share idx_dtype). The scores row
 * stride is max_pages_per_seq * 64.
 *  logical_out, physical_out  optional device [B*n_q, top_k] int32 copies of the
 *                             selection (NULL to skip)
 * Workspace: dsa_workspace_size(paging, 0, top_k, DSA_OP_LAYER).
 */
dsa_status dsa_decode_layer(const dsa_paging* paging,
                            const void* q_idx, dsa_dtype idx_dtype, const float* q_scale,
                            const float* head_w, const void* k_cache, const float* k_scale,
                            const void* q_mla, const void* kv_cache, dsa_dtype kv_dtype,
                            const float* kv_scale,
                            int32_t top_k, float softmax_scale,
                            void* out, dsa_dtype out_dtype, float* lse,
                            int32_t* logical_out, int32_t* physical_out,
                            void* workspace, size_t ws_bytes, void* stream);

/*
 * Token-sharded decode: one long sequence per row spread over R ranks (one GPU each),
 * joined by one exchange step. The pages say only that the context reaches 1M tokens
 * (Russian news item on colibri); this split is the library's long-context extension and
 * its result is the unsharded step's: the union of the ranks' local top-k lists holds a
 * global top-k, and merging the ranks' softmax states by their log-sum-exp gives the
 * softmax over the union.
 *
 * Rank r holds tokens [token_offset[b], token_offset[b] + seq_lens[b]) of every row b in
 * its own paged caches, described by its own `local` paging (q_pos must be NULL: every
 * query sees its whole row). Per decode step, on every rank:
 *   1. dsa_indexer_scores(local, ...) over the rank's tokens;
 *   2. dsa_shard_local_topk: local top-k, as (score, global token) candidates;
 *   3. the caller gathers every rank's candidates (e.g. an NCCL all-gather) into
 *      all_score / all_token [R, Bq, top_k], rank-major;
 *   4. dsa_shard_select: the global selection, and this rank's share of it as slots;
 *   5. mla_sparse_decode over those slots with fp32 `out` and `lse`: the rank's state;
 *   6. the caller gathers every rank's out [R, Bq, 64, 512] and lse [R, Bq, 64];
 *   7. dsa_shard_merge: the log-sum-exp merge into the step's output.
 * Every rank passes identical gathered arrays to steps 4 and 7 and gets identical results.
 */

/* Step 2: top-k of this rank's scores (as dsa_topk_pagemap) and the exchange payload
 *  cand_score  device [B*n_q, top_k] fp32: the selected scores, -inf in unused entries
 *  cand_token  device [B*n_q, top_k] int32: their global tokens token_offset[b] + s, -1 unused
 *  token_offset device [B] int32 >= 0 (a global token past 2^31 - 1 is a device-side error)
 * Workspace: dsa_workspace_size(local, L_max, top_k, DSA_OP_SHARD_LOCAL).
 * DSA_ERR_UNSUPPORTED when local->q_pos is not NULL. */
dsa_status dsa_shard_local_topk(const dsa_paging* local, const float* scores, int64_t L_max, int32_t top_k,
                                const int32_t* token_offset, float* cand_score, int32_t* cand_token,
                                void* workspace, size_t ws_bytes, void* stream);

/* Step 4: the global selection among every rank's candidates
 *  all_score, all_token  device [n_ranks, B*n_q, top_k] as gathered (rank-major)
 *  physical_out device [B*n_q, top_k] int32: the physical slots (in `local`'s block table)
 *               of the selected tokens this rank holds, first, then -1
 *  logical_out  device [B*n_q, top_k] int32 or NULL: the whole selection as global tokens
 *               (unordered, -1 after the k selected), the same on every rank
 * Per query k = min(top_k, valid candidates) are selected: the highest scores, and among
 * equal scores at the boundary the lower global tokens (unlike dsa_topk_pagemap, whose
 * boundary ties are arbitrary, so that every rank takes the same decision). A selected
 * token of this rank outside [token_offset[b], token_offset[b] + seq_lens[b]) is a
 * device-side error and is dropped. 1 <= n_ranks, 0 <= rank < n_ranks,
 * n_ranks * top_k < 2^30. Workspace: dsa_workspace_size(local, 0, top_k,
 * DSA_OP_SHARD_SELECT). DSA_ERR_UNSUPPORTED when local->q_pos is not NULL. */
dsa_status dsa_shard_select(const dsa_paging* local, int32_t n_ranks, int32_t rank, const float* all_score,
                            const int32_t* all_token, int32_t top_k, const int32_t* token_offset,
                            int32_t* physical_out, int32_t* logical_out, void* workspace, size_t ws_bytes,
                            void* stream);

/* Step 7: log-sum-exp merge of the ranks' attention states
 *  all_out  device [n_ranks, Bq, 64, 512] fp32 (16-byte aligned): each rank's normalised output
 *  all_lse  device [n_ranks, Bq, 64] fp32: each rank's lse (-inf: no selected token there)
 *  out      device [Bq, 64, 512] in out_dtype (DSA_BF16, 8-byte aligned, or DSA_FP32,
 *           16-byte aligned): sum_r exp(lse_r - LSE) out_r, LSE = log sum_r exp(lse_r)
 *  lse      device [Bq, 64] fp32 LSE, or NULL
 * A (query, head) with every lse_r = -inf gets out = 0 and lse = -inf. No workspace. */
dsa_status dsa_shard_merge(int32_t Bq, int32_t n_ranks, const float* all_out, const float* all_lse, void* out,
                           dsa_dtype out_dtype, float* lse, void* stream);

/* Bytes of workspace `op` needs for this paging (L_max only matters for DSA_OP_INDEXER
 * and DSA_OP_TOPK, where it may be 0). Returns 0 when the arguments are invalid. */
size_t dsa_workspace_size(const dsa_paging* paging, int64_t L_max, int32_t top_k, int32_t op);

/* Bytes of workspace mla_sparse_decode needs for Bq queries and top_k slots each
 * (depends on the current device's SM count). 0 when the arguments are invalid. */
size_t mla_workspace_size(int32_t Bq, int32_t top_k);

/* Number of KV splits mla_sparse_decode will use on the current device. */
int32_t mla_num_splits(int32_t Bq, int32_t top_k);

/* Synchronises `stream`, returns the sticky device error recorded in `workspace`
 * (DSA_OK if none) and clears it. */
dsa_status dsa_get_error(void* workspace, void* stream);

/* Static description of a status code. Never NULL. */
const char* dsa_status_string(dsa_status status);

/* Number of kernel launches the most recent successful call on this host thread
 * issued (for launch accounting). */
int32_t dsa_last_launch_count(void);

/*
 * The step before the decode path, for each query's new token (the position q_pos[q], or
 * seq_lens[b] - 1 when q_pos is NULL; the token's row must already be counted in
 * seq_lens): partial interleaved RoPE ("Show HN: colibri", features: MLA attention with
 * partial interleaved RoPE) on the 64 rope columns of the projected indexer query (the
 * first 64 of each head's 128), the indexer key (the first 64 of 128) and the latent row
 * (columns 512..575), pair i of them turned by pos * rope_base^(-2i/64); E4M3
 * quantisation with amax/448 fp32 scales (1 for an all-zero vector), one per (query,
 * head), one per key, one per 128-column latent group (plus one for the rope columns in
 * DSA_FP8_E4M3); and the key and latent rows written at the token's slot
 * block_table[b, pos / 64] * 64 + pos % 64 of the paged caches.
 *  idx_q      device [Bq, 64, 128] bf16, idx_k [Bq, 128] bf16, latent [Bq, 576] bf16
 *             (projected, before RoPE; 16-byte aligned)
 *  q_mla      device [Bq, 64, 576] bf16 absorbed MLA queries, columns 512..575 rotated
 *             in place; or NULL
 *  q_idx_out  device [Bq, 64, 128] e4m3 and q_scale_out [Bq, 64] fp32: the indexer's
 *             query inputs (q_idx, q_scale of dsa_indexer_scores)
 *  k_cache    device [num_pages, 64, 128] e4m3 with k_scale [num_pages, 64] fp32
 *  kv_cache   device latent cache in kv_dtype: DSA_FP8_E4M3 with kv_scale [slots, 5],
 *             DSA_FP8_E4M3_ROPE_BF16 (656-byte rows) or DSA_BF16, kv_scale NULL
 *  status     optional device [2] uint32 (8-byte aligned, zero before the call): receives
 *             DSA_ERR_DEVICE_BOUNDS for a position or page outside the table; that
 *             token's cache rows are then not written
 * Two queries must not name the same slot. Out-of-place, no workspace, one launch.
 */
dsa_status dsa_rope_quantize_append(const dsa_paging* paging, const void* idx_q, const void* idx_k,
                                    const void* latent, void* q_mla, float rope_base, void* q_idx_out,
                                    float* q_scale_out, void* k_cache, float* k_scale, void* kv_cache,
                                    dsa_dtype kv_dtype, float* kv_scale, unsigned int* status, void* stream);

/*
 * Test hook for the bounded waits of the fp8-cache MLA decode kernel (the kernel
 * mla_sparse_decode, mla_sparse_decode_noalloc and dsa_decode_layer run for an fp8 latent
 * cache). It applies to the later calls made on this host thread.
 *  wait_limit_cycles  bound of every wait in SM clock cycles; 0 restores the default
 *                     (4e9 cycles). Draining in-flight copies and MMAs on the way out
 *                     always uses the default bound.
 *  stall              1: the softmax warps wait on a barrier that nothing arrives on, so
 *                     that wait runs out after wait_limit_cycles; the kernel then stops
 *                     every role, drains its copies and MMAs, frees its tensor memory,
 *                     writes empty split partials and records DSA_ERR_TIMEOUT. 0: normal.
 * Returns DSA_ERR_INVALID_ARG for a negative limit or a stall value other than 0 or 1.
 */
dsa_status dsa_test_set_wait_hooks(int64_t wait_limit_cycles, int32_t stall);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
