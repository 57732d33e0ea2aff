/*
 * dsa.h - C ABI of the B200 (sm_100a) DSA decode path:
 *   head gate -> kpool_compress (with k_norm) -> index_scores -> top-k pools
 *   + token expansion -> NoPE sparse MLA.
 *
 * Sources, cited by page title and section:
 *   [mod.rs] "spark_model/layers/glm5next_dsa/mod.rs": module doc "Shape of
 *            the pipeline" and "Traps carried from Slice 8"; the docs of
 *            KERNEL_KV_LORA_DIM, KERNEL_MAX_KPOOL, Glm5NextDsaKernels and
 *            MASKED_ATTN_MAX_KEYS; Glm5NextDsaConfig::{select_k, out_width,
 *            kv_cache_dim, validate}.
 *   [PR227]  "feat(glm53): indexer fp32 head-gate split-K" (stkernel PR #227),
 *            description and the splitk_applicable predicate.
 *   [tap]    "glm53 step tap" README, "What it records".
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless stated otherwise. The caller owns
 *     every buffer; no entry point allocates, frees or synchronises.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously. The calls capture into CUDA graphs.
 *   - bf16 tensors are passed as `dsa_bf16` (raw bit patterns, uint16_t).
 *   - Bulk tensors must be 16-byte aligned; int32 index arrays 4-byte aligned.
 *   - Host-side checks run first. On any status other than DSA_OK nothing is
 *     launched and no output is touched. DSA_ERR_CUDA means a launch failed
 *     (cudaGetLastError after the launch); outputs are then undefined.
 *   - There is no fallback path: an unsupported shape is refused with
 *     DSA_ERR_UNSUPPORTED, never routed elsewhere ([mod.rs] Glm5NextDsaKernels
 *     doc: a missing DSA entry point is a hard error).
 *   - Every kernel is launched with programmatic dependent launch: it may
 *     start while the kernel before it on the stream drains, and waits for
 *     that kernel (griddepcontrol.wait) before reading anything an earlier
 *     stage of this path writes. Before that wait it already reads inputs the
 *     path never writes: hidden and w (head gate); ape, ln_w, ln_b,
 *     req_start, valid, k and gate (kpool_compress); ape (kpool_compress_tokens); q_idx and q_req
 *     (index_scores); q_req (top-k); q, q_req and req_start (sparse MLA). Write those before
 *     the kernel that immediately precedes the call on the stream, or
 *     separate that kernel from the call by a copy, an event wait or a host
 *     synchronisation.
 *   - Request geometry lives on the device: request b owns cache rows
 *     [req_start[b], req_start[b+1]) (T_b rows). Token ids are LOGICAL, i.e.
 *     relative to the request; the physical row is req_start[b] + id ([tap]:
 *     mla.topk logical vs mla.kvidx physical indices). Device-side values the
 *     host cannot see (req_start, q_req, q_pos, ids) never cause an access out
 *     of the documented buffers: a query whose q_req is outside [0, B) has no
 *     candidates, and ids outside [0, T_b) are ignored.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t dsa_bf16;
typedef struct CUstream_st *dsa_stream_t;

enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent sizes */
    DSA_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
    DSA_ERR_ALIGNMENT = 3,     /* pointer not aligned as required */
    DSA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    DSA_ERR_CUDA = 5           /* the CUDA runtime reported a launch error */
};

/* Fixed geometry of the kernels (see each entry point). */
#define DSA_INDEX_DIM 128          /* indexer head dim D */
#define DSA_MAX_INDEX_HEADS 16     /* indexer heads H (= head-gate N) */
#define DSA_MAX_KPOOL 8            /* [mod.rs] KERNEL_MAX_KPOOL */
#define DSA_KV_LORA 512            /* [mod.rs] KERNEL_KV_LORA_DIM; NoPE: kv_cache_dim */
#define DSA_MAX_SELECT 4096        /* largest select_k (pools per query) */
#define DSA_MAX_MLA_HEADS 128      /* MLA heads per query */

/*
 * Sticky device-side error word. A kernel that gives up a bounded wait (an
 * mbarrier phase that never completes) ORs a code into it and returns early
 * instead of spinning; its outputs are then undefined. This call synchronises
 * the current device, copies the word to *value (host pointer) and, if
 * `reset` is nonzero, clears it. It is a diagnostic, not part of the hot path.
 * Codes: 1 = a bounded wait timed out.
 */
int dsa_device_status(int *value, int reset);

/*
 * Failure-detection self-check. Launches one CTA that waits, through the
 * bounded wait every kernel of the path uses, on an mbarrier phase that nothing
 * completes. The wait gives up after its bound (about two seconds of SM clock
 * cycles), ORs code 1 into the device error word and the kernel writes 0 to
 * *result (a device int; 1 would mean the wait completed). The kernel then
 * returns normally, so the context stays usable. A diagnostic for tests: it
 * occupies the stream for about two seconds.
 */
int dsa_selftest_bounded_wait(int *result, dsa_stream_t stream);

/* Name of a status code (static string, never NULL). */
const char *dsa_status_string(int status);
/* ABI revision of this header; bumps on any signature or contract change. */
int dsa_abi_version(void);
#define DSA_ABI_VERSION 1

/*
 * a1. Indexer head gate [PR227]: out[m, n] = sum_k hidden[m, k] * w[k, n].
 *   hidden fp32 [M, K] row-major; w fp32 [K, N] row-major; out fp32 [M, N].
 *   fp32 products and fp32 accumulation; K is split over a cluster of CTAs and
 *   the partial sums are combined in a fixed order (for many rows, where the
 *   clusters would take more than two waves of the device, one CTA takes 16
 *   rows over the whole of K instead), so results are deterministic (they
 *   differ from a sequential sum only in rounding).
 *   Requires 1 <= N <= 16, K >= 1 with K % 4 == 0; M == 0 is a no-op.
 *   Alignment: hidden 16 bytes; w and out 4 bytes.
 */
int dsa_head_gate(const float *hidden, const float *w, float *out, int M, int K, int N,
                  dsa_stream_t stream);

/*
 * Routing predicate of the head gate (the PR's splitk_applicable, as a status):
 * the status dsa_head_gate returns for these sizes before it looks at any
 * pointer -- DSA_OK when the kernel serves them, DSA_ERR_UNSUPPORTED or
 * DSA_ERR_INVALID_ARG otherwise. Launches nothing.
 */
int dsa_head_gate_supported(int M, int K, int N);

/*
 * a2+a3. kpool_compress with the k_norm LayerNorm fused in
 * ([mod.rs] "Shape of the pipeline" first arrow, traps 1-4, KERNEL_MAX_KPOOL).
 *   k, gate   bf16 [total_tokens, D] row-major (indexer keys; per-token,
 *             per-channel compress-gate logits)
 *   tok_valid uint8 [total_tokens] (nonzero = valid)
 *   req_start int32 [B + 1], non-decreasing, req_start[0] >= 0
 *   ape       fp32 [kpool, D]; ln_w, ln_b bf16 [D]; eps >= 0 (LayerNorm eps)
 * For request b: f_b = first valid token (T_b if none); pool p has slot
 * tokens t_s = f_b + p*kpool + s; it is valid iff every t_s < T_b and is
 * valid. kn_t = bf16(LayerNorm(k_t) * ln_w + ln_b) (biased variance); per
 * channel c, w_s = softmax over s of (gate[t_s, c] + ape[s, c]);
 * pooled[p, c] = bf16(sum_s w_s * kn_{t_s}[c]).
 * Outputs:
 *   pool_keys   bf16 [B, max_pools, D]: pooled key of each valid pool, zero for
 *               an invalid pool p < n_span_b, rows p >= n_span_b NOT written,
 *               with n_span_b = min(max_pools, floor((T_b - f_b) / kpool)).
 *   pool_idx    int32 [B, max_pools, kpool]: t_s (logical) for valid pools,
 *               -1 for every slot of an invalid pool (all rows written).
 *   pool_valid  uint8 [B, max_pools] (all rows written).
 *   first_valid int32 [B]: f_b.
 * The caller sizes max_pools >= ceil(T_b / kpool) for every request; tokens
 * past max_pools * kpool after f_b are not pooled.
 * Requires D == 128, 1 <= kpool <= 8 (DSA_ERR_UNSUPPORTED otherwise: the page
 * refuses larger kpool instead of truncating), B >= 0, max_pools >= 0.
 */
int dsa_kpool_compress(const dsa_bf16 *k, const dsa_bf16 *gate, const uint8_t *tok_valid,
                       const int32_t *req_start, int B, int D, int kpool, int max_pools,
                       const float *ape, const dsa_bf16 *ln_w, const dsa_bf16 *ln_b, float eps,
                       dsa_bf16 *pool_keys, int32_t *pool_idx, uint8_t *pool_valid,
                       int32_t *first_valid, dsa_stream_t stream);

/*
 * f1. indexer_store ([mod.rs] Glm5NextDsaKernels::indexer_store: the staged
 * indexer row is placed at a position resolved on the device and marked
 * valid, so a captured graph replays over the live position).
 *   k_new, gate_new bf16 [n, D]: the new tokens' indexer keys and gate logits
 *   valid_new uint8 [n] (nonzero = valid) or NULL (every new token valid)
 *   tok_req, tok_pos int32 [n]: request b and position t of each new token
 *   req_start int32 [B + 1]: as for dsa_kpool_compress
 *   For each i with 0 <= tok_req[i] < B and 0 <= tok_pos[i] < T_b, row
 *   r = req_start[b] + tok_pos[i] gets k[r, :] = k_new[i, :],
 *   gate[r, :] = gate_new[i, :] and tok_valid[r] = valid_new[i] != 0 (1 when
 *   valid_new is NULL); other new tokens are skipped and nothing else is
 *   written. Two new tokens for one row race (the caller keeps them distinct).
 * Requires D == 128, n >= 0, B >= 0; n == 0 or B == 0 launches nothing.
 * Alignment: k_new, gate_new, k, gate 16 bytes; tok_req, tok_pos, req_start 4.
 */
int dsa_indexer_store(const dsa_bf16 *k_new, const dsa_bf16 *gate_new, const uint8_t *valid_new,
                      const int32_t *tok_req, const int32_t *tok_pos, int n, int D,
                      const int32_t *req_start, int B, dsa_bf16 *k, dsa_bf16 *gate,
                      uint8_t *tok_valid, dsa_stream_t stream);

/*
 * f1. kpool_compress of the pools that hold a range of new tokens (the pooled
 * keys updated in place at the new tokens' pools instead of compressed anew:
 * PR #290 page, the later commit that keeps KPOOL_UPDATE_DIRECT_POS in the
 * profile; pool arithmetic as for dsa_kpool_compress).
 *   Inputs and outputs are those of dsa_kpool_compress, plus
 *   tok_begin, tok_end int32 [B]: request b's changed token rows are
 *             [tok_begin[b], tok_end[b]) (clamped to [0, T_b); empty allowed).
 *   first_valid int32 [B] is read, then written: on entry it holds f_b as
 *   the previous compress of the request left it (any other value, e.g. -1,
 *   asks for every pool of b). If the new f_b differs from it, every pool
 *   row p < max_pools of b is written as dsa_kpool_compress writes it.
 *   Otherwise exactly the pools p < max_pools that hold a changed token,
 *   f_b + p*kpool <= tok_end[b]-1 and f_b + (p+1)*kpool - 1 >= tok_begin[b],
 *   are; every other pool row is left untouched.
 *   So, with req_start unchanged and every row changed since the outputs
 *   held dsa_kpool_compress's result inside the ranges given, the outputs
 *   hold dsa_kpool_compress's result again (byte for byte: the pooled keys
 *   are computed in the same order).
 * Requires D == 128, 1 <= kpool <= 8, B >= 0, max_pools >= 0. One CTA per
 * request; its time grows with the pools it writes.
 */
int dsa_kpool_compress_tokens(const dsa_bf16 *k, const dsa_bf16 *gate, const uint8_t *tok_valid,
                              const int32_t *req_start, int B, int D, int kpool, int max_pools,
                              const float *ape, const dsa_bf16 *ln_w, const dsa_bf16 *ln_b,
                              float eps, const int32_t *tok_begin, const int32_t *tok_end,
                              dsa_bf16 *pool_keys, int32_t *pool_idx, uint8_t *pool_valid,
                              int32_t *first_valid, dsa_stream_t stream);

/*
 * a4. index_scores ([mod.rs] "Shape of the pipeline" second arrow:
 * [Q, P] scores plus candidate validity).
 *   q_idx  bf16 [Q, H, D] indexer queries; gate_w fp32 [Q, H] (head gate of a1)
 *   q_req, q_pos int32 [Q]: request and position of each query
 *   pool_keys, pool_valid, first_valid: as written by dsa_kpool_compress
 *   cand[q, p]   = pool_valid[b, p] and f_b + p*kpool + kpool - 1 <= q_pos[q]
 *   scores[q, p] = sum_h gate_w[q, h] * max(0, <q_idx[q, h, :], pool_keys[b, p, :]>)
 *                  in fp32, and -inf where cand is 0.
 *   Outputs scores fp32 [Q, max_pools] and cand uint8 [Q, max_pools], fully
 *   written. Pool keys of non-candidates are never read.
 * Requires D == 128, 1 <= H <= 16, 1 <= kpool <= 8.
 */
int dsa_index_scores(const dsa_bf16 *q_idx, const float *gate_w, const int32_t *q_req,
                     const int32_t *q_pos, int Q, int H, int D, const dsa_bf16 *pool_keys,
                     const uint8_t *pool_valid, const int32_t *first_valid, int B, int kpool,
                     int max_pools, float *scores, uint8_t *cand, dsa_stream_t stream);

/*
 * a5+a6. topk_pools + expand_selection ([mod.rs] "Shape of the pipeline" third
 * and fourth arrows; Glm5NextDsaConfig::select_k and out_width; trap 6).
 *   Candidates (cand != 0) of query q are ranked by (score descending, pool id
 *   ascending); -0.0 equals +0.0 and a NaN score ranks as -inf. The first
 *   n_q = min(select_k, number of candidates) of that ranking are selected.
 *   top_pools int32 [Q, select_k]: the selected pool ids in ascending order,
 *             then -1 (the pages fix no order for the list; by id it is
 *             unique, and the expanded token ids ascend within a request).
 *   token_ids int32 [Q, select_k * kpool]: token_ids[q, j*kpool + s] =
 *             pool_idx[b, top_pools[q, j], s] for j < n_q, -1 after; every
 *             element is written (the -1 sentinel tail in full).
 *   Selection is exact and deterministic (ties go to the lowest pool id).
 * Requires 1 <= kpool <= 8, 0 <= select_k <= 4096, max_pools >= 0.
 */
int dsa_topk_expand(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                    const int32_t *q_req, int Q, int B, int max_pools, int kpool, int select_k,
                    int32_t *top_pools, int32_t *token_ids, dsa_stream_t stream);

/*
 * f4. topk_pools + expand_selection with always_select_tail ([mod.rs]
 * Glm5NextDsaConfig::out_width: the tail adds kpool - 1 slots to the index
 * row; the step tap's idx.tail_slot).
 *   As dsa_topk_expand, but token_ids rows are out_width = select_k * kpool +
 *   kpool - 1 wide: the first select_k * kpool slots as dsa_topk_expand writes
 *   them, then kpool - 1 tail slots for the query's trailing partial pool.
 *   With f = first_valid[b] and n = (q_pos[q] - f + 1) mod kpool (the tokens
 *   after the query's last complete pool), tail slot s holds the logical id
 *   q_pos[q] + 1 - n + s when s < n, that token is < T_b and tok_valid marks it
 *   valid; every other tail slot is -1 (all of them when q_pos[q] < f or the
 *   query's request is out of range). Those tokens are in no selectable pool
 *   (the pool holding them ends after q_pos), so the row has no duplicates.
 *   q_pos int32 [Q]; first_valid int32 [B] (as written by dsa_kpool_compress);
 *   tok_valid uint8 [total_tokens]; req_start int32 [B + 1].
 * Requires what dsa_topk_expand requires; select_k == 0 writes the tail only.
 */
int dsa_topk_expand_tail(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                         const int32_t *q_req, const int32_t *q_pos, const int32_t *first_valid,
                         const uint8_t *tok_valid, const int32_t *req_start, int Q, int B,
                         int max_pools, int kpool, int select_k, int32_t *top_pools,
                         int32_t *token_ids, dsa_stream_t stream);

/*
 * f3. The fused indexer: a1 + a4 + a5 + a6 in one launch ([PR227] the
 * FUSED_K_GATE arm, which computes the head gate inside the indexer instead of
 * as a separate GEMM; [mod.rs] "Shape of the pipeline" second to fourth
 * arrows).
 *   hidden fp32 [Q, K], w fp32 [K, H]: the head gate's operands; one gate row
 *             per query (gate_w[q, h] = sum_k hidden[q, k] * w[k, h]).
 *   q_idx, q_req, q_pos, pool_keys, pool_valid, first_valid: as for
 *             dsa_index_scores; pool_idx, select_k: as for dsa_topk_expand.
 * Outputs, each as the separate call writes it: gate_w fp32 [Q, H] (as
 * dsa_head_gate), scores fp32 [Q, max_pools] and cand uint8 [Q, max_pools]
 * (as dsa_index_scores, from this gate_w), top_pools int32 [Q, select_k] and
 * token_ids int32 [Q, select_k * kpool] (as dsa_topk_expand, from these
 * scores: the same ranking, ties and -1 tail).
 * One thread-block cluster per query -- 8 CTAs, or 16 when so few queries
 * would leave most of the device idle and the device holds that many such
 * clusters at once -- splits K for the gate and the pools for the scores and
 * the select; partial gates, the radix histograms of every pass and the
 * winners' counts are exchanged through distributed shared memory, so nothing
 * but the outputs goes to global memory and results are deterministic. The gate's K-split differs from
 * dsa_head_gate's, so gate_w (and the scores after it) may differ from the
 * separate calls' in the last bits; both are held to the same tolerance.
 * hidden, w, q_idx, q_req and q_pos are read before the wait on the preceding
 * kernel (see the conventions above).
 * Requires D == 128, 1 <= H <= 16, K >= 1, 1 <= kpool <= 8,
 * 0 <= select_k <= 4096 and max_pools <= 32768 (DSA_ERR_UNSUPPORTED above:
 * dsa_index_scores + dsa_topk_expand serve larger pool counts).
 * Alignment: hidden, w 4 bytes; q_idx, pool_keys 16; int32 arrays 4.
 */
int dsa_indexer_select(const float *hidden, const float *w, int K, const dsa_bf16 *q_idx,
                       const int32_t *q_req, const int32_t *q_pos, int Q, int H, int D,
                       const dsa_bf16 *pool_keys, const uint8_t *pool_valid,
                       const int32_t *first_valid, const int32_t *pool_idx, int B, int kpool,
                       int max_pools, int select_k, float *gate_w, float *scores, uint8_t *cand,
                       int32_t *top_pools, int32_t *token_ids, dsa_stream_t stream);

/*
 * a7. NoPE MLA restricted to the selected tokens ([mod.rs] "Shape of the
 * pipeline" last arrow; MASKED_ATTN_MAX_KEYS doc: set-membership mask, so a
 * per-row gather is exact; trap 5: qk_rope_head_dim == 0, the 512-wide latent
 * row is both key and value).
 *   q         bf16 [Q, Hm, 512] (queries absorbed into the latent space)
 *   kv        bf16 [kv_rows, 512] latent cache (row stride 1024 bytes);
 *             request b owns rows req_start[b] .. req_start[b+1]-1.
 *   kv_rows   rows of kv, 0 <= kv_rows <= INT32_MAX (DSA_ERR_UNSUPPORTED
 *             above: the row gather addresses rows with 32-bit coordinates);
 *             kv may be NULL when it is 0. A row at or past kv_rows is never
 *             read: its id counts as invalid.
 *   token_ids int32 [Q, W] logical ids; -1 and ids outside [0, T_b) ignored.
 *             Ids in a row must be distinct (dsa_topk_expand guarantees it;
 *             the set semantics of the page collapses duplicates).
 *   For each head: z_j = sm_scale * <q[q,h,:], kv[row(j),:]>,
 *   out[q,h,:] = bf16(sum_j softmax(z)_j * kv[row(j),:]) (fp32 accumulation),
 *   lse[q,h] = log(sum_j exp(z_j)) (natural log; -inf and out = 0 when no id
 *   is valid). lse may be NULL. Precision: the P.V product takes the softmax
 *   weights as bf16, and split partials merged through the workspace are
 *   stored as bf16 rows; each moves an output by at most 2^-9 of the largest
 *   selected value in its channel (the row sums and lse stay fp32).
 *   workspace: device scratch of dsa_sparse_mla_workspace_size(Q, Hm, W) bytes
 *   (16-byte aligned; contents need no initialisation; not shared between
 *   calls that may overlap).
 *   A query's ids are cut into splits so the grid fills at most one wave of
 *   148 CTAs, each split holding at least four 48-id chunks (half the row's
 *   chunks when it has fewer than eight). The workspace holds the splits'
 *   partial results, which a second kernel merges in split order.
 * Requires kv_lora == 512 and rope_dim == 0 (DSA_ERR_UNSUPPORTED otherwise,
 * as the page's config validation refuses any other latent width), Hm a
 * multiple of 16 with 16 <= Hm <= 128, W >= 0.
 */
size_t dsa_sparse_mla_workspace_size(int Q, int Hm, int W);
/*
 * Number of kernels dsa_sparse_mla_decode launches for this shape (1 for one
 * split, 2 when the splits merge through the workspace); 0 for an empty or
 * invalid shape. An inspection aid for callers that account for
 * launches; it launches nothing.
 */
int dsa_sparse_mla_launch_count(int Q, int Hm, int W);
int dsa_sparse_mla_decode(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                          const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids, int Q, int B, int Hm,
                          int W, int kv_lora, int rope_dim, float sm_scale, dsa_bf16 *out,
                          float *lse, void *workspace, size_t workspace_bytes,
                          dsa_stream_t stream);

/*
 * f2. Sparse MLA over a block-table paged latent cache ([mod.rs] the serve
 * path is the block-table paged MLA decode taught to walk a selected-index
 * row instead of 0..seq_len).
 *   Arguments, outputs, workspace and refusals are those of
 *   dsa_sparse_mla_decode, except for where a token's latent row lives:
 *   kv          bf16 [kv_rows, 512]: the pool of cache pages, page_size rows
 *               each (kv_rows a multiple of page_size is not required).
 *   block_table int32 [B, max_blocks]: request b's logical token t is in page
 *               block_table[b, t / page_size], row t % page_size of it, i.e.
 *               cache row block_table[b, t / page_size] * page_size + t % page_size.
 *   seq_len     int32 [B]: T_b, the request's token count.
 *   An id is ignored (like -1) when it is outside [0, T_b), its page index is
 *   >= max_blocks, its block number is negative, or its row is >= kv_rows.
 *   Results equal dsa_sparse_mla_decode's on the contiguous cache holding the
 *   same rows (the kernels are the same but for the row lookup).
 * Requires page_size >= 1 and max_blocks >= 0 (DSA_ERR_INVALID_ARG otherwise).
 * seq_len joins q, q_req and req_start among the inputs read before the wait
 * on the preceding kernel; block_table is read after it.
 */
int dsa_sparse_mla_decode_paged(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                                const int32_t *block_table, int max_blocks, int page_size,
                                const int32_t *seq_len, const int32_t *q_req,
                                const int32_t *token_ids, int Q, int B, int Hm, int W, int kv_lora,
                                int rope_dim, float sm_scale, dsa_bf16 *out, float *lse,
                                void *workspace, size_t workspace_bytes, dsa_stream_t stream);

/*
 * f2. The paged sparse MLA over an fp8 latent cache ([mod.rs] names the fp8
 * variant of the block-table paged MLA decode; it gives no scale layout).
 *   As dsa_sparse_mla_decode_paged, except that
 *   kv8       uint8 [kv_rows, 512]: OCP FP8 E4M3 codes (S.1111.111 is NaN),
 *   kv_scale  one fp32 scale for the whole cache (finite, > 0): latent value
 *             = kv_scale * E4M3(code).
 *   The rows enter the tensor-core products widened to bf16, which is exact;
 *   kv_scale is applied to the logits and to the output, so the result is
 *   that of the bf16 kernel on the scaled cache up to fp32 rounding.
 * DSA_ERR_INVALID_ARG for a kv_scale that is not finite and positive.
 */
int dsa_sparse_mla_decode_paged_fp8(const dsa_bf16 *q, const uint8_t *kv8, float kv_scale,
                                    int64_t kv_rows, const int32_t *block_table, int max_blocks,
                                    int page_size, const int32_t *seq_len, const int32_t *q_req,
                                    const int32_t *token_ids, int Q, int B, int Hm, int W,
                                    int kv_lora, int rope_dim, float sm_scale, dsa_bf16 *out,
                                    float *lse, void *workspace, size_t workspace_bytes,
                                    dsa_stream_t stream);

/*
 * dsa_sparse_mla_decode without a workspace argument. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory where they call the MLA: code that runs on an execution path whose
 * memory is fixed before it starts (an engine that reserves every buffer at
 * start-up and forbids allocation per step, or a plugin that only receives
 * the input and output pointers of the op it implements). Such a caller has
 * nowhere to take the split-KV scratch from, so this variant uses a scratch
 * area owned by the library instead.
 *   Arguments, outputs and refusals are those of dsa_sparse_mla_decode, and
 *   the computation and results are the same.
 *   The scratch is a static device array of DSA_NOALLOC_SCRATCH_BYTES bytes
 *   that every GPU which loads the library keeps until the process exits. A
 *   call whose split-KV scratch (dsa_sparse_mla_workspace_size(Q, Hm, W))
 *   exceeds it returns DSA_ERR_WORKSPACE and launches nothing. The split
 *   geometry keeps every grid within 148 CTAs, so no call needs more than
 *   148 x 64 x 1032 bytes (about 9.8 MB: a bf16 row of 512 plus m and l per
 *   head and split): the refusal is a guard that no present shape reaches.
 *   Nothing is allocated or freed: no cudaMalloc, no cudaFree, no allocating
 *   library routine. Each call looks up the scratch's device address
 *   (cudaGetSymbolAddress with the calling thread's device current: a host
 *   query that launches nothing), so the address stays right after a
 *   cudaDeviceReset. The array itself comes into being when the CUDA runtime
 *   loads this library's device code on a device, which under the default
 *   lazy module loading happens at the first call into the library there: if
 *   that first call is this one, the load (and its allocation) happens inside
 *   it. So make one call of any entry point on each device before the region
 *   where nothing may be allocated, and before any stream capture on it.
 *   Every call shares the one scratch area and leaves its last contents there;
 *   nothing in it needs to start at zero (every value the merge reads is
 *   written by the same call first). Calls whose kernels may overlap on the
 *   GPU -- on different streams without ordering between them -- race on the
 *   scratch and must not be made.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (16u << 20)
/* DSA_NOALLOC_SCRATCH_BYTES as the loaded library was built with it. */
size_t dsa_noalloc_scratch_bytes(void);
int dsa_sparse_mla_decode_noalloc(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                                  const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids, int Q, int B,
                                  int Hm, int W, int kv_lora, int rope_dim, float sm_scale,
                                  dsa_bf16 *out, float *lse, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
