// The C ABI of libdsa.so (declared in include/dsa.h). This file is the single
// translation unit of the library: it includes every stage's kernels so the
// sticky device error word is one symbol without relocatable device code.
#include "common.cuh"
#include "head_gate.cuh"
#include "kpool_compress.cuh"
#include "kpool_compress_tokens.cuh"
#include "indexer_store.cuh"
#include "index_scores.cuh"
#include "topk_expand.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"

// ---------------------------------------------------------------------------------------
// Library-owned scratch for dsa_sparse_mla_decode_noalloc: the split-KV partial
// rows that dsa_sparse_mla_decode keeps in the caller's workspace. It is a
// file-scope device array, so every GPU that loads this library holds
// DSA_NOALLOC_SCRATCH_BYTES of it until the process exits. In host code the
// name g_mla_scratch only stands in for the symbol; its device address comes
// from cudaGetSymbolAddress with the call's device current.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_mla_scratch[DSA_NOALLOC_SCRATCH_BYTES];

namespace {
// The scratch's device address on the current device, looked up on every call:
// a host-side query that launches and allocates nothing. Nothing is cached, so
// after cudaDeviceReset (the module, and the array with it, is loaded anew and
// may sit elsewhere) the next call still passes the right address.
int scratch_address(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_scratch) != cudaSuccess || !p) {
        (void)cudaGetLastError();
        return DSA_ERR_CUDA;
    }
    *out = p;
    return DSA_OK;
}
}  // namespace

// Failure-detection self-check: one CTA waits on an mbarrier phase that nothing
// completes, through the same bounded wait as every kernel of the path.
static __global__ void selftest_wait_kernel(int *result) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        dsa::mbar_init(&bar, 1);
        dsa::fence_mbarrier_init();
    }
    __syncthreads();
    const bool ok = dsa::mbar_wait(&bar, 0);   // phase 0 never completes: gives up
    if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

extern "C" {

const char *dsa_status_string(int status) {
    switch (status) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
        case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
        case DSA_ERR_ALIGNMENT: return "DSA_ERR_ALIGNMENT";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
        default: return "DSA_ERR_UNKNOWN";
    }
}

int dsa_abi_version(void) { return DSA_ABI_VERSION; }

int dsa_device_status(int *value, int reset) {
    if (!value) return DSA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(value, dsa::g_device_error, sizeof(int)) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (reset) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(dsa::g_device_error, &zero, sizeof(int)) != cudaSuccess)
            return DSA_ERR_CUDA;
    }
    return DSA_OK;
}

int dsa_selftest_bounded_wait(int *result, dsa_stream_t stream) {
    if (!result) return DSA_ERR_INVALID_ARG;
    if (!dsa::aligned(result, 4)) return DSA_ERR_ALIGNMENT;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(result);
    return dsa::launch_status();
}

int dsa_head_gate_supported(int M, int K, int N) { return dsa::head_gate_shape_status(M, K, N); }

int dsa_head_gate(const float *hidden, const float *w, float *out, int M, int K, int N,
                  dsa_stream_t stream) {
    return dsa::head_gate_launch(hidden, w, out, M, K, N, reinterpret_cast<cudaStream_t>(stream));
}

int dsa_kpool_compress(const dsa_bf16 *k, const dsa_bf16 *gate, const uint8_t *tok_valid,
                       const int32_t *req_start, int B, int D, int kpool, int max_pools,
                       const float *ape, const dsa_bf16 *ln_w, const dsa_bf16 *ln_b, float eps,
                       dsa_bf16 *pool_keys, int32_t *pool_idx, uint8_t *pool_valid,
                       int32_t *first_valid, dsa_stream_t stream) {
    return dsa::kpool_compress_launch(k, gate, tok_valid, req_start, B, D, kpool, max_pools, ape,
                                      ln_w, ln_b, eps, pool_keys, pool_idx, pool_valid,
                                      first_valid, reinterpret_cast<cudaStream_t>(stream));
}

int dsa_indexer_store(const dsa_bf16 *k_new, const dsa_bf16 *gate_new, const uint8_t *valid_new,
                      const int32_t *tok_req, const int32_t *tok_pos, int n, int D,
                      const int32_t *req_start, int B, dsa_bf16 *k, dsa_bf16 *gate,
                      uint8_t *tok_valid, dsa_stream_t stream) {
    return dsa::indexer_store_launch(k_new, gate_new, valid_new, tok_req, tok_pos, n, D, req_start,
                                     B, k, gate, tok_valid, reinterpret_cast<cudaStream_t>(stream));
}

int dsa_kpool_compress_tokens(const dsa_bf16 *k, const dsa_bf16 *gate, const uint8_t *tok_valid,
                              const int32_t *req_start, int B, int D, int kpool, int max_pools,
                              const float *ape, const dsa_bf16 *ln_w, const dsa_bf16 *ln_b,
                              float eps, const int32_t *tok_begin, const int32_t *tok_end,
                              dsa_bf16 *pool_keys, int32_t *pool_idx, uint8_t *pool_valid,
                              int32_t *first_valid, dsa_stream_t stream) {
    return dsa::kpool_compress_tokens_launch(k, gate, tok_valid, req_start, B, D, kpool, max_pools,
                                             ape, ln_w, ln_b, eps, tok_begin, tok_end, pool_keys,
                                             pool_idx, pool_valid, first_valid,
                                             reinterpret_cast<cudaStream_t>(stream));
}

int dsa_index_scores(const dsa_bf16 *q_idx, const float *gate_w, const int32_t *q_req,
                     const int32_t *q_pos, int Q, int H, int D, const dsa_bf16 *pool_keys,
                     const uint8_t *pool_valid, const int32_t *first_valid, int B, int kpool,
                     int max_pools, float *scores, uint8_t *cand, dsa_stream_t stream) {
    return dsa::index_scores_launch(q_idx, gate_w, q_req, q_pos, Q, H, D, pool_keys, pool_valid,
                                    first_valid, B, kpool, max_pools, scores, cand,
                                    reinterpret_cast<cudaStream_t>(stream));
}

int dsa_topk_expand(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                    const int32_t *q_req, int Q, int B, int max_pools, int kpool, int select_k,
                    int32_t *top_pools, int32_t *token_ids, dsa_stream_t stream) {
    const dsa::TailArgs no_tail{nullptr, nullptr, nullptr, nullptr, 0};
    return dsa::topk_expand_launch(scores, cand, pool_idx, q_req, Q, B, max_pools, kpool,
                                   select_k, no_tail, top_pools, token_ids,
                                   reinterpret_cast<cudaStream_t>(stream));
}

int dsa_topk_expand_tail(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                         const int32_t *q_req, const int32_t *q_pos, const int32_t *first_valid,
                         const uint8_t *tok_valid, const int32_t *req_start, int Q, int B,
                         int max_pools, int kpool, int select_k, int32_t *top_pools,
                         int32_t *token_ids, dsa_stream_t stream) {
    if (kpool <= 0) return DSA_ERR_INVALID_ARG;
    const dsa::TailArgs tail{q_pos, first_valid, tok_valid, req_start, kpool - 1};
    return dsa::topk_expand_launch(scores, cand, pool_idx, q_req, Q, B, max_pools, kpool,
                                   select_k, tail, top_pools, token_ids,
                                   reinterpret_cast<cudaStream_t>(stream));
}

int dsa_indexer_select(const float *hidden, const float *w, int K, const dsa_bf16 *q_idx,
                       const int32_t *q_req, const int32_t *q_pos, int Q, int H, int D,
                       const dsa_bf16 *pool_keys, const uint8_t *pool_valid,
                       const int32_t *first_valid, const int32_t *pool_idx, int B, int kpool,
                       int max_pools, int select_k, float *gate_w, float *scores, uint8_t *cand,
                       int32_t *top_pools, int32_t *token_ids, dsa_stream_t stream) {
    return dsa::indexer_launch(hidden, w, K, q_idx, q_req, q_pos, Q, H, D, pool_keys, pool_valid,
                               first_valid, pool_idx, B, kpool, max_pools, select_k, gate_w,
                               scores, cand, top_pools, token_ids,
                               reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_sparse_mla_workspace_size(int Q, int Hm, int W) {
    return dsa::mla_workspace_bytes(Q, Hm, W);
}

int dsa_sparse_mla_launch_count(int Q, int Hm, int W) {
    return dsa::sparse_mla_launch_count(Q, Hm, W);
}

int dsa_sparse_mla_decode(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                          const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids, int Q, int B, int Hm,
                          int W, int kv_lora, int rope_dim, float sm_scale, dsa_bf16 *out,
                          float *lse, void *workspace, size_t workspace_bytes,
                          dsa_stream_t stream) {
    return dsa::sparse_mla_launch(q, kv, kv_rows, req_start, q_req, token_ids, Q, B, Hm, W,
                                  kv_lora, rope_dim, sm_scale, out, lse, workspace, workspace_bytes,
                                  reinterpret_cast<cudaStream_t>(stream));
}

int dsa_sparse_mla_decode_paged(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                                const int32_t *block_table, int max_blocks, int page_size,
                                const int32_t *seq_len, const int32_t *q_req,
                                const int32_t *token_ids, int Q, int B, int Hm, int W, int kv_lora,
                                int rope_dim, float sm_scale, dsa_bf16 *out, float *lse,
                                void *workspace, size_t workspace_bytes, dsa_stream_t stream) {
    return dsa::sparse_mla_launch_paged(q, kv, kv_rows, block_table, max_blocks, page_size,
                                        seq_len, q_req, token_ids, Q, B, Hm, W, kv_lora, rope_dim,
                                        sm_scale, out, lse, workspace, workspace_bytes,
                                        reinterpret_cast<cudaStream_t>(stream));
}

int dsa_sparse_mla_decode_paged_fp8(const dsa_bf16 *q, const uint8_t *kv8, float kv_scale,
                                    int64_t kv_rows, const int32_t *block_table, int max_blocks,
                                    int page_size, const int32_t *seq_len, const int32_t *q_req,
                                    const int32_t *token_ids, int Q, int B, int Hm, int W,
                                    int kv_lora, int rope_dim, float sm_scale, dsa_bf16 *out,
                                    float *lse, void *workspace, size_t workspace_bytes,
                                    dsa_stream_t stream) {
    return dsa::sparse_mla_launch_paged_fp8(q, kv8, kv_scale, kv_rows, block_table, max_blocks,
                                            page_size, seq_len, q_req, token_ids, Q, B, Hm, W,
                                            kv_lora, rope_dim, sm_scale, out, lse, workspace,
                                            workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t dsa_noalloc_scratch_bytes(void) { return (size_t)DSA_NOALLOC_SCRATCH_BYTES; }

int dsa_sparse_mla_decode_noalloc(const dsa_bf16 *q, const dsa_bf16 *kv, int64_t kv_rows,
                                  const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids, int Q, int B,
                                  int Hm, int W, int kv_lora, int rope_dim, float sm_scale,
                                  dsa_bf16 *out, float *lse, dsa_stream_t stream) {
    size_t need = 0;
    if (Q > 0 && Hm > 0 && W >= 0) {
        need = dsa::mla_workspace_bytes(Q, Hm, W);
        if (need > (size_t)DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    if (need > 0) {
        const int st = scratch_address(&scratch);
        if (st != DSA_OK) return st;
    }
    return dsa::sparse_mla_launch(q, kv, kv_rows, req_start, q_req, token_ids, Q, B, Hm, W,
                                  kv_lora, rope_dim, sm_scale, out, lse, scratch, need,
                                  reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
