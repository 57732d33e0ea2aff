/*
 * CPU oracle for the GLM-5.3-Flash DSA decode path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link or
 * call this code: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it. It shares no code with the CUDA kernels.
 *
 * Every stage is written as its plain definition with binary64 accumulation
 * and correctly rounded conversions to the stage's storage type:
 *   kn -> bf16, pooled key -> bf16, gate/scores -> fp32, attention out -> bf16.
 * bf16 values are passed as raw uint16 bit patterns.
 *
 * Status: 0 on success, negative on a malformed argument.
 */
#ifndef DSA_ORACLE_H
#define DSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Round a binary64 value to the nearest bf16 (ties to even); return its bits. */
uint16_t orc_bf16_from_f64(double x);
/* Widen bf16 bits to binary64 (exact). */
double orc_f64_from_bf16(uint16_t bits);

/* a1 head gate: out[m,n] = fp32(sum_k hidden[m,k] * w[k,n]). Row-major. */
int orc_head_gate(const float *hidden, const float *w, float *out, int M, int K, int N,
                  int threads);

/* a2 k_norm on one token row: bf16(LayerNorm(x) * ln_w + ln_b), biased variance. */
int orc_layernorm_row(const uint16_t *x, const uint16_t *ln_w, const uint16_t *ln_b,
                      double eps, int D, uint16_t *out);

/* a2+a3 kpool_compress. See dsa_oracle.c for the exact contract. */
int orc_kpool_compress(const uint16_t *k, const uint16_t *gate, const uint8_t *valid,
                       const int32_t *req_start, int B, int D, int kpool, int max_pools,
                       const float *ape, const uint16_t *ln_w, const uint16_t *ln_b,
                       double eps, uint16_t *pool_keys, int32_t *pool_idx,
                       uint8_t *pool_valid, int32_t *first_valid, int threads);

/* a4 index_scores. */
int orc_index_scores(const uint16_t *q_idx, const float *gate_w, const int32_t *q_req,
                     const int32_t *q_pos, int Q, int H, int D, const uint16_t *pool_keys,
                     const uint8_t *pool_valid, const int32_t *first_valid, int B,
                     int kpool, int max_pools, float *scores, uint8_t *cand, int threads);

/* a5+a6 topk_pools + expand_selection. */
int orc_topk_expand(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                    const int32_t *q_req, int Q, int B, int max_pools, int kpool,
                    int select_k, int32_t *top_pools, int32_t *token_ids, int threads);

/* a7 NoPE MLA over the selected tokens, as dense attention under a set mask. */
int orc_sparse_mla(const uint16_t *q, const uint16_t *kv, const int32_t *req_start,
                   const int32_t *q_req, const int32_t *token_ids, int Q, int B, int Hm,
                   int W, int L, double sm_scale, uint16_t *out, float *lse, int threads);
/* f2 the same over an fp8 (E4M3) latent cache with one cache-wide scale. */
double orc_f64_from_e4m3(uint8_t b);
int orc_sparse_mla_fp8(const uint16_t *q, const uint8_t *kv8, double kv_scale,
                       const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids,
                       int Q, int B, int Hm, int W, int L, double sm_scale, uint16_t *out,
                       float *lse, int threads);

#ifdef __cplusplus
}
#endif

#endif /* DSA_ORACLE_H */
