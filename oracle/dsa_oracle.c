/*
 * CPU oracle for the GLM-5.3-Flash DSA decode path.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, the package smoke check and the
 * bench's CPU-baseline leg; never by the product path. It shares no code,
 * header, table or helper with the CUDA kernels.
 *
 * Sources (web pages; cited by title and section):
 *   [mod.rs]  "spark_model/layers/glm5next_dsa/mod.rs" (Atlas docs),
 *             module doc "Shape of the pipeline" and "Traps carried from
 *             Slice 8", the KERNEL_MAX_KPOOL and MASKED_ATTN_MAX_KEYS docs,
 *             Glm5NextDsaConfig::{select_k, out_width, kv_cache_dim, validate}.
 *   [PR227]   "feat(glm53): indexer fp32 head-gate split-K" (stkernel PR #227),
 *             description: the fp32 [M,4096]x[4096,16] head-gate product.
 *   [tap]     "glm53 step tap" README, "What it records": the indexer
 *             checkpoints idx.{q,k,w,gate,topk} and mla.{topk,kvidx}.
 *
 * Readings where the pages leave a step open are marked READING and are the
 * plainest reading the rest supports.
 *
 * Arithmetic: every sum is a plain left-to-right binary64 loop; results are
 * rounded once, to the stage's storage type, with correctly rounded
 * conversions (C's double->float conversion under round-to-nearest-even, and
 * orc_bf16_from_f64 below).
 */
#include "dsa_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_EINVAL (-1)

static int orc_threads(int threads) {
#ifdef _OPENMP
    return threads > 0 ? threads : omp_get_max_threads();
#else
    (void)threads;
    return 1;
#endif
}

double orc_f64_from_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * bf16 has 8 significant bits and float32's exponent range. For a finite x,
 * let 2^E <= |x| < 2^(E+1), clamped to E >= -126 (the subnormal range keeps a
 * fixed spacing). Representable neighbours are multiples of q = 2^(E-7);
 * |x|/q and n*q are exact, and nearbyint under the default rounding mode
 * rounds to the nearest integer with ties to even, which is ties-to-even on
 * the last significand bit. A result of 2^128 or more overflows to infinity.
 */
uint16_t orc_bf16_from_f64(double x) {
    if (isnan(x)) return (uint16_t)0x7FC0;
    if (x == 0.0) return signbit(x) ? (uint16_t)0x8000 : (uint16_t)0x0000;
    if (isinf(x)) return x > 0 ? (uint16_t)0x7F80 : (uint16_t)0xFF80;
    double ax = fabs(x);
    int e2;
    (void)frexp(ax, &e2);          /* ax = m * 2^e2, 0.5 <= m < 1 */
    int E = e2 - 1;                /* 2^E <= ax < 2^(E+1) */
    if (E < -126) E = -126;
    double q = ldexp(1.0, E - 7);
    double r = nearbyint(ax / q) * q;
    if (r >= ldexp(1.0, 128)) return x > 0 ? (uint16_t)0x7F80 : (uint16_t)0xFF80;
    float f = (float)(x < 0 ? -r : r);   /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

static float orc_f32(double x) { return (float)x; }   /* round to nearest even */

/*
 * OCP 8-bit floating point, E4M3 (the "fn" variant: no infinities): sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits. Exponent field 0 is subnormal,
 * m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7); the codes S.1111.111 are NaN, so
 * the largest magnitude is 1.75 * 2^8 = 448.
 */
double orc_f64_from_e4m3(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 0xF, m = b & 0x7;
    if (e == 0xF && m == 0x7) return NAN;
    double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* a1: head gate [PR227]. out[m,n] = sum_k hidden[m,k] * w[k,n], fp32 result. */
int orc_head_gate(const float *hidden, const float *w, float *out, int M, int K, int N,
                  int threads) {
    if (M < 0 || K < 0 || N < 0) return ORC_EINVAL;
    int nt = orc_threads(threads);
    #pragma omp parallel for num_threads(nt) schedule(static)
    for (int m = 0; m < M; ++m) {
        for (int n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int k = 0; k < K; ++k)
                acc += (double)hidden[(size_t)m * K + k] * (double)w[(size_t)k * N + n];
            out[(size_t)m * N + n] = orc_f32(acc);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/*
 * a2: k_norm [mod.rs, trap 1; Glm5NextDsaKernels::k_norm doc]. indexer.k_norm
 * is nn.LayerNorm: subtract the mean, divide by sqrt(biased variance + eps),
 * scale by the weight and add the bias. The in-place kernel the page names
 * reads and writes bf16, so the normalised row is stored as bf16.
 */
int orc_layernorm_row(const uint16_t *x, const uint16_t *ln_w, const uint16_t *ln_b,
                      double eps, int D, uint16_t *out) {
    if (D <= 0) return ORC_EINVAL;
    double mean = 0.0;
    for (int c = 0; c < D; ++c) mean += orc_f64_from_bf16(x[c]);
    mean /= D;
    double var = 0.0;
    for (int c = 0; c < D; ++c) {
        double d = orc_f64_from_bf16(x[c]) - mean;
        var += d * d;
    }
    var /= D;
    double rstd = 1.0 / sqrt(var + eps);
    for (int c = 0; c < D; ++c) {
        double y = (orc_f64_from_bf16(x[c]) - mean) * rstd * orc_f64_from_bf16(ln_w[c])
                   + orc_f64_from_bf16(ln_b[c]);
        out[c] = orc_bf16_from_f64(y);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/*
 * a2+a3: kpool_compress [mod.rs, "Shape of the pipeline" first arrow; traps
 * 1-4; KERNEL_MAX_KPOOL doc].
 *
 * Request b owns token rows [req_start[b], req_start[b+1]) of k, gate and
 * valid; T_b is their count. For each request:
 *   f_b = index (within the request) of the first token whose valid byte is
 *         nonzero, or T_b when there is none (trap 3: pooling starts at the
 *         first valid token; left padding is skipped, never pooled).
 *   Pool p (0 <= p < max_pools) has slot tokens t_s = f_b + p*kpool + s,
 *   s = 0..kpool-1. It is valid iff every slot token exists (t_s < T_b) and is
 *   valid (trap 4: a pool counts only if every slot is valid, so a trailing
 *   partial pool is not a pool).
 *   kn_t = bf16 k_norm of token row t (a2).
 *   For each channel c: the logits l_s = gate[t_s,c] + ape[s,c] are
 *   softmax-normalised over the slot axis s (trap 2: per channel, over pool
 *   slots, not over channels and not over pools), and
 *   pooled[p,c] = bf16( sum_s softmax_s(l)[s] * kn_{t_s}[c] ).
 *
 * Outputs (row-major):
 *   pool_keys [B, max_pools, D] bf16: the pooled key of each valid pool; zero
 *     for an invalid pool p < n_span_b; rows p >= n_span_b are not written,
 *     where n_span_b = min(max_pools, floor((T_b - f_b)/kpool)) is the number
 *     of pool slots whose tokens all lie inside the request.
 *   pool_idx [B, max_pools, kpool] int32: t_s for valid pools, -1 otherwise.
 *   pool_valid [B, max_pools] uint8: 1 for valid pools, 0 otherwise.
 *   first_valid [B] int32: f_b.
 * READING: the gate logits are a per-token [T, D] tensor stored like k (bf16);
 * ape is an fp32 [kpool, D] table; the norm applies per token before pooling.
 */
int orc_kpool_compress(const uint16_t *k, const uint16_t *gate, const uint8_t *valid,
                       const int32_t *req_start, int B, int D, int kpool, int max_pools,
                       const float *ape, const uint16_t *ln_w, const uint16_t *ln_b,
                       double eps, uint16_t *pool_keys, int32_t *pool_idx,
                       uint8_t *pool_valid, int32_t *first_valid, int threads) {
    if (B < 0 || D <= 0 || kpool <= 0 || max_pools < 0) return ORC_EINVAL;
    for (int b = 0; b < B; ++b)
        if (req_start[b + 1] < req_start[b]) return ORC_EINVAL;

    /* first valid token of each request */
    for (int b = 0; b < B; ++b) {
        int T = req_start[b + 1] - req_start[b];
        int f = 0;
        while (f < T && valid[req_start[b] + f] == 0) ++f;
        first_valid[b] = f;
    }

    int nt = orc_threads(threads);
    long long n_items = (long long)B * max_pools;
    #pragma omp parallel num_threads(nt)
    {
        uint16_t *kn = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)kpool * D);
        double *lg = (double *)malloc(sizeof(double) * (size_t)kpool);
        #pragma omp for schedule(dynamic, 64)
        for (long long it = 0; it < n_items; ++it) {
            int b = (int)(it / max_pools);
            int p = (int)(it % max_pools);
            int rs = req_start[b];
            int T = req_start[b + 1] - rs;
            int f = first_valid[b];
            size_t pool = (size_t)b * max_pools + p;
            int in_span = (long long)f + (long long)(p + 1) * kpool <= T;
            int ok = in_span;
            for (int s = 0; s < kpool && ok; ++s)
                if (valid[rs + f + p * kpool + s] == 0) ok = 0;
            pool_valid[pool] = (uint8_t)ok;
            for (int s = 0; s < kpool; ++s)
                pool_idx[pool * kpool + s] = ok ? f + p * kpool + s : -1;
            if (!in_span) continue;
            uint16_t *key = pool_keys + pool * D;
            if (!ok) {
                for (int c = 0; c < D; ++c) key[c] = 0;
                continue;
            }
            for (int s = 0; s < kpool; ++s) {
                size_t row = (size_t)(rs + f + p * kpool + s);
                orc_layernorm_row(k + row * D, ln_w, ln_b, eps, D, kn + (size_t)s * D);
            }
            for (int c = 0; c < D; ++c) {
                double mx = -INFINITY;
                for (int s = 0; s < kpool; ++s) {
                    size_t row = (size_t)(rs + f + p * kpool + s);
                    lg[s] = orc_f64_from_bf16(gate[row * D + c]) + (double)ape[(size_t)s * D + c];
                    if (lg[s] > mx) mx = lg[s];
                }
                double den = 0.0;
                for (int s = 0; s < kpool; ++s) den += exp(lg[s] - mx);
                double acc = 0.0;
                for (int s = 0; s < kpool; ++s)
                    acc += exp(lg[s] - mx) / den * orc_f64_from_bf16(kn[(size_t)s * D + c]);
                key[c] = orc_bf16_from_f64(acc);
            }
        }
        free(kn);
        free(lg);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/*
 * a4: index_scores [mod.rs, "Shape of the pipeline" second arrow: [Q, P]
 * scores plus candidate validity].
 *   b = q_req[q], f = first_valid[b].
 *   cand[q,p] = pool_valid[b,p] and the pool's last slot token
 *               f + p*kpool + kpool - 1 is at or before q_pos[q]
 *               (READING: causal candidacy; a decode query sits at T_b - 1).
 *   scores[q,p] = sum_h gate_w[q,h] * max(0, sum_c q_idx[q,h,c] * key[b,p,c])
 *               (READING: head-gated ReLU dot with no further scale; the head
 *               gate is the tap's idx.w), fp32; -inf where not cand.
 */
int orc_index_scores(const uint16_t *q_idx, const float *gate_w, const int32_t *q_req,
                     const int32_t *q_pos, int Q, int H, int D, const uint16_t *pool_keys,
                     const uint8_t *pool_valid, const int32_t *first_valid, int B,
                     int kpool, int max_pools, float *scores, uint8_t *cand, int threads) {
    if (Q < 0 || H <= 0 || D <= 0 || kpool <= 0 || max_pools < 0) return ORC_EINVAL;
    for (int q = 0; q < Q; ++q)
        if (q_req[q] < 0 || q_req[q] >= B) return ORC_EINVAL;
    int nt = orc_threads(threads);
    long long n_items = (long long)Q * max_pools;
    #pragma omp parallel for num_threads(nt) schedule(dynamic, 256)
    for (long long it = 0; it < n_items; ++it) {
        int q = (int)(it / max_pools);
        int p = (int)(it % max_pools);
        int b = q_req[q];
        size_t pool = (size_t)b * max_pools + p;
        long long last = (long long)first_valid[b] + (long long)p * kpool + kpool - 1;
        int c_ok = pool_valid[pool] != 0 && last <= q_pos[q];
        cand[(size_t)q * max_pools + p] = (uint8_t)c_ok;
        if (!c_ok) {
            scores[(size_t)q * max_pools + p] = -INFINITY;
            continue;
        }
        double s = 0.0;
        for (int h = 0; h < H; ++h) {
            double dot = 0.0;
            for (int c = 0; c < D; ++c)
                dot += orc_f64_from_bf16(q_idx[((size_t)q * H + h) * D + c])
                       * orc_f64_from_bf16(pool_keys[pool * D + c]);
            s += (double)gate_w[(size_t)q * H + h] * (dot > 0.0 ? dot : 0.0);
        }
        scores[(size_t)q * max_pools + p] = orc_f32(s);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/*
 * a5+a6: topk_pools and expand_selection [mod.rs, "Shape of the pipeline"
 * third and fourth arrows; Glm5NextDsaConfig::select_k and out_width; trap 6].
 *   Candidates of query q are ranked by (score descending, pool id ascending)
 *   (READING: lowest pool id wins ties; a NaN score ranks as -inf), and the
 *   n_q = min(select_k, #candidates) best are selected.
 *   READING: the page fixes which pools are selected, not their order in the
 *   row; top_pools[q, :n_q] lists the selected pools in ascending pool id, and
 *   -1 after.
 *   token_ids[q, j*kpool + s] = pool_idx[b, top_pools[q, j], s] for j < n_q and
 *   -1 for every later slot: out_width = select_k * kpool with the tail
 *   option off, and the -1 sentinel row is written in full.
 */
typedef struct { float score; int id; } orc_cand_t;

static int orc_rank_cmp(const void *pa, const void *pb) {
    const orc_cand_t *a = (const orc_cand_t *)pa, *b = (const orc_cand_t *)pb;
    float sa = isnan(a->score) ? -INFINITY : a->score;
    float sb = isnan(b->score) ? -INFINITY : b->score;
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

static int orc_id_cmp(const void *pa, const void *pb) {
    const orc_cand_t *a = (const orc_cand_t *)pa, *b = (const orc_cand_t *)pb;
    return (a->id > b->id) - (a->id < b->id);
}

int orc_topk_expand(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                    const int32_t *q_req, int Q, int B, int max_pools, int kpool,
                    int select_k, int32_t *top_pools, int32_t *token_ids, int threads) {
    if (Q < 0 || max_pools < 0 || kpool <= 0 || select_k < 0) return ORC_EINVAL;
    for (int q = 0; q < Q; ++q)
        if (q_req[q] < 0 || q_req[q] >= B) return ORC_EINVAL;
    int nt = orc_threads(threads);
    #pragma omp parallel num_threads(nt)
    {
        orc_cand_t *list = (orc_cand_t *)malloc(sizeof(orc_cand_t) * (size_t)(max_pools + 1));
        #pragma omp for schedule(dynamic, 1)
        for (int q = 0; q < Q; ++q) {
            int n = 0;
            for (int p = 0; p < max_pools; ++p)
                if (cand[(size_t)q * max_pools + p]) {
                    list[n].score = scores[(size_t)q * max_pools + p];
                    list[n].id = p;
                    ++n;
                }
            qsort(list, (size_t)n, sizeof(orc_cand_t), orc_rank_cmp);
            int nq = n < select_k ? n : select_k;
            qsort(list, (size_t)nq, sizeof(orc_cand_t), orc_id_cmp);   /* selected set by id */
            int b = q_req[q];
            for (int j = 0; j < select_k; ++j) {
                int pid = j < nq ? list[j].id : -1;
                top_pools[(size_t)q * select_k + j] = pid;
                for (int s = 0; s < kpool; ++s)
                    token_ids[((size_t)q * select_k + j) * kpool + s] =
                        pid >= 0 ? pool_idx[((size_t)b * max_pools + pid) * kpool + s] : -1;
            }
        }
        free(list);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/*
 * a7: NoPE MLA restricted to the selected tokens [mod.rs, "Shape of the
 * pipeline" last arrow; MASKED_ATTN_MAX_KEYS doc: the reference semantics is a
 * dense [Q, kv_len] mask of pure set membership, duplicates collapsing; trap
 * 5: no rope section, so the latent row is the whole key and value;
 * kv_cache_dim = kv_lora_rank].
 *   b = q_req[q]; the mask over the request's T_b tokens is set at every
 *   token_ids[q, j] in [0, T_b) (logical ids; physical row = req_start[b]+id,
 *   as the tap's mla.topk vs mla.kvidx pair shows). Then, for each head h,
 *   over the masked positions t in increasing order:
 *     z_t = sm_scale * <q[q,h,:], kv[row(t),:]>,
 *     out[q,h,:] = bf16( sum_t softmax(z)_t * kv[row(t),:] ),
 *     lse[q,h]   = fp32( log sum_t exp(z_t) ).
 *   An empty mask gives out = 0 and lse = -inf.
 * READING: sm_scale is an argument (the pages do not print it).
 */
/* latent value c of cache row r: bf16, or E4M3 times one cache-wide scale */
static double orc_kv_at(const uint16_t *kv, const uint8_t *kv8, double kv_scale, size_t r, int L,
                        int c) {
    if (kv) return orc_f64_from_bf16(kv[r * (size_t)L + c]);
    return kv_scale * orc_f64_from_e4m3(kv8[r * (size_t)L + c]);
}

static int orc_sparse_mla_any(const uint16_t *q, const uint16_t *kv, const uint8_t *kv8,
                              double kv_scale, const int32_t *req_start, const int32_t *q_req,
                              const int32_t *token_ids, int Q, int B, int Hm, int W, int L,
                              double sm_scale, uint16_t *out, float *lse, int threads) {
    if (Q < 0 || Hm <= 0 || W < 0 || L <= 0) return ORC_EINVAL;
    for (int i = 0; i < Q; ++i)
        if (q_req[i] < 0 || q_req[i] >= B) return ORC_EINVAL;
    int nt = orc_threads(threads);
    long long n_items = (long long)Q * Hm;
    #pragma omp parallel num_threads(nt)
    {
        int cap = 0;
        uint8_t *mask = NULL;
        double *z = NULL;
        double *acc = (double *)malloc(sizeof(double) * (size_t)L);
        #pragma omp for schedule(dynamic, 1)
        for (long long it = 0; it < n_items; ++it) {
            int i = (int)(it / Hm);
            int h = (int)(it % Hm);
            int b = q_req[i];
            int rs = req_start[b];
            int T = req_start[b + 1] - rs;
            if (T > cap) {
                free(mask);
                free(z);
                cap = T;
                mask = (uint8_t *)malloc((size_t)cap);
                z = (double *)malloc(sizeof(double) * (size_t)cap);
            }
            if (T > 0) memset(mask, 0, (size_t)T);
            for (int j = 0; j < W; ++j) {
                int id = token_ids[(size_t)i * W + j];
                if (id >= 0 && id < T) mask[id] = 1;
            }
            const uint16_t *qh = q + ((size_t)i * Hm + h) * L;
            double mx = -INFINITY;
            int any = 0;
            for (int t = 0; t < T; ++t) {
                if (!mask[t]) continue;
                double dot = 0.0;
                for (int c = 0; c < L; ++c)
                    dot += orc_f64_from_bf16(qh[c]) *
                           orc_kv_at(kv, kv8, kv_scale, (size_t)(rs + t), L, c);
                z[t] = sm_scale * dot;
                if (z[t] > mx) mx = z[t];
                any = 1;
            }
            uint16_t *o = out + ((size_t)i * Hm + h) * L;
            if (!any) {
                for (int c = 0; c < L; ++c) o[c] = 0;
                if (lse) lse[(size_t)i * Hm + h] = -INFINITY;
                continue;
            }
            double den = 0.0;
            for (int t = 0; t < T; ++t)
                if (mask[t]) den += exp(z[t] - mx);
            for (int c = 0; c < L; ++c) acc[c] = 0.0;
            for (int t = 0; t < T; ++t) {
                if (!mask[t]) continue;
                double pr = exp(z[t] - mx) / den;
                for (int c = 0; c < L; ++c)
                    acc[c] += pr * orc_kv_at(kv, kv8, kv_scale, (size_t)(rs + t), L, c);
            }
            for (int c = 0; c < L; ++c) o[c] = orc_bf16_from_f64(acc[c]);
            if (lse) lse[(size_t)i * Hm + h] = orc_f32(mx + log(den));
        }
        free(mask);
        free(z);
        free(acc);
    }
    return 0;
}

int orc_sparse_mla(const uint16_t *q, const uint16_t *kv, const int32_t *req_start,
                   const int32_t *q_req, const int32_t *token_ids, int Q, int B, int Hm,
                   int W, int L, double sm_scale, uint16_t *out, float *lse, int threads) {
    if (!kv && Q > 0 && W > 0) return ORC_EINVAL;
    return orc_sparse_mla_any(q, kv, NULL, 0.0, req_start, q_req, token_ids, Q, B, Hm, W, L,
                              sm_scale, out, lse, threads);
}

/*
 * f2: the same attention over an fp8 latent cache: row value c is
 * kv_scale * E4M3(kv8[row, c]) (one scale for the whole cache).
 * READING: the pages name an fp8 variant of the paged MLA decode and give no
 * scale layout; one cache-wide fp32 scale is the plainest.
 */
int orc_sparse_mla_fp8(const uint16_t *q, const uint8_t *kv8, double kv_scale,
                       const int32_t *req_start, const int32_t *q_req, const int32_t *token_ids,
                       int Q, int B, int Hm, int W, int L, double sm_scale, uint16_t *out,
                       float *lse, int threads) {
    if (!kv8 && Q > 0 && W > 0) return ORC_EINVAL;
    return orc_sparse_mla_any(q, NULL, kv8, kv_scale, req_start, q_req, token_ids, Q, B, Hm, W, L,
                              sm_scale, out, lse, threads);
}
