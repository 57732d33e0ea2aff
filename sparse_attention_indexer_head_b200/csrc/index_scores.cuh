// a4. index_scores: [Q, P] head-gated ReLU dot scores plus candidate validity
// ("spark_model/layers/glm5next_dsa/mod.rs", "Shape of the pipeline", second
// arrow).
//
// Per query q of request b and pool p:
//   cand = pool_valid[b,p] && last slot token of p <= q_pos[q]
//   score = sum_h gate_w[q,h] * max(0, <q_idx[q,h,:], key[b,p,:]>), -inf if !cand.
//
// On the 5th-generation tensor cores the per-query [16 heads x 128] by
// [128 x pools] product is a dense contraction; the ReLU and the head gate are
// applied to the fp32 dots in the epilogue.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma.cuh"

namespace dsa {

constexpr int kScorePools = 128;                    // pools per CTA (the MMA's M)
constexpr int kScoreThreads = 128;                  // one thread per pool in the epilogue
constexpr int kScoreHeads = DSA_MAX_INDEX_HEADS;    // 16 (the MMA's N)
constexpr uint32_t kScoreKeyAtom = kScorePools * 128;   // 16 KB: one 64-channel column
constexpr uint32_t kScoreQAtom = kScoreHeads * 128;     // 2 KB
constexpr int kScoreSmem = 2 * kScoreKeyAtom + 2 * kScoreQAtom + 1024;   // + alignment slack

// One CTA scores 128 pools of one query on the tensor cores:
//   D[128 pools x 16 heads] = keys[128 x 128] . q_idx[16 x 128]^T
// as 8 tcgen05 MMAs (M=128, N=16, K=16) into tensor memory. Both operands come
// in by 2-D TMA tile loads into the 128B-swizzled K-major layout (two 64-channel
// atoms each). Thread t then owns pool p0+t: it reads its 16 head dots from
// tensor memory and adds g_h * relu(dot_h) over h in order. The key tile is
// requested right after the dependency wait, before the candidate flags are
// known; tiles with no candidate pool skip the MMAs. Keys of non-candidates
// inside a tile are read (one 32 KB box) but do not enter any score.
__global__ void __launch_bounds__(kScoreThreads)
index_scores_kernel(const __grid_constant__ CUtensorMap key_map,
                    const __grid_constant__ CUtensorMap q_map, const float *__restrict__ gate_w,
                    const int32_t *__restrict__ q_req, const int32_t *__restrict__ q_pos, int H,
                    const uint8_t *__restrict__ pool_valid,
                    const int32_t *__restrict__ first_valid, int B, int kpool, int max_pools,
                    float *__restrict__ scores, uint8_t *__restrict__ cand) {
    extern __shared__ uint8_t sc_smem_raw[];
    __shared__ __align__(8) uint64_t q_bar, load_bar, mma_bar;
    __shared__ uint32_t tmem_base;

    const uint32_t raw = smem_u32(sc_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sK = base, sQ = base + 2 * kScoreKeyAtom;

    const int q = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int p0 = blockIdx.x * kScorePools;
    const int p = p0 + tid;

    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 32);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&q_bar, 1);
        mbar_init(&load_bar, 1);
        mbar_init(&mma_bar, 1);
        fence_mbarrier_init();
        // the query's 16 x 128 head rows are a step input: in flight before the wait
        mbar_arrive_expect_tx(&q_bar, 2 * kScoreQAtom);
        tma_load_2d(sQ, &q_map, 0, q * H, &q_bar);
        tma_load_2d(sQ + kScoreQAtom, &q_map, 64, q * H, &q_bar);
    }
    const int b = q_req[q];                   // a step input, like the query rows
    const bool req_ok = b >= 0 && b < B;
    pdl_wait();
    pdl_launch_dependents();
    if (tid == 0 && req_ok) {
        // The key tile (written by the predecessor) is requested at once, while
        // the candidate flags are read; rows past the key map read as zeros.
        mbar_arrive_expect_tx(&load_bar, 2 * kScoreKeyAtom);
        const int row = b * max_pools + p0;
        tma_load_2d(sK, &key_map, 0, row, &load_bar);
        tma_load_2d(sK + kScoreKeyAtom, &key_map, 64, row, &load_bar);
    }

    bool is_cand = false;
    if (req_ok && p < max_pools) {
        const long long last = (long long)first_valid[b] + (long long)p * kpool + kpool - 1;
        is_cand = pool_valid[(size_t)b * max_pools + p] != 0 && last <= (long long)q_pos[q];
    }
    float g[kScoreHeads];
#pragma unroll
    for (int h = 0; h < kScoreHeads; ++h) g[h] = (req_ok && h < H) ? __ldg(gate_w + (size_t)q * H + h) : 0.f;

    tc::fence_before_sync();
    const bool any = __syncthreads_or(is_cand) != 0;
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;

    bool ok = true;
    if (any) {
        if (tid == 0) {
            ok = mbar_wait(&load_bar, 0) && mbar_wait(&q_bar, 0);
            if (ok) {
                tc::fence_after_sync();
                constexpr uint32_t idesc = tc::idesc_bf16(kScorePools, kScoreHeads, false, false);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off_k = (kk >> 2) * kScoreKeyAtom + (kk & 3) * 32;
                    const uint32_t off_q = (kk >> 2) * kScoreQAtom + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem, tc::desc_sw128(sK + off_k, 16, 1024),
                                    tc::desc_sw128(sQ + off_q, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                }
            }
            tc::mma_commit(&mma_bar);   // arrives even when no MMA was issued
        }
        __syncwarp();
        ok = mbar_wait(&mma_bar, 0) && ok;
        ok = __syncthreads_and(ok) != 0;
        tc::fence_after_sync();
    }

    if (!any && tid == 0) {   // every copy lands before the CTA leaves
        (void)mbar_wait(&q_bar, 0);
        if (req_ok) (void)mbar_wait(&load_bar, 0);
    }

    float score = -INFINITY;
    if (any && ok) {
        uint32_t d[kScoreHeads];
        tc::tmem_ld16(tmem + ((uint32_t)(32 * warp) << 16), d);
        tc::tmem_wait_ld();
        float sacc = 0.f;
#pragma unroll
        for (int h = 0; h < kScoreHeads; ++h) sacc = fmaf(g[h], fmaxf(__uint_as_float(d[h]), 0.f), sacc);
        if (is_cand) score = sacc;
    }
    if (p < max_pools) {
        const size_t out_i = (size_t)q * max_pools + p;
        scores[out_i] = is_cand ? score : -INFINITY;
        cand[out_i] = is_cand ? 1 : 0;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 32);
}

// Many queries (chunked prefill): queries that share a request share its key
// tiles, so one CTA takes a group of up to kScoreGroup consecutive queries and
// kScoreTilesPerCta consecutive key tiles. Each run of equal q_req in the group
// is one MMA product per tile:
//   D[128 pools x 16·len] = keys[128 x 128] . q_idx[16·len x 128]^T
// (8 MMAs, M=128, N=16·len, K=16), the run's query rows loaded once, the key
// tile streamed into one stage that is refilled as soon as the MMAs have read
// it (so the next tile's load overlaps this tile's epilogue). The epilogue is
// the single-query kernel's, per query of the run: thread t owns pool p0+t and
// adds g_h * relu(dot_h) over h in order. Requires H == 16 (a query's rows are
// then the next 16 rows of q_idx). Queries of different requests in one group
// form separate runs, so any q_req is served; the launch picks this kernel
// when there are many queries.
constexpr int kScoreGroup = 16;                          // queries a CTA (N = 256)
constexpr int kScoreTilesPerCta = 8;
constexpr uint32_t kScoreQgAtom = kScoreGroup * kScoreHeads * 128;   // 32 KB
constexpr int kScoreMqSmem = 2 * kScoreKeyAtom + 2 * kScoreQgAtom + 1024;
constexpr int kScoreMqMinQueries = 256;

__global__ void __launch_bounds__(kScoreThreads)
index_scores_mq_kernel(const __grid_constant__ CUtensorMap key_map,
                       const __grid_constant__ CUtensorMap qg_map, const float *__restrict__ gate_w,
                       const int32_t *__restrict__ q_req, const int32_t *__restrict__ q_pos, int Q,
                       const uint8_t *__restrict__ pool_valid,
                       const int32_t *__restrict__ first_valid, int B, int kpool, int max_pools,
                       float *__restrict__ scores, uint8_t *__restrict__ cand) {
    extern __shared__ uint8_t sc_smem_raw[];
    __shared__ __align__(8) uint64_t q_bar, load_bar, mma_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int s_req[kScoreGroup], s_pos[kScoreGroup], s_first[kScoreGroup];
    __shared__ float s_g[kScoreGroup][kScoreHeads];

    const uint32_t raw = smem_u32(sc_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const uint32_t sK = base, sQ = base + 2 * kScoreKeyAtom;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int q0 = blockIdx.y * kScoreGroup, nq = min(kScoreGroup, Q - q0);
    const int n_tiles = (max_pools + kScorePools - 1) / kScorePools;
    const int t0 = blockIdx.x * kScoreTilesPerCta, t1 = min(n_tiles, t0 + kScoreTilesPerCta);

    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 256);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&q_bar, 1);
        mbar_init(&load_bar, 1);
        mbar_init(&mma_bar, 1);
        fence_mbarrier_init();
    }
    // the group's requests, positions and gate rows are step inputs (the gate
    // rows come from the head-gate stage: read after the wait)
    if (tid < kScoreGroup) {
        const int r = tid < nq ? q_req[q0 + tid] : -1;
        s_req[tid] = (r >= 0 && r < B) ? r : -1;
        s_pos[tid] = tid < nq ? q_pos[q0 + tid] : -1;
    }
    pdl_wait();
    pdl_launch_dependents();
    for (int i = tid; i < kScoreGroup * kScoreHeads; i += kScoreThreads)
        s_g[i / kScoreHeads][i % kScoreHeads] =
            (i / kScoreHeads) < nq ? __ldg(gate_w + (size_t)(q0 + i / kScoreHeads) * kScoreHeads + i % kScoreHeads)
                                   : 0.f;
    if (tid < kScoreGroup) s_first[tid] = s_req[tid] >= 0 ? first_valid[s_req[tid]] : 0;
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = tmem_base;

    auto load_keys = [&](int b, int t) {
        mbar_arrive_expect_tx(&load_bar, 2 * kScoreKeyAtom);
        const int row = b * max_pools + t * kScorePools;
        tma_load_2d(sK, &key_map, 0, row, &load_bar);
        tma_load_2d(sK + kScoreKeyAtom, &key_map, 64, row, &load_bar);
    };
    uint32_t n_load = 0, n_mma = 0, n_q = 0;   // completed phases of the three barriers
    bool ok = true;
    for (int j0 = 0; j0 < nq;) {
        // the run of queries j0 .. j1-1 with one request
        const int b = s_req[j0];
        int j1 = j0 + 1;
        while (j1 < nq && s_req[j1] == b) ++j1;
        const int len = j1 - j0;
        if (b >= 0 && t0 < t1) {
            if (tid == 0) {
                // the run's query rows (16 a query; rows past the array read as zeros)
                mbar_arrive_expect_tx(&q_bar, 2 * kScoreQgAtom);
                tma_load_2d(sQ, &qg_map, 0, (q0 + j0) * kScoreHeads, &q_bar);
                tma_load_2d(sQ + kScoreQgAtom, &qg_map, 64, (q0 + j0) * kScoreHeads, &q_bar);
                load_keys(b, t0);
            }
            int pos_max = -1;
            for (int j = j0; j < j1; ++j) pos_max = max(pos_max, s_pos[j]);
            const int f = s_first[j0];
            // this thread's pool in each of the CTA's tiles: validity loads all in flight
            bool pvr[kScoreTilesPerCta];
#pragma unroll
            for (int u = 0; u < kScoreTilesPerCta; ++u) {
                const int pu = (t0 + u) * kScorePools + tid;
                pvr[u] = t0 + u < t1 && pu < max_pools && pool_valid[(size_t)b * max_pools + pu] != 0;
            }
            for (int t = t0; t < t1; ++t) {
                const int p = t * kScorePools + tid;
                bool pv = false;
#pragma unroll
                for (int u = 0; u < kScoreTilesPerCta; ++u) pv = (t - t0 == u) ? pvr[u] : pv;
                const long long last = (long long)f + (long long)p * kpool + kpool - 1;
                tc::fence_before_sync();
                const bool any = __syncthreads_or(pv && last <= (long long)pos_max) != 0;
                tc::fence_after_sync();
                if (tid == 0) {
                    bool w = mbar_wait(&load_bar, n_load & 1);
                    if (t == t0) w = w && mbar_wait(&q_bar, n_q & 1);
                    if (w && any) {
                        tc::fence_after_sync();
                        const uint32_t idesc = tc::idesc_bf16(kScorePools, kScoreHeads * len, false, false);
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk) {
                            const uint32_t off_k = (kk >> 2) * kScoreKeyAtom + (kk & 3) * 32;
                            const uint32_t off_q = (kk >> 2) * kScoreQgAtom + (kk & 3) * 32;
                            tc::mma_bf16_ss(tmem, tc::desc_sw128(sK + off_k, 16, 1024),
                                            tc::desc_sw128(sQ + off_q, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                        }
                    }
                    tc::mma_commit(&mma_bar);   // arrives even when no MMA was issued
                    w = mbar_wait(&mma_bar, n_mma & 1) && w;
                    // the stage is free: the next tile's keys come in during this epilogue
                    if (w && t + 1 < t1) load_keys(b, t + 1);
                    if (!w) ok = false;
                }
                ++n_load;
                ++n_mma;
                if (t == t0) ++n_q;
                tc::fence_before_sync();
                ok = __syncthreads_and(ok) != 0;
                tc::fence_after_sync();
                // four queries' head dots a tensor-memory wait (64 columns)
                for (int jq = j0; jq < j1; jq += 4) {
                    uint32_t d[4][kScoreHeads];
                    if (any && ok) {
                        const uint32_t ta = tmem + (uint32_t)(kScoreHeads * (jq - j0)) + ((uint32_t)(32 * warp) << 16);
                        tc::tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&d[0][0]));
                        tc::tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&d[2][0]));
                        tc::tmem_wait_ld();
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = jq + u;
                        if (j >= j1) break;
                        const bool is_cand = pv && last <= (long long)s_pos[j];
                        float score = -INFINITY;
                        if (any && ok) {
                            float sacc = 0.f;
#pragma unroll
                            for (int h = 0; h < kScoreHeads; ++h)
                                sacc = fmaf(s_g[j][h], fmaxf(__uint_as_float(d[u][h]), 0.f), sacc);
                            if (is_cand) score = sacc;
                        }
                        if (p < max_pools) {
                            const size_t out_i = (size_t)(q0 + j) * max_pools + p;
                            scores[out_i] = is_cand ? score : -INFINITY;
                            cand[out_i] = is_cand ? 1 : 0;
                        }
                    }
                }
                tc::fence_before_sync();
                __syncthreads();        // D is read before the next tile's MMAs overwrite it
                tc::fence_after_sync();
            }
        } else {
            // no request (or no tile): no candidates
            for (int t = t0; t < t1; ++t) {
                const int p = t * kScorePools + tid;
                if (p < max_pools)
                    for (int j = j0; j < j1; ++j) {
                        const size_t out_i = (size_t)(q0 + j) * max_pools + p;
                        scores[out_i] = -INFINITY;
                        cand[out_i] = 0;
                    }
            }
        }
        j0 = j1;
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

inline int index_scores_launch(const void *q_idx, const float *gate_w, const int32_t *q_req,
                               const int32_t *q_pos, int Q, int H, int D, const void *pool_keys,
                               const uint8_t *pool_valid, const int32_t *first_valid, int B,
                               int kpool, int max_pools, float *scores, uint8_t *cand,
                               cudaStream_t stream) {
    if (Q < 0 || H <= 0 || D <= 0 || B < 0 || kpool <= 0 || max_pools < 0)
        return DSA_ERR_INVALID_ARG;
    if (D != kD || H > kScoreHeads || kpool > DSA_MAX_KPOOL) return DSA_ERR_UNSUPPORTED;
    if (Q == 0 || max_pools == 0) return DSA_OK;
    if (Q > 65535 || (long long)B * max_pools >= (1ll << 31) || (long long)Q * H >= (1ll << 31))
        return DSA_ERR_UNSUPPORTED;
    if (!q_idx || !gate_w || !q_req || !q_pos || !scores || !cand ||
        (B > 0 && (!pool_keys || !pool_valid || !first_valid)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(gate_w, 4) || !aligned(q_req, 4) || !aligned(q_pos, 4) ||
        !aligned(pool_keys, 16) || !aligned(first_valid, 4) || !aligned(scores, 4))
        return DSA_ERR_ALIGNMENT;
    CUtensorMap key_map, q_map;
    // With B == 0 every query has no candidate and the key map is never used.
    const void *kbase = B > 0 ? pool_keys : q_idx;
    const uint64_t krows = B > 0 ? (uint64_t)B * max_pools : (uint64_t)Q * H;
    if (!make_map_bf16_2d(&key_map, kbase, krows, kD, kD * 2, 64, kScorePools) ||
        !make_map_bf16_2d(&q_map, q_idx, (uint64_t)Q * H, kD, kD * 2, 64, kScoreHeads))
        return DSA_ERR_CUDA;
    if (Q >= kScoreMqMinQueries && H == kScoreHeads) {
        // many queries: groups of 16 share their request's key tiles
        CUtensorMap qg_map;
        if (!make_map_bf16_2d(&qg_map, q_idx, (uint64_t)Q * H, kD, kD * 2, 64, kScoreGroup * kScoreHeads))
            return DSA_ERR_CUDA;
        if (!ensure_smem_attr(reinterpret_cast<const void *>(index_scores_mq_kernel), kScoreMqSmem))
            return DSA_ERR_CUDA;
        const dim3 grid(ceil_div(ceil_div(max_pools, kScorePools), kScoreTilesPerCta),
                        ceil_div(Q, kScoreGroup));
        if (launch_pdl(index_scores_mq_kernel, grid, dim3(kScoreThreads), kScoreMqSmem, stream, key_map,
                       qg_map, gate_w, q_req, q_pos, Q, pool_valid, first_valid, B, kpool, max_pools,
                       scores, cand) != cudaSuccess)
            return DSA_ERR_CUDA;
        return launch_status();
    }
    if (!ensure_smem_attr(reinterpret_cast<const void *>(index_scores_kernel), kScoreSmem))
        return DSA_ERR_CUDA;
    dim3 grid(ceil_div(max_pools, kScorePools), Q);
    if (launch_pdl(index_scores_kernel, grid, dim3(kScoreThreads), kScoreSmem, stream, key_map, q_map,
                   gate_w, q_req, q_pos, H, pool_valid, first_valid, B, kpool, max_pools, scores,
                   cand) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
