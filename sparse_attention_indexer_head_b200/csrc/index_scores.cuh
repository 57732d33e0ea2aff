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
