// a4. index_scores: [Q, P] head-gated ReLU dot scores plus candidate validity
// ("spark_model/layers/glm5next_dsa/mod.rs", "Shape of the pipeline", second
// arrow).
//
// Per query q of request b and pool p:
//   cand = pool_valid[b,p] && last slot token of p <= q_pos[q]
//   score = sum_h gate_w[q,h] * max(0, <q_idx[q,h,:], key[b,p,:]>), -inf if !cand.
//
// Kernel: a CTA scores 32 pools of one query with four threads per pool (four
// heads each). The query (16 heads x 128 channels) sits transposed in shared
// memory as fp32; the pool key row is read with 16-byte loads. Keys of
// non-candidates are never read.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kScoreThreads = 128;                   // 32 pools x 4 head groups
constexpr int kScorePools = kScoreThreads / 4;
constexpr int kScoreHeads = DSA_MAX_INDEX_HEADS;     // 16

// Thread (pool, hq) computes heads 4hq..4hq+3 of one pool over all 128
// channels (two interleaved fp32 chains per head), adds g_h * relu(dot_h) for
// its heads, and the four head groups of a pool are folded with two shuffles
// in a fixed order. The four lanes of a pool read the same 256-byte key row
// (served by L1 after the first); q is read from shared memory as one
// broadcast 16-byte load per channel.
__global__ void __launch_bounds__(kScoreThreads)
index_scores_kernel(const __nv_bfloat16 *__restrict__ q_idx, const float *__restrict__ gate_w,
                    const int32_t *__restrict__ q_req, const int32_t *__restrict__ q_pos, int H,
                    const __nv_bfloat16 *__restrict__ pool_keys,
                    const uint8_t *__restrict__ pool_valid,
                    const int32_t *__restrict__ first_valid, int B, int kpool, int max_pools,
                    float *__restrict__ scores, uint8_t *__restrict__ cand) {
    __shared__ __align__(16) float qs[kD * kScoreHeads];   // qs[c][h]
    __shared__ float gs[kScoreHeads];

    const int q = blockIdx.y;
    const int tid = threadIdx.x;
    const int b = q_req[q];
    const bool req_ok = b >= 0 && b < B;

    // 16 heads x 16 vectors of 8 channels: coalesced 16-byte loads, stored transposed.
    for (int i = tid; i < kScoreHeads * (kD / 8); i += kScoreThreads) {
        const int h = i % kScoreHeads, c8 = i / kScoreHeads;   // consecutive threads: heads
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (req_ok && h < H) unpack8(ldg_nc_v4(q_idx + ((size_t)q * H + h) * kD + 8 * c8), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) qs[(8 * c8 + e) * kScoreHeads + h] = x[e];
    }
    if (tid < kScoreHeads) gs[tid] = (req_ok && tid < H) ? gate_w[(size_t)q * H + tid] : 0.f;
    __syncthreads();

    const int hq = tid & 3;
    const int p = blockIdx.x * kScorePools + (tid >> 2);
    bool is_cand = false;
    if (req_ok && p < max_pools) {
        const long long last = (long long)first_valid[b] + (long long)p * kpool + kpool - 1;
        is_cand = pool_valid[(size_t)b * max_pools + p] != 0 && last <= (long long)q_pos[q];
    }
    float part = 0.f;
    if (is_cand) {
        const __nv_bfloat16 *key = pool_keys + ((size_t)b * max_pools + p) * kD;
        uint4 kr[kD / 8];   // the whole key row: 16 loads in flight at once
#pragma unroll
        for (int c8 = 0; c8 < kD / 8; ++c8) kr[c8] = ldg_nc_v4(key + 8 * c8);
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int c8 = 0; c8 < kD / 8; ++c8) {
            float kv[8];
            unpack8(kr[c8], kv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 qv = *reinterpret_cast<const float4 *>(qs + (8 * c8 + j) * kScoreHeads + 4 * hq);
                float *a = acc[j & 1];
                a[0] = fmaf(qv.x, kv[j], a[0]);
                a[1] = fmaf(qv.y, kv[j], a[1]);
                a[2] = fmaf(qv.z, kv[j], a[2]);
                a[3] = fmaf(qv.w, kv[j], a[3]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
            part = fmaf(gs[4 * hq + u], fmaxf(acc[0][u] + acc[1][u], 0.f), part);
    }
    // Fold the four head groups of the pool: (g0 + g1) + (g2 + g3).
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (hq == 0 && p < max_pools) {
        const size_t out_i = (size_t)q * max_pools + p;
        scores[out_i] = is_cand ? part : -INFINITY;
        cand[out_i] = is_cand ? 1 : 0;
    }
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
    if (Q > 65535) return DSA_ERR_UNSUPPORTED;
    if (!q_idx || !gate_w || !q_req || !q_pos || !scores || !cand ||
        (B > 0 && (!pool_keys || !pool_valid || !first_valid)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(gate_w, 4) || !aligned(q_req, 4) || !aligned(q_pos, 4) ||
        !aligned(pool_keys, 16) || !aligned(first_valid, 4) || !aligned(scores, 4))
        return DSA_ERR_ALIGNMENT;
    dim3 grid(ceil_div(max_pools, kScorePools), Q);
    index_scores_kernel<<<grid, kScoreThreads, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16 *>(q_idx), gate_w, q_req, q_pos, H,
        reinterpret_cast<const __nv_bfloat16 *>(pool_keys), pool_valid, first_valid, B, kpool,
        max_pools, scores, cand);
    return launch_status();
}

}  // namespace dsa
