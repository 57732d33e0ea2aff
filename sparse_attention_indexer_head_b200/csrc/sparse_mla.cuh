// a7. NoPE MLA restricted to the selected tokens
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" last
// arrow; MASKED_ATTN_MAX_KEYS doc: the reference is dense attention under a
// set-membership mask, so gathering the selected rows is exact; trap 5: NoPE,
// the 512-wide latent row is both key and value).
//
// Split-KV decode: a query's W selected ids are cut into S contiguous splits;
// one CTA per (split, query) gathers its latent rows and runs an online
// softmax for every head, writing an unnormalised partial (O, running max m,
// running sum l); a combine kernel merges the S partials of each (query, head)
// in split order (deterministic) and writes bf16 out and the log-sum-exp.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kL = DSA_KV_LORA;      // 512
constexpr int kMlaThreads = 256;     // 8 warps
constexpr int kMlaWarps = 8;
constexpr int kMlaHeadsPerPass = 8;  // heads a warp holds accumulators for
constexpr int kMlaTargetCtas = 2 * 148;
constexpr int kMlaMinSplitTokens = 64;
// A partial row is O[512], m, l, padded to 516 floats so every row starts on a
// 16-byte boundary (float4 stores).
constexpr int kPartStride = kL + 4;

inline int mla_num_splits(int Q, int W) {
    if (Q <= 0 || W <= 0) return 1;
    const int want = ceil_div(kMlaTargetCtas, Q);
    const int most = ceil_div(W, kMlaMinSplitTokens);
    return max(1, min(want, most));
}

inline size_t mla_part_floats(int Q, int Hm, int S) {
    return (size_t)Q * S * Hm * kPartStride;
}

inline size_t mla_workspace_bytes(int Q, int Hm, int W) {
    if (Q <= 0 || Hm <= 0) return 0;
    return mla_part_floats(Q, Hm, mla_num_splits(Q, W)) * sizeof(float);
}

__global__ void __launch_bounds__(kMlaThreads)
mla_split_kernel(const __nv_bfloat16 *__restrict__ qm, const __nv_bfloat16 *__restrict__ kv,
                 const int32_t *__restrict__ req_start, const int32_t *__restrict__ q_req,
                 const int32_t *__restrict__ token_ids, int B, int Hm, int W, int S,
                 float scale_log2, float *__restrict__ part) {
    extern __shared__ __align__(16) uint8_t mla_smem[];
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(mla_smem);   // [Hm][512]

    const int split = blockIdx.x, q = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = q_req[q];
    const bool req_ok = b >= 0 && b < B;
    const int rs = req_ok ? req_start[b] : 0;
    const int T = req_ok ? max(0, req_start[b + 1] - rs) : 0;
    const int per = (W + S - 1) / S;
    const int j0 = min(W, split * per), j1 = min(W, j0 + per);

    {
        const uint4 *src = reinterpret_cast<const uint4 *>(qm + (size_t)q * Hm * kL);
        uint4 *dst = reinterpret_cast<uint4 *>(qs);
        for (int i = tid; i < Hm * kL / 8; i += kMlaThreads) dst[i] = __ldg(src + i);
    }
    __syncthreads();

    const int heads_per_warp = Hm / kMlaWarps;   // Hm is a multiple of 16
    for (int g0 = 0; g0 < heads_per_warp; g0 += kMlaHeadsPerPass) {
        const int ng = min(kMlaHeadsPerPass, heads_per_warp - g0);
        float acc[kMlaHeadsPerPass][16];
        float m[kMlaHeadsPerPass], l[kMlaHeadsPerPass];
#pragma unroll
        for (int hh = 0; hh < kMlaHeadsPerPass; ++hh) {
            m[hh] = -INFINITY;
            l[hh] = 0.f;
#pragma unroll
            for (int d = 0; d < 16; ++d) acc[hh][d] = 0.f;
        }
        for (int j = j0; j < j1; ++j) {
            const int id = token_ids[(size_t)q * W + j];
            if (id < 0 || id >= T) continue;   // warp-uniform
            const uint4 *row = reinterpret_cast<const uint4 *>(kv + ((size_t)rs + id) * kL + 16 * lane);
            float x[16];
            unpack8(__ldg(row), *reinterpret_cast<float(*)[8]>(x));
            unpack8(__ldg(row + 1), *reinterpret_cast<float(*)[8]>(x + 8));
#pragma unroll
            for (int hh = 0; hh < kMlaHeadsPerPass; ++hh) {
                if (hh >= ng) break;
                const int h = warp + kMlaWarps * (g0 + hh);
                const uint4 *qr = reinterpret_cast<const uint4 *>(qs + (size_t)h * kL + 16 * lane);
                float qv[16];
                unpack8(qr[0], *reinterpret_cast<float(*)[8]>(qv));
                unpack8(qr[1], *reinterpret_cast<float(*)[8]>(qv + 8));
                float dot = 0.f;
#pragma unroll
                for (int d = 0; d < 16; ++d) dot = fmaf(qv[d], x[d], dot);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                const float z = dot * scale_log2;
                const float mn = fmaxf(m[hh], z);
                const float alpha = ex2(m[hh] - mn);
                const float p = ex2(z - mn);
                l[hh] = fmaf(l[hh], alpha, p);
#pragma unroll
                for (int d = 0; d < 16; ++d) acc[hh][d] = fmaf(acc[hh][d], alpha, p * x[d]);
                m[hh] = mn;
            }
        }
#pragma unroll
        for (int hh = 0; hh < kMlaHeadsPerPass; ++hh) {
            if (hh >= ng) break;
            const int h = warp + kMlaWarps * (g0 + hh);
            float *po = part + (((size_t)q * S + split) * Hm + h) * kPartStride;
            float4 *dst = reinterpret_cast<float4 *>(po + 16 * lane);
#pragma unroll
            for (int d4 = 0; d4 < 4; ++d4)
                dst[d4] = make_float4(acc[hh][4 * d4], acc[hh][4 * d4 + 1], acc[hh][4 * d4 + 2],
                                      acc[hh][4 * d4 + 3]);
            if (lane == 0) {
                po[kL] = m[hh];
                po[kL + 1] = l[hh];
            }
        }
    }
}

// One CTA per (head, query); 128 threads x 4 channels.
__global__ void __launch_bounds__(128)
mla_combine_kernel(const float *__restrict__ part, int Hm, int S, __nv_bfloat16 *__restrict__ out,
                   float *__restrict__ lse) {
    const int h = blockIdx.x, q = blockIdx.y, tid = threadIdx.x;
    const float *base = part + ((size_t)q * S * Hm + h) * kPartStride;
    const size_t sstride = (size_t)Hm * kPartStride;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, base[s * sstride + kL]);
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    float lsum = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < S; ++s) {
            const float *ps = base + s * sstride;
            const float ms = ps[kL];
            if (ms == -INFINITY) continue;
            const float w = ex2(ms - M);
            lsum = fmaf(ps[kL + 1], w, lsum);
            const float4 v = *reinterpret_cast<const float4 *>(ps + 4 * tid);
            o[0] = fmaf(v.x, w, o[0]);
            o[1] = fmaf(v.y, w, o[1]);
            o[2] = fmaf(v.z, w, o[2]);
            o[3] = fmaf(v.w, w, o[3]);
        }
    }
    const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(o[0] * inv, o[1] * inv);
    packed.y = pack_bf16x2(o[2] * inv, o[3] * inv);
    *reinterpret_cast<uint2 *>(out + ((size_t)q * Hm + h) * kL + 4 * tid) = packed;
    if (lse && tid == 0)
        lse[(size_t)q * Hm + h] = lsum > 0.f ? (M + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
}

inline int sparse_mla_launch(const void *q, const void *kv, const int32_t *req_start,
                             const int32_t *q_req, const int32_t *token_ids, int Q, int B, int Hm,
                             int W, int kv_lora, int rope_dim, float sm_scale, void *out,
                             float *lse, void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (Q < 0 || B < 0 || Hm <= 0 || W < 0 || kv_lora <= 0 || rope_dim < 0)
        return DSA_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || sm_scale == INFINITY || sm_scale == -INFINITY)
        return DSA_ERR_INVALID_ARG;
    if (kv_lora != kL || rope_dim != 0 || Hm % 16 != 0 || Hm > DSA_MAX_MLA_HEADS)
        return DSA_ERR_UNSUPPORTED;
    if (Q == 0) return DSA_OK;
    if (Q > 65535) return DSA_ERR_UNSUPPORTED;
    if (!q || !q_req || !out || (W > 0 && !token_ids) || (B > 0 && (!kv || !req_start)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(req_start, 4) || !aligned(q_req, 4) ||
        !aligned(token_ids, 4) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(ws, 16))
        return DSA_ERR_ALIGNMENT;
    const int S = mla_num_splits(Q, W);
    if (!ws || ws_bytes < mla_workspace_bytes(Q, Hm, W)) return DSA_ERR_WORKSPACE;
    float *part = reinterpret_cast<float *>(ws);
    const int smem = Hm * kL * 2;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(mla_split_kernel), smem))
        return DSA_ERR_CUDA;
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    mla_split_kernel<<<dim3(S, Q), kMlaThreads, smem, stream>>>(
        reinterpret_cast<const __nv_bfloat16 *>(q), reinterpret_cast<const __nv_bfloat16 *>(kv),
        req_start, q_req, token_ids, B, Hm, W, S, scale_log2, part);
    int st = launch_status();
    if (st != DSA_OK) return st;
    mla_combine_kernel<<<dim3(Hm, Q), 128, 0, stream>>>(part, Hm, S,
                                                          reinterpret_cast<__nv_bfloat16 *>(out),
                                                          lse);
    return launch_status();
}

}  // namespace dsa
