// f1. kpool_compress over the pools that hold a token range of each request
// (the pooled keys updated in place where a step's new tokens landed, instead
// of compressed anew: PR #290 page, the later commit that keeps the
// KPOOL_UPDATE_DIRECT_POS knob in the profile). The pool arithmetic is the full
// kernel's (kpool_compress.cuh), shared function by function, so a recomputed
// pool has the same bits.
#pragma once

#include "kpool_compress.cuh"

namespace dsa {

// Those pools are computed exactly as the full kernel computes them and
// first_valid is written; every other pool is left as it was. When
// first_valid[b] as held before the call differs from the request's first
// valid token now, the pool grid has moved and every pool of the request is
// recomputed.
//
// One CTA (four warps) per request; a half-warp per pool: its kpool k and gate
// rows are staged in shared memory, their LayerNorm statistics taken a lane a
// row (row_stats, in the full kernel's read order), then the same slot softmax
// and pooling as the full kernel (compress_pool).
constexpr int kTokWarps = 4;

template <int KP>
__global__ void __launch_bounds__(kTokWarps * 32)
kpool_compress_tokens_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ gate,
                             const uint8_t *__restrict__ valid, const int32_t *__restrict__ req_start,
                             int max_pools, const int32_t *__restrict__ tok_begin,
                             const int32_t *__restrict__ tok_end, const float *__restrict__ ape,
                             const __nv_bfloat16 *__restrict__ ln_w, const __nv_bfloat16 *__restrict__ ln_b,
                             float eps, __nv_bfloat16 *__restrict__ pool_keys,
                             int32_t *__restrict__ pool_idx, uint8_t *__restrict__ pool_valid,
                             int32_t *__restrict__ first_valid) {
    constexpr int kHW = kTokWarps * 2;                     // half-warps: pools per round
    __shared__ __align__(16) float s_ape[KP * kD];         // ape * log2(e), [slot][half][lane][4]
    __shared__ __align__(16) __nv_bfloat16 s_rows[kHW][2][KP][kD];   // per half-warp: k rows, gate rows
    __shared__ __align__(16) float4 s_st[kHW][KP];         // per half-warp: stat_pairs
    __shared__ int s_f, s_fold, s_tb, s_te;

    const int b = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hw = tid >> 4, l = tid & 15;
    for (int i = tid; i < KP * kD; i += kTokWarps * 32) {
        const int sl = i / kD, c = i % kD;
        s_ape[(sl * 2 + ((c >> 2) & 1)) * 64 + 4 * (c >> 3) + (c & 3)] = ape[i] * kLog2e;
    }
    pdl_wait();
    pdl_launch_dependents();
    float2 lw[4], lb[4];
    unpack8x2(ldg_nc_v4(ln_w + 8 * l), lw);
    unpack8x2(ldg_nc_v4(ln_b + 8 * l), lb);

    const int rs = req_start[b];
    const int T = max(0, req_start[b + 1] - rs);
    if (warp == 0) {
        const int f = first_valid_scan(valid, rs, T);
        if (lane == 0) s_f = f;
    } else if (tid == 32) {        // the request's range and previous first valid token, meanwhile
        s_tb = tok_begin[b];
        s_te = tok_end[b];
        s_fold = first_valid[b];
    }
    __syncthreads();
    const int f = s_f;
    if (tid == 0) first_valid[b] = f;
    if (max_pools <= 0) return;
    const int n_span = min(max_pools, (T - f) / KP);
    int p_lo = 0, p_hi = max_pools - 1;
    if (s_fold == f) {             // a first valid token that moved shifts every pool: all of them
        const int tb = max(s_tb, 0), te = min(s_te, T);
        if (te <= tb || te - 1 < f) return;      // no pool holds the range
        p_lo = tb > f ? (tb - f) / KP : 0;
        p_hi = min(max_pools - 1, (te - 1 - f) / KP);
    }
    const size_t pool_base = (size_t)b * max_pools;

    for (int p0 = p_lo; p0 <= p_hi; p0 += kHW) {          // uniform over the block
        const int p = p0 + hw;
        const bool act = p <= p_hi, in_span = act && p < n_span;
        const size_t row0 = (size_t)rs + f + (size_t)p * KP;
        if (in_span) {
#pragma unroll
            for (int sl = 0; sl < KP; ++sl) {
                *reinterpret_cast<uint4 *>(&s_rows[hw][0][sl][8 * l]) =
                    ldg_nc_v4(k + (row0 + sl) * kD + 8 * l);
                *reinterpret_cast<uint4 *>(&s_rows[hw][1][sl][8 * l]) =
                    ldg_nc_v4(gate + (row0 + sl) * kD + 8 * l);
            }
        }
        __syncwarp();
        // LayerNorm statistics of the pool's rows, lane l < KP of each half-warp
        // taking row l. The full kernel keys a row's read order by its index in
        // its tile of CmpCfg<KP>::kTP pools; the same key gives the same bits.
        if (in_span && l < KP) {
            const int tok_in_tile = (p % CmpCfg<KP>::kTP) * KP + l;
            s_st[hw][l] = stat_pairs(row_stats(&s_rows[hw][0][l][0], tok_in_tile & 7, eps));
        }
        __syncwarp();
        // pool valid iff every slot token is valid
        const bool tv = in_span && l < KP && valid[row0 + l] != 0;
        const uint32_t ball = __ballot_sync(0xffffffffu, tv);
        const uint32_t mine = (ball >> (16 * (hw & 1))) & ((1u << KP) - 1u);
        const bool ok = in_span && mine == (1u << KP) - 1u;
        const uint4 o = compress_pool<KP>(&s_rows[hw][0][0][8 * l], &s_rows[hw][1][0][8 * l],
                                          &s_st[hw][0], s_ape, lw, lb, l, ok);
        if (act) {
            if (in_span) *reinterpret_cast<uint4 *>(pool_keys + (pool_base + p) * kD + 8 * l) = o;
            if (l < KP) pool_idx[(pool_base + p) * KP + l] = ok ? f + p * KP + l : -1;
            if (l == 0) pool_valid[pool_base + p] = ok ? 1 : 0;
        }
        __syncwarp();
    }
}

template <int KP>
inline int kpool_compress_tokens_launch_kp(const __nv_bfloat16 *k, const __nv_bfloat16 *gate,
                                           const uint8_t *valid, const int32_t *req_start, int B,
                                           int max_pools, const int32_t *tok_begin,
                                           const int32_t *tok_end, const float *ape,
                                           const __nv_bfloat16 *ln_w, const __nv_bfloat16 *ln_b,
                                           float eps, __nv_bfloat16 *keys, int32_t *idx, uint8_t *pv,
                                           int32_t *fv, cudaStream_t stream) {
    if (launch_pdl(kpool_compress_tokens_kernel<KP>, dim3(B), dim3(kTokWarps * 32), 0, stream, k,
                   gate, valid, req_start, max_pools, tok_begin, tok_end, ape, ln_w, ln_b, eps, keys,
                   idx, pv, fv) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

inline int kpool_compress_tokens_launch(const void *k, const void *gate, const uint8_t *valid,
                                        const int32_t *req_start, int B, int D, int kpool,
                                        int max_pools, const float *ape, const void *ln_w,
                                        const void *ln_b, float eps, const int32_t *tok_begin,
                                        const int32_t *tok_end, void *keys, int32_t *idx,
                                        uint8_t *pv, int32_t *fv, cudaStream_t stream) {
    if (B < 0 || max_pools < 0 || kpool <= 0 || D <= 0) return DSA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1e30f) return DSA_ERR_INVALID_ARG;
    if (D != kD || kpool > DSA_MAX_KPOOL) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (B > (1 << 30)) return DSA_ERR_UNSUPPORTED;
    if (!k || !gate || !valid || !req_start || !ape || !ln_w || !ln_b || !fv || !tok_begin ||
        !tok_end || (max_pools > 0 && (!keys || !idx || !pv)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(gate, 16) || !aligned(valid, 16) || !aligned(req_start, 4) ||
        !aligned(ape, 16) || !aligned(ln_w, 16) || !aligned(ln_b, 16) || !aligned(keys, 16) ||
        !aligned(idx, 4) || !aligned(fv, 4) || !aligned(tok_begin, 4) || !aligned(tok_end, 4))
        return DSA_ERR_ALIGNMENT;
    auto K = reinterpret_cast<const __nv_bfloat16 *>(k);
    auto G = reinterpret_cast<const __nv_bfloat16 *>(gate);
    auto W = reinterpret_cast<const __nv_bfloat16 *>(ln_w);
    auto Bi = reinterpret_cast<const __nv_bfloat16 *>(ln_b);
    auto O = reinterpret_cast<__nv_bfloat16 *>(keys);
#define DSA_TOK_CASE(KPV)                                                                        \
    case KPV:                                                                                    \
        return kpool_compress_tokens_launch_kp<KPV>(K, G, valid, req_start, B, max_pools,        \
                                                    tok_begin, tok_end, ape, W, Bi, eps, O, idx, \
                                                    pv, fv, stream);
    switch (kpool) {
        DSA_TOK_CASE(1) DSA_TOK_CASE(2) DSA_TOK_CASE(3) DSA_TOK_CASE(4)
        DSA_TOK_CASE(5) DSA_TOK_CASE(6) DSA_TOK_CASE(7) DSA_TOK_CASE(8)
    }
#undef DSA_TOK_CASE
    return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
