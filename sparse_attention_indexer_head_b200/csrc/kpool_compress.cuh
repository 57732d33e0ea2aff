// a2+a3. kpool_compress with the k_norm LayerNorm fused in
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" first
// arrow; traps 1-4; KERNEL_MAX_KPOOL).
//
// B200 design. The op streams the k and gate caches once (256 B per token row
// each) and writes one 256 B key per pool: it is HBM-bound, so the kernel is a
// TMA-fed stream with all arithmetic in registers:
//   * a CTA owns a tile of TP = floor(128/kpool) consecutive pools of one
//     request, i.e. up to 128 contiguous token rows of k and of gate; one
//     thread issues two 1-D bulk copies (cp.async.bulk) of those rows into
//     shared memory, completing on an mbarrier;
//   * a half-warp handles one pool; lane l owns channels 8l..8l+7 (one 16-byte
//     vector of each row), LayerNorm statistics are half-warp shuffle sums;
//   * the per-channel softmax over the kpool slots is done in fp32 registers
//     (max-subtracted, exp2 with log2(e) folded into the logits);
//   * the first valid token is found by a warp-wide ballot scan of the
//     request's validity bytes (16-byte loads).
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kCmpConsumers = 256;                 // 8 consumer warps
constexpr int kCmpThreads = kCmpConsumers + 32;   // + 1 producer warp
constexpr int kCmpTileTokens = 128;               // token rows per tile (k and gate each)
constexpr int kCmpStages = 3;
constexpr int kCmpStageBytes = 2 * kCmpTileTokens * 128 * 2;   // 64 KB: k rows | gate rows
constexpr int kD = DSA_INDEX_DIM;   // 128 channels
constexpr float kLog2e = 1.4426950408889634f;

// First index in [0, T) of request rows [rs, rs+T) whose valid byte is nonzero;
// T if none. Executed by one full warp; the result is returned to every lane.
DSA_DEVINL int first_valid_scan(const uint8_t *__restrict__ valid, int rs, int T) {
    const int lane = threadIdx.x & 31;
    const long long beg = rs, end = (long long)rs + T;
    const long long a0 = beg & ~15LL;   // 16-byte chunks covering [beg, end)
    for (long long base = a0; base < end; base += 32 * 16) {
        const long long chunk = base + 16LL * lane;
        int hit = 16;   // first nonzero byte offset within this lane's chunk
        if (chunk >= beg && chunk + 16 <= end) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(valid + chunk));
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 3; q >= 0; --q)
#pragma unroll
                for (int bb = 3; bb >= 0; --bb)
                    if ((w4[q] >> (8 * bb)) & 0xFF) hit = 4 * q + bb;
        } else if (chunk < end) {
            // partial chunk at either end of the request: byte loads inside [beg, end)
            for (int o = 15; o >= 0; --o) {
                const long long pos = chunk + o;
                if (pos >= beg && pos < end && __ldg(valid + pos) != 0) hit = o;
            }
        }
        const uint32_t ball = __ballot_sync(0xffffffffu, hit < 16);
        if (ball) {
            const int src = __ffs(ball) - 1;
            const int h = __shfl_sync(0xffffffffu, hit, src);
            return (int)(base + 16LL * src + h - beg);
        }
    }
    return T;
}

// Half-warp (16 lanes) butterfly sum; lanes of the other half-warp run their own.
DSA_DEVINL float hsum16(float v) {
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// One pool on a half-warp: lane l owns channels 8l..8l+7 of the kpool slot rows
// at krow/grow (shared memory). Returns the packed bf16 pooled key chunk (zero
// when the pool is invalid).
template <int KP>
DSA_DEVINL uint4 compress_pool(const __nv_bfloat16 *krow, const __nv_bfloat16 *grow,
                               const float *s_ape, const float (&lw)[8], const float (&lb)[8],
                               float eps, int l, bool ok) {
    // Pass 1: LayerNorm statistics and pool logits (log2 units) per slot.
    float mean[KP], rstd[KP], lg[KP][8];
#pragma unroll
    for (int s = 0; s < KP; ++s) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4 *>(krow + s * kD), x);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) sum += x[c];
        const float mu = hsum16(sum) * (1.0f / kD);
        float sq = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float d = x[c] - mu;
            sq = fmaf(d, d, sq);
        }
        const float var = hsum16(sq) * (1.0f / kD);
        mean[s] = mu;
        rstd[s] = __frsqrt_rn(var + eps);
        float g[8];
        unpack8(*reinterpret_cast<const uint4 *>(grow + s * kD), g);
        const float4 a0 = *reinterpret_cast<const float4 *>(s_ape + s * kD + 8 * l);
        const float4 a1 = *reinterpret_cast<const float4 *>(s_ape + s * kD + 8 * l + 4);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c) lg[s][c] = fmaf(g[c], kLog2e, av[c]);
    }
    // Pass 2: per-channel softmax over slots, weighted sum of the bf16 k_norm rows.
    float mx[8], den[8], acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        mx[c] = lg[0][c];
#pragma unroll
        for (int s = 1; s < KP; ++s) mx[c] = fmaxf(mx[c], lg[s][c]);
        den[c] = 0.f;
        acc[c] = 0.f;
    }
#pragma unroll
    for (int s = 0; s < KP; ++s) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4 *>(krow + s * kD), x);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float y = fmaf((x[c] - mean[s]) * rstd[s], lw[c], lb[c]);
            const float kn = round_bf16(y);
            const float e = ex2(lg[s][c] - mx[c]);
            den[c] += e;
            acc[c] = fmaf(e, kn, acc[c]);
        }
    }
    uint4 o = make_uint4(0, 0, 0, 0);
    if (ok) {
        float v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = __fdiv_rn(acc[c], den[c]);
        o.x = pack_bf16x2(v[0], v[1]);
        o.y = pack_bf16x2(v[2], v[3]);
        o.z = pack_bf16x2(v[4], v[5]);
        o.w = pack_bf16x2(v[6], v[7]);
    }
    return o;
}

struct CmpMeta {
    int b, p0, p1, n_in, f, rs;
};

// Persistent kernel: CTA c owns a contiguous range of (request, pool-tile) work
// items. Warp 8 is the producer: it finds each request's first valid token (a
// warp ballot scan, cached across the request's tiles) and streams the tile's
// contiguous k and gate rows into a 3-stage shared-memory ring with two 1-D
// bulk copies per tile. Warps 0-7 consume: a half-warp per pool.
template <int KP>
__global__ void __launch_bounds__(kCmpThreads, 1)
kpool_compress_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ gate,
                      const uint8_t *__restrict__ valid, const int32_t *__restrict__ req_start,
                      int B, int max_pools, int tiles_per_req, int n_tiles,
                      const float *__restrict__ ape, const __nv_bfloat16 *__restrict__ ln_w,
                      const __nv_bfloat16 *__restrict__ ln_b, float eps,
                      __nv_bfloat16 *__restrict__ pool_keys, int32_t *__restrict__ pool_idx,
                      uint8_t *__restrict__ pool_valid, int32_t *__restrict__ first_valid) {
    constexpr int TP = kCmpTileTokens / KP;   // pools per tile
    extern __shared__ __align__(128) uint8_t cmp_smem[];
    __shared__ __align__(16) float s_ape[KP * kD];   // ape * log2(e)
    __shared__ __align__(8) uint64_t full[kCmpStages], empty[kCmpStages];
    __shared__ CmpMeta meta[kCmpStages];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int t_begin = (int)((long long)blockIdx.x * n_tiles / G);
    const int t_end = (int)((long long)(blockIdx.x + 1) * n_tiles / G);

    if (tid == 0) {
        for (int s = 0; s < kCmpStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCmpConsumers / 32);
        }
        fence_mbarrier_init();
    }
    for (int i = tid; i < KP * kD; i += kCmpThreads) s_ape[i] = ape[i] * kLog2e;
    __syncthreads();

    if (warp == kCmpConsumers / 32) {
        // ---------------------------------------------------------------- producer warp
        int cur_b = -1, cur_f = 0, cur_rs = 0, cur_T = 0;
        for (int t = t_begin, i = 0; t < t_end; ++t, ++i) {
            const int s = i % kCmpStages;
            bool ok = true;
            if (i >= kCmpStages) ok = mbar_wait(&empty[s], ((i / kCmpStages) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int b = t / tiles_per_req, j = t - b * tiles_per_req;
            if (b != cur_b) {
                cur_rs = req_start[b];
                cur_T = max(0, req_start[b + 1] - cur_rs);
                cur_f = first_valid_scan(valid, cur_rs, cur_T);
                cur_b = b;
            }
            const int p0 = j * TP;
            const int p1 = min(p0 + TP, max_pools);
            const int n_span = min(max_pools, (cur_T - cur_f) / KP);
            const int n_in = max(0, min(p1, n_span) - p0);
            if (lane == 0) {
                meta[s] = CmpMeta{b, p0, p1, n_in, cur_f, cur_rs};
                if (n_in > 0) {
                    const uint32_t bytes = (uint32_t)(n_in * KP * kD * 2);
                    const size_t row0 = (size_t)cur_rs + cur_f + (size_t)p0 * KP;
                    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(cmp_smem + s * kCmpStageBytes);
                    mbar_arrive_expect_tx(&full[s], 2 * bytes);
                    bulk_g2s(sk, k + row0 * kD, bytes, &full[s]);
                    bulk_g2s(sk + kCmpTileTokens * kD, gate + row0 * kD, bytes, &full[s]);
                } else {
                    mbar_arrive(&full[s]);
                }
            }
            __syncwarp();
        }
        return;
    }

    // -------------------------------------------------------------------- consumer warps
    const int hw = tid >> 4;     // half-warp: one pool at a time
    const int l = tid & 15;      // channels 8l .. 8l+7
    float lw[8], lb[8];
    unpack8(ldg_nc_v4(ln_w + 8 * l), lw);
    unpack8(ldg_nc_v4(ln_b + 8 * l), lb);

    for (int t = t_begin, i = 0; t < t_end; ++t, ++i) {
        const int s = i % kCmpStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kCmpStages) & 1))) break;
        const CmpMeta m = meta[s];
        const __nv_bfloat16 *sk = reinterpret_cast<const __nv_bfloat16 *>(cmp_smem + s * kCmpStageBytes);
        const __nv_bfloat16 *sg = sk + kCmpTileTokens * kD;
        const size_t pool_base = (size_t)m.b * max_pools;
        if (m.p0 == 0 && tid == 0) first_valid[m.b] = m.f;

        // Pools of this tile past the request's span: no key, index -1, invalid.
        for (int x = m.n_in * KP + tid; x < (m.p1 - m.p0) * KP; x += kCmpConsumers)
            pool_idx[(pool_base + m.p0) * KP + x] = -1;
        for (int x = m.n_in + tid; x < m.p1 - m.p0; x += kCmpConsumers)
            pool_valid[pool_base + m.p0 + x] = 0;

        // Warp-uniform loop: the two half-warps of a warp take pools ii and ii+1;
        // a half-warp past the tile computes on a loaded row and stores nothing.
        for (int ii = 2 * warp; ii < m.n_in; ii += kCmpConsumers / 16) {
            const bool active = ii + (hw & 1) < m.n_in;
            const int pi = active ? ii + (hw & 1) : ii;
            const int p = m.p0 + pi;
            // Slot validity: lane s < KP reads the valid byte of slot token s.
            const size_t tok0 = (size_t)m.rs + m.f + (size_t)p * KP;
            const bool lane_ok = l >= KP || valid[tok0 + l] != 0;
            const uint32_t half_mask = 0xFFFFu << (tid & 16);
            const bool ok = (__ballot_sync(0xffffffffu, lane_ok) & half_mask) == half_mask;
            const uint4 o = compress_pool<KP>(sk + (size_t)pi * KP * kD + 8 * l,
                                              sg + (size_t)pi * KP * kD + 8 * l, s_ape, lw, lb,
                                              eps, l, ok);
            if (!active) continue;
            *reinterpret_cast<uint4 *>(pool_keys + (pool_base + p) * kD + 8 * l) = o;
            if (l < KP) pool_idx[(pool_base + p) * KP + l] = ok ? m.f + p * KP + l : -1;
            if (l == 0) pool_valid[pool_base + p] = ok ? 1 : 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

template <int KP>
inline int kpool_compress_launch_kp(const __nv_bfloat16 *k, const __nv_bfloat16 *gate,
                                    const uint8_t *valid, const int32_t *req_start, int B,
                                    int max_pools, const float *ape, const __nv_bfloat16 *ln_w,
                                    const __nv_bfloat16 *ln_b, float eps, __nv_bfloat16 *keys,
                                    int32_t *idx, uint8_t *pv, int32_t *fv, cudaStream_t stream) {
    constexpr int TP = kCmpTileTokens / KP;
    const int smem = kCmpStages * kCmpStageBytes;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(kpool_compress_kernel<KP>), smem))
        return DSA_ERR_CUDA;
    const int tiles_per_req = max(1, ceil_div(max_pools, TP));
    const long long n_tiles = (long long)tiles_per_req * B;
    if (n_tiles > (1ll << 30)) return DSA_ERR_UNSUPPORTED;
    const int grid = (int)std::min<long long>(n_tiles, sm_count());
    kpool_compress_kernel<KP><<<grid, kCmpThreads, smem, stream>>>(
        k, gate, valid, req_start, B, max_pools, tiles_per_req, (int)n_tiles, ape, ln_w, ln_b, eps,
        keys, idx, pv, fv);
    return launch_status();
}

inline int kpool_compress_launch(const void *k, const void *gate, const uint8_t *valid,
                                 const int32_t *req_start, int B, int D, int kpool, int max_pools,
                                 const float *ape, const void *ln_w, const void *ln_b, float eps,
                                 void *keys, int32_t *idx, uint8_t *pv, int32_t *fv,
                                 cudaStream_t stream) {
    if (B < 0 || max_pools < 0 || kpool <= 0 || D <= 0) return DSA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 1e30f) return DSA_ERR_INVALID_ARG;
    if (D != kD || kpool > DSA_MAX_KPOOL) return DSA_ERR_UNSUPPORTED;
    if (B == 0) return DSA_OK;
    if (!k || !gate || !valid || !req_start || !ape || !ln_w || !ln_b || !fv ||
        (max_pools > 0 && (!keys || !idx || !pv)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(gate, 16) || !aligned(valid, 16) || !aligned(req_start, 4) ||
        !aligned(ape, 16) || !aligned(ln_w, 16) || !aligned(ln_b, 16) || !aligned(keys, 16) ||
        !aligned(idx, 4) || !aligned(fv, 4))
        return DSA_ERR_ALIGNMENT;
    auto K = reinterpret_cast<const __nv_bfloat16 *>(k);
    auto G = reinterpret_cast<const __nv_bfloat16 *>(gate);
    auto W = reinterpret_cast<const __nv_bfloat16 *>(ln_w);
    auto Bi = reinterpret_cast<const __nv_bfloat16 *>(ln_b);
    auto O = reinterpret_cast<__nv_bfloat16 *>(keys);
#define DSA_CMP_CASE(KPV)                                                                        \
    case KPV:                                                                                    \
        return kpool_compress_launch_kp<KPV>(K, G, valid, req_start, B, max_pools, ape, W, Bi, \
                                             eps, O, idx, pv, fv, stream);
    switch (kpool) {
        DSA_CMP_CASE(1) DSA_CMP_CASE(2) DSA_CMP_CASE(3) DSA_CMP_CASE(4)
        DSA_CMP_CASE(5) DSA_CMP_CASE(6) DSA_CMP_CASE(7) DSA_CMP_CASE(8)
    }
#undef DSA_CMP_CASE
    return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa
