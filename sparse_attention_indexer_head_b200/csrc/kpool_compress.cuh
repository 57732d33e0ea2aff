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

constexpr int kCmpThreads = 256;
constexpr int kCmpTileTokens = 128;
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

template <int KP>
__global__ void __launch_bounds__(kCmpThreads)
kpool_compress_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ gate,
                      const uint8_t *__restrict__ valid, const int32_t *__restrict__ req_start,
                      int B, int max_pools, const float *__restrict__ ape,
                      const __nv_bfloat16 *__restrict__ ln_w, const __nv_bfloat16 *__restrict__ ln_b,
                      float eps, __nv_bfloat16 *__restrict__ pool_keys,
                      int32_t *__restrict__ pool_idx, uint8_t *__restrict__ pool_valid,
                      int32_t *__restrict__ first_valid) {
    constexpr int TP = kCmpTileTokens / KP;   // pools per tile
    extern __shared__ __align__(128) uint8_t cmp_smem[];
    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(cmp_smem);
    __nv_bfloat16 *sg = sk + TP * KP * kD;
    __shared__ __align__(16) float s_ape[KP * kD];   // ape * log2(e)
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_f;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int b = blockIdx.y;
    const int p0 = blockIdx.x * TP;

    const int rs = req_start[b];
    const int T = max(0, req_start[b + 1] - rs);
    if (warp == 0) {
        const int f = first_valid_scan(valid, rs, T);
        if (tid == 0) {
            s_f = f;
            mbar_init(&bar, 1);
            fence_mbarrier_init();
        }
    }
    for (int i = tid; i < KP * kD; i += kCmpThreads) s_ape[i] = ape[i] * kLog2e;
    __syncthreads();
    const int f = s_f;
    if (blockIdx.x == 0 && tid == 0) first_valid[b] = f;
    if (p0 >= max_pools) return;

    const int n_span = min(max_pools, (T - f) / KP);
    const int p1 = min(p0 + TP, max_pools);
    const int n_in = max(0, min(p1, n_span) - p0);   // pools of this tile inside the request

    if (n_in > 0 && tid == 0) {
        const uint32_t bytes = (uint32_t)(n_in * KP * kD * 2);
        const size_t row0 = (size_t)rs + f + (size_t)p0 * KP;
        mbar_arrive_expect_tx(&bar, 2 * bytes);
        bulk_g2s(sk, k + row0 * kD, bytes, &bar);
        bulk_g2s(sg, gate + row0 * kD, bytes, &bar);
    }

    // Pools of this tile past the request's span: no key, index -1, invalid.
    const size_t pool_base = (size_t)b * max_pools;
    for (int i = n_in * KP + tid; i < (p1 - p0) * KP; i += kCmpThreads)
        pool_idx[(pool_base + p0) * KP + i] = -1;
    for (int i = n_in + tid; i < p1 - p0; i += kCmpThreads) pool_valid[pool_base + p0 + i] = 0;
    if (n_in == 0) return;

    const int hw = tid >> 4;     // half-warp: one pool at a time
    const int l = tid & 15;      // channels 8l .. 8l+7
    float lw[8], lb[8];
    unpack8(ldg_nc_v4(ln_w + 8 * l), lw);
    unpack8(ldg_nc_v4(ln_b + 8 * l), lb);

    if (!mbar_wait(&bar, 0)) return;

    // Warp-uniform loop: the two half-warps of a warp take pools ii and ii+1;
    // a half-warp past the tile computes on a loaded row and stores nothing.
    for (int ii = 2 * warp; ii < n_in; ii += kCmpThreads / 16) {
        const bool active = ii + (hw & 1) < n_in;
        const int i = active ? ii + (hw & 1) : ii;
        const int p = p0 + i;
        const __nv_bfloat16 *krow = sk + (size_t)i * KP * kD + 8 * l;
        const __nv_bfloat16 *grow = sg + (size_t)i * KP * kD + 8 * l;

        // Slot validity: lane s < KP reads the valid byte of slot token s.
        const size_t tok0 = (size_t)rs + f + (size_t)p * KP;
        const bool lane_ok = l >= KP || valid[tok0 + l] != 0;
        const uint32_t half_mask = 0xFFFFu << (tid & 16);
        const bool ok = (__ballot_sync(0xffffffffu, lane_ok) & half_mask) == half_mask;

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
        if (!active) continue;
        *reinterpret_cast<uint4 *>(pool_keys + (pool_base + p) * kD + 8 * l) = o;
        if (l < KP) pool_idx[(pool_base + p) * KP + l] = ok ? f + p * KP + l : -1;
        if (l == 0) pool_valid[pool_base + p] = ok ? 1 : 0;
    }
}

template <int KP>
inline int kpool_compress_launch_kp(const __nv_bfloat16 *k, const __nv_bfloat16 *gate,
                                    const uint8_t *valid, const int32_t *req_start, int B,
                                    int max_pools, const float *ape, const __nv_bfloat16 *ln_w,
                                    const __nv_bfloat16 *ln_b, float eps, __nv_bfloat16 *keys,
                                    int32_t *idx, uint8_t *pv, int32_t *fv, cudaStream_t stream) {
    constexpr int TP = kCmpTileTokens / KP;
    const int smem = 2 * TP * KP * kD * 2;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(kpool_compress_kernel<KP>), smem))
        return DSA_ERR_CUDA;
    dim3 grid(max(1, ceil_div(max_pools, TP)), B);
    kpool_compress_kernel<KP><<<grid, kCmpThreads, smem, stream>>>(
        k, gate, valid, req_start, B, max_pools, ape, ln_w, ln_b, eps, keys, idx, pv, fv);
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
    if (B > 65535) return DSA_ERR_UNSUPPORTED;
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
