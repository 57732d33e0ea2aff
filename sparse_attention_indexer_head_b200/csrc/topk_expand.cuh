// a5+a6. topk_pools + expand_selection
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" third and
// fourth arrows; Glm5NextDsaConfig::select_k / out_width; trap 6, the -1
// sentinel row written in full).
//
// One CTA per query. Scores become order-preserving uint32 keys (candidates
// only; -0 folded onto +0, NaN onto -inf, non-candidates 0). A 4-pass 8-bit
// MSB radix select finds the n_q-th largest key tau exactly; the winners are
// every key above tau plus the lowest-id keys equal to tau (an id-ordered
// block scan), compacted into shared memory as (key << 32 | ~id) and bitonic
// sorted, so the order is (score desc, pool id asc) and the result is
// bit-exact and deterministic. The expansion gathers pool_idx rows and writes
// every slot of the [select_k * kpool] row, -1 past n_q.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkSmemKeys = 32768;   // pools whose keys are cached in shared memory

DSA_DEVINL uint32_t score_key(float s, bool is_cand) {
    if (!is_cand) return 0u;
    if (s != s) s = -INFINITY;      // NaN ranks as -inf
    if (s == 0.f) s = 0.f;          // -0 ranks as +0
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of v over the block (thread order); *total gets the sum.
DSA_DEVINL int block_excl_scan(int v, int *s_warp, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kTopkWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < kTopkWarps) s_warp[lane] = w;   // inclusive warp totals
    }
    __syncthreads();
    const int before = (warp ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[kTopkWarps - 1];
    __syncthreads();
    return before;
}

// One warp-local bitonic stage in registers: v is element i, its partner is
// i ^ stride (same warp since stride < 32); the lower index of a pair keeps the
// larger key when the run of `size` containing it sorts descending.
DSA_DEVINL unsigned long long bitonic_reg_stage(unsigned long long v, int i, int size, int stride) {
    const unsigned long long p = __shfl_xor_sync(0xffffffffu, v, stride);
    const bool desc = (i & size) == 0;
    const bool lower = (i & stride) == 0;
    const bool keep_max = lower == desc;
    return keep_max ? (v > p ? v : p) : (v < p ? v : p);
}

// In-place descending bitonic sort of a[0..n2) in shared memory (n2 a power of
// two, at most 8 * kTopkThreads). Called by the whole block.
DSA_DEVINL void bitonic_sort_desc(unsigned long long *a, int n2) {
    const int tid = threadIdx.x;
    const int R = (n2 + kTopkThreads - 1) / kTopkThreads;   // elements per thread
    auto reg_round = [&](int size_lo, int size_hi, int first_stride) {
        // sizes size_lo..size_hi (powers of two); the first size starts at
        // first_stride, later ones at size/2; every stride here is < 32.
        for (int r = 0; r < R; ++r) {
            const int i = tid + r * kTopkThreads;
            unsigned long long v = i < n2 ? a[i] : 0ull;
            for (int size = size_lo; size <= size_hi; size <<= 1)
                for (int stride = (size == size_lo ? first_stride : size >> 1); stride > 0; stride >>= 1)
                    v = bitonic_reg_stage(v, i, size, stride);
            if (i < n2) a[i] = v;
        }
    };
    __syncthreads();
    reg_round(2, min(n2, 32), 1);
    for (int size = 64; size <= n2; size <<= 1) {
        for (int stride = size >> 1; stride >= 32; stride >>= 1) {
            __syncthreads();
            for (int i = tid; i < n2; i += kTopkThreads) {
                const int l = i ^ stride;
                if (l > i) {
                    const unsigned long long x = a[i], y = a[l];
                    const bool desc = (i & size) == 0;
                    if (desc ? (x < y) : (x > y)) {
                        a[i] = y;
                        a[l] = x;
                    }
                }
            }
        }
        __syncthreads();
        reg_round(size, size, 16);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads)
topk_expand_kernel(const float *__restrict__ scores, const uint8_t *__restrict__ cand,
                   const int32_t *__restrict__ pool_idx, const int32_t *__restrict__ q_req, int B,
                   int P, int KP, int K, int n2max, int keys_in_smem,
                   int32_t *__restrict__ top_pools, int32_t *__restrict__ token_ids) {
    extern __shared__ __align__(16) uint8_t topk_smem[];
    unsigned long long *slist = reinterpret_cast<unsigned long long *>(topk_smem);   // [n2max]
    uint32_t *skeys = reinterpret_cast<uint32_t *>(slist + n2max);             // [P] if cached
    __shared__ int hist[256];
    __shared__ int s_warp[kTopkWarps];
    __shared__ int s_pick[2];

    const int tid = threadIdx.x;
    const int q = blockIdx.x;
    const int b = q_req[q];
    const bool req_ok = b >= 0 && b < B;
    const float *srow = scores + (size_t)q * P;
    const uint8_t *crow = cand + (size_t)q * P;

    auto key_at = [&](int p) -> uint32_t {
        if (keys_in_smem) return skeys[p];
        return req_ok ? score_key(srow[p], crow[p] != 0) : 0u;
    };

    // Keys: four loads of each array in flight per thread before any use.
    int cnt = 0;
    for (int p0 = 0; p0 < P; p0 += 4 * kTopkThreads) {
        float sv[4];
        uint8_t cv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = p0 + tid + u * kTopkThreads;
            sv[u] = (req_ok && p < P) ? srow[p] : 0.f;
            cv[u] = (req_ok && p < P) ? crow[p] : (uint8_t)0;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = p0 + tid + u * kTopkThreads;
            const uint32_t k = score_key(sv[u], cv[u] != 0);
            if (keys_in_smem && p < P) skeys[p] = k;
            cnt += k != 0u;
        }
    }
    int n_cand;
    (void)block_excl_scan(cnt, s_warp, &n_cand);
    const int nq = min(K, n_cand);

    // Radix select of the nq-th largest key.
    uint32_t prefix = 0, pmask = 0;
    int remaining = nq;
    if (nq > 0) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0;
            __syncthreads();
            // Warp-aggregated increments: lanes with the same digit elect one
            // leader, so a few crowded bins do not serialise the whole block.
            for (int base = (tid & ~31); base < P; base += kTopkThreads) {
                const int p = base + (tid & 31);
                uint32_t d = 0x100u;   // no bin
                if (p < P) {
                    const uint32_t k = key_at(p);
                    if ((k & pmask) == prefix) d = (k >> shift) & 0xFF;
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, d);
                if (d != 0x100u && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[d], __popc(peers));
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns bins 255-8l down to 248-8l
                int c[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    c[i] = hist[255 - 8 * tid - i];
                    sum += c[i];
                }
                int above = sum;   // inclusive scan over lanes (descending bins)
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, above, off);
                    if (tid >= off) above += y;
                }
                int run = above - sum;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run < remaining && remaining <= run + c[i]) {
                        s_pick[0] = 255 - 8 * tid - i;
                        s_pick[1] = run;
                    }
                    run += c[i];
                }
            }
            __syncthreads();
            remaining -= s_pick[1];
            prefix |= (uint32_t)s_pick[0] << shift;
            pmask |= 0xFFu << shift;
            __syncthreads();
        }
    }
    const uint32_t tau = prefix;   // the nq-th largest key (when nq > 0)
    const int r = remaining;       // keys equal to tau to take, lowest ids first

    // Selection in id order over contiguous per-thread chunks.
    const int chunk = (P + kTopkThreads - 1) / kTopkThreads;
    const int p_lo = min(P, tid * chunk), p_hi = min(P, p_lo + chunk);
    int gt = 0, eq = 0;
    if (nq > 0)
        for (int p = p_lo; p < p_hi; ++p) {
            const uint32_t k = key_at(p);
            gt += k > tau;
            eq += k == tau;
        }
    int tot;
    const int gt_before = block_excl_scan(gt, s_warp, &tot);
    const int eq_before = block_excl_scan(eq, s_warp, &tot);
    if (nq > 0) {
        int pos = gt_before + min(eq_before, r);
        int eqr = eq_before;
        for (int p = p_lo; p < p_hi; ++p) {
            const uint32_t k = key_at(p);
            const unsigned long long comp =
                ((unsigned long long)k << 32) | (unsigned long long)(~(uint32_t)p);
            if (k > tau) {
                slist[pos++] = comp;
            } else if (k == tau) {
                if (eqr < r) slist[pos++] = comp;
                ++eqr;
            }
        }
    }
    int n2 = 1;
    while (n2 < nq) n2 <<= 1;
    for (int i = nq + tid; i < n2; i += kTopkThreads) slist[i] = 0ull;
    __syncthreads();

    // Bitonic sort, descending, of n2 (a power of two, <= 4096) composite keys.
    // Element i lives with thread i mod 512. Stages whose partner distance is
    // below 32 stay inside a warp and run in registers with shuffles; the
    // others (partner distance >= 32) run in shared memory between block
    // barriers: 10 of the 45 stages for 512 elements.
    bitonic_sort_desc(slist, n2);
    for (int j = tid; j < K; j += kTopkThreads)
        top_pools[(size_t)q * K + j] = j < nq ? (int32_t)(~(uint32_t)slist[j]) : -1;
    // Expansion: four pool_idx gathers in flight per thread before the stores.
    for (int e0 = 0; e0 < K * KP; e0 += 4 * kTopkThreads) {
        int32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + tid + u * kTopkThreads;
            const int j = e / KP, s = e - j * KP;
            v[u] = -1;
            if (e < K * KP && j < nq) {
                const int pid = (int)(~(uint32_t)slist[j]);
                v[u] = pool_idx[((size_t)b * P + pid) * KP + s];
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + tid + u * kTopkThreads;
            if (e < K * KP) token_ids[(size_t)q * K * KP + e] = v[u];
        }
    }
}

inline int topk_expand_launch(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                              const int32_t *q_req, int Q, int B, int max_pools, int kpool,
                              int select_k, int32_t *top_pools, int32_t *token_ids,
                              cudaStream_t stream) {
    if (Q < 0 || B < 0 || max_pools < 0 || kpool <= 0 || select_k < 0) return DSA_ERR_INVALID_ARG;
    if (kpool > DSA_MAX_KPOOL || select_k > DSA_MAX_SELECT) return DSA_ERR_UNSUPPORTED;
    if (Q == 0 || select_k == 0) return DSA_OK;
    if (!q_req || !top_pools || !token_ids ||
        (max_pools > 0 && (!scores || !cand || (B > 0 && !pool_idx))))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(pool_idx, 4) || !aligned(q_req, 4) ||
        !aligned(top_pools, 4) || !aligned(token_ids, 4))
        return DSA_ERR_ALIGNMENT;
    int n2max = 1;
    while (n2max < select_k) n2max <<= 1;
    const int keys_in_smem = max_pools <= kTopkSmemKeys ? 1 : 0;
    const int smem = n2max * 8 + (keys_in_smem ? max_pools * 4 : 0);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(topk_expand_kernel), smem))
        return DSA_ERR_CUDA;
    topk_expand_kernel<<<Q, kTopkThreads, smem, stream>>>(scores, cand, pool_idx, q_req, B,
                                                          max_pools, kpool, select_k, n2max,
                                                          keys_in_smem, top_pools, token_ids);
    return launch_status();
}

}  // namespace dsa
