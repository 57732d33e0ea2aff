// a5+a6. topk_pools + expand_selection
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" third and
// fourth arrows; Glm5NextDsaConfig::select_k / out_width; trap 6, the -1
// sentinel row written in full).
//
// One CTA per query. Scores become order-preserving uint32 keys (candidates
// only; -0 folded onto +0, NaN onto -inf, non-candidates 0). An 8-bit MSB
// radix select finds the n_q-th largest key tau exactly: two passes, then,
// when at most 32 keys share those 16 bits with tau, a rank among them on one
// warp, else two more passes; the winners are
// every key above tau plus the lowest-id keys equal to tau (placed by warps
// over contiguous id ranges with ballot ranks), written in ascending pool id,
// so the result is bit-exact and deterministic. The expansion gathers pool_idx rows and writes every slot of
// the [select_k * kpool] row, -1 past n_q.
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

// Adds each lane's digit d (0x100: the lane has none) to a shared-memory
// histogram: one atomic for the warp when every lane that has a digit has the
// same one (the top digit of scores of one magnitude, or equal scores), else
// one atomic a lane (digits spread over the bins). Exact integer counts either
// way. Every lane of the warp calls it.
DSA_DEVINL void hist_add_warp(int *h, uint32_t d) {
    const uint32_t act = __ballot_sync(0xffffffffu, d != 0x100u);
    if (act == 0u) return;
    const int lead = __ffs(act) - 1;
    const uint32_t dl = __shfl_sync(0xffffffffu, d, lead);
    if (__all_sync(0xffffffffu, d == 0x100u || d == dl)) {
        if ((int)(threadIdx.x & 31) == lead) atomicAdd(&h[dl], __popc(act));
    } else if (d != 0x100u) {
        atomicAdd(&h[d], 1);
    }
}

// Tail slots (always_select_tail): after the K * KP pool slots, a row carries
// KP - 1 slots for the query's trailing partial pool. With f the request's first
// valid token and n = (q_pos - f + 1) mod KP tokens past the query's last
// complete pool, slot s < n holds token q_pos + 1 - n + s when it exists and is
// valid; every other tail slot is -1 (also when q_pos < f).
struct TailArgs {
    const int32_t *q_pos;
    const int32_t *first_valid;
    const uint8_t *valid;
    const int32_t *req_start;
    int slots;              // 0 (no tail) or KP - 1
};

__global__ void __launch_bounds__(kTopkThreads)
topk_expand_kernel(const float *__restrict__ scores, const uint8_t *__restrict__ cand,
                   const int32_t *__restrict__ pool_idx, const int32_t *__restrict__ q_req, int B,
                   int P, int KP, int K, int keys_in_smem, TailArgs tail,
                   int32_t *__restrict__ top_pools, int32_t *__restrict__ token_ids) {
    extern __shared__ __align__(16) uint8_t topk_smem[];
    int32_t *slist = reinterpret_cast<int32_t *>(topk_smem);                  // [K] selected ids
    uint32_t *skeys = reinterpret_cast<uint32_t *>(topk_smem) + K;           // [P] if cached
    __shared__ int hist[2][256];          // double-buffered radix histograms
    __shared__ int2 s_warp2[kTopkWarps];
    __shared__ int s_pick[2][3];          // per pass parity: (digit, count above it, count in it)
    __shared__ int s_ncand, s_nsmall, s_req;
    __shared__ uint32_t s_small[32], s_tau;

    const int tid = threadIdx.x;
    const int q = blockIdx.x;
    const int b = q_req[q];                   // a step input: read before the wait
    const bool req_ok = b >= 0 && b < B;
    pdl_wait();
    pdl_launch_dependents();
    const float *srow = scores + (size_t)q * P;
    const uint8_t *crow = cand + (size_t)q * P;

    auto key_at = [&](int p) -> uint32_t {
        if (keys_in_smem) return skeys[p];
        return req_ok ? score_key(srow[p], crow[p] != 0) : 0u;
    };

    // Keys: four loads of each array in flight per thread before any use; the
    // histogram of the top byte (the first radix pass) and the candidate count
    // are built on the way.
    if (tid < 256) {
        hist[0][tid] = 0;
        hist[1][tid] = 0;
    }
    if (tid == 0) {
        s_ncand = 0;
        s_nsmall = 0;
    }
    __syncthreads();
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
            hist_add_warp(hist[0], p < P ? (k >> 24) : 0x100u);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((tid & 31) == 0) atomicAdd(&s_ncand, cnt);
    __syncthreads();
    const int nq = min(K, s_ncand);

    // Radix select of the nq-th largest key, 8 bits per pass, most significant
    // first. Pass i builds its histogram in hist[i & 1] (cleared one pass
    // earlier) and its pick in s_pick[i & 1], so a pass takes two barriers.
    uint32_t prefix = 0, pmask = 0;
    int remaining = nq;
    if (nq > 0) {
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass, hb = pass & 1;
            if (pass > 0) {
                // the other buffer's pass is over (its pick was read): clear it for the next
                if (tid < 256) hist[hb ^ 1][tid] = 0;
                // Only keys under the chosen prefix count, and they spread over the
                // next byte (crowded bins, e.g. equal scores, take one atomic a warp).
                for (int base = (tid & ~31); base < P; base += kTopkThreads) {
                    const int p = base + (tid & 31);
                    uint32_t d = 0x100u;   // no bin
                    if (p < P) {
                        const uint32_t k = key_at(p);
                        if ((k & pmask) == prefix) d = (k >> shift) & 0xFF;
                    }
                    hist_add_warp(hist[hb], d);
                }
                __syncthreads();
            }
            if (tid < 32) {
                // lane l owns bins 255-8l down to 248-8l
                int c[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    c[i] = hist[hb][255 - 8 * tid - i];
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
                        s_pick[hb][0] = 255 - 8 * tid - i;
                        s_pick[hb][1] = run;
                        s_pick[hb][2] = c[i];
                    }
                    run += c[i];
                }
            }
            __syncthreads();
            remaining -= s_pick[hb][1];
            prefix |= (uint32_t)s_pick[hb][0] << shift;
            pmask |= 0xFFu << shift;
            if (pass == 1 && s_pick[hb][2] <= 32) {
                // At most 32 keys share the top 16 bits of the answer (the usual
                // case: keys of similar magnitude differ from the second byte on).
                // Gather them and rank them on one warp instead of two more passes.
                const int lane = tid & 31;
                for (int base = (tid & ~31); base < P; base += kTopkThreads) {
                    const int p = base + lane;
                    const uint32_t k = p < P ? key_at(p) : 0u;
                    const bool m = p < P && (k & pmask) == prefix;
                    const uint32_t bal = __ballot_sync(0xffffffffu, m);
                    if (bal) {
                        int off = 0;
                        if (lane == 0) off = atomicAdd(&s_nsmall, __popc(bal));
                        off = __shfl_sync(0xffffffffu, off, 0);
                        if (m) s_small[off + __popc(bal & ((1u << lane) - 1u))] = k;
                    }
                }
                __syncthreads();
                if (tid < 32) {
                    const int n = s_nsmall;            // the bin's count, <= 32
                    const uint32_t mine = tid < n ? s_small[tid] : 0u;
                    int gt = 0, ge = 0;
                    for (int j = 0; j < n; ++j) {
                        const uint32_t kj = s_small[j];
                        gt += kj > mine;
                        ge += kj >= mine;
                    }
                    // the remaining-th largest of the bin (equal keys write equal values)
                    if (tid < n && gt < remaining && remaining <= ge) {
                        s_tau = mine;
                        s_req = remaining - gt;
                    }
                }
                __syncthreads();
                prefix = s_tau;
                remaining = s_req;
                break;
            }
        }
    }
    const uint32_t tau = prefix;   // the nq-th largest key (when nq > 0)
    const int r = remaining;       // keys equal to tau to take, lowest ids first

    // Selection in id order: warp w places the keys of a contiguous range, 32
    // consecutive keys a step (conflict-free reads, ballot ranks): every key above
    // tau, then the r lowest-id keys equal to it.
    const int lane = tid & 31, warp = tid >> 5;
    const int span = (((P + kTopkWarps - 1) / kTopkWarps) + 31) & ~31;
    const int wlo = min(P, warp * span), whi = min(P, wlo + span);
    const uint32_t below = (1u << lane) - 1u;
    int wgt = 0, weq = 0;
    if (nq > 0)
        for (int p0 = wlo; p0 < whi; p0 += 32) {
            const int p = p0 + lane;
            const uint32_t k = p < whi ? key_at(p) : 0u;
            wgt += __popc(__ballot_sync(0xffffffffu, p < whi && k > tau));
            weq += __popc(__ballot_sync(0xffffffffu, p < whi && k == tau));
        }
    if (lane == 0) s_warp2[warp] = make_int2(wgt, weq);
    __syncthreads();
    int gt_before = 0, eq_before = 0;
    for (int w2 = 0; w2 < warp; ++w2) {
        gt_before += s_warp2[w2].x;
        eq_before += s_warp2[w2].y;
    }
    if (nq > 0) {
        int pos = gt_before + min(eq_before, r), eqs = eq_before;
        for (int p0 = wlo; p0 < whi; p0 += 32) {
            const int p = p0 + lane;
            const uint32_t k = p < whi ? key_at(p) : 0u;
            const bool g = p < whi && k > tau, e = p < whi && k == tau;
            const uint32_t be = __ballot_sync(0xffffffffu, e);
            const bool take = g || (e && eqs + __popc(be & below) < r);
            const uint32_t bt = __ballot_sync(0xffffffffu, take);
            if (take) slist[pos + __popc(bt & below)] = p;
            pos += __popc(bt);
            eqs += __popc(be);
        }
    }
    __syncthreads();

    const size_t wout = (size_t)K * KP + tail.slots;   // row width of token_ids
    if (tid < tail.slots) {
        int id = -1;
        if (req_ok) {
            const int f = tail.first_valid[b], qp = tail.q_pos[q];
            const int rs = tail.req_start[b], T = tail.req_start[b + 1] - rs;
            if (qp >= f) {
                const int n = (int)(((long long)qp - f + 1) % KP);
                const long long t = (long long)qp + 1 - n + tid;
                if (tid < n && t >= 0 && t < T && tail.valid[(size_t)rs + t] != 0) id = (int)t;
            }
        }
        token_ids[(size_t)q * wout + (size_t)K * KP + tid] = id;
    }
    for (int j = tid; j < K; j += kTopkThreads)
        top_pools[(size_t)q * K + j] = j < nq ? slist[j] : -1;
    // Expansion: with kpool a multiple of 4, no tail slots and 16-byte aligned
    // rows, a selected pool's ids move as kpool/4 vector loads and stores;
    // otherwise four scalar gathers in flight per thread before the stores.
    if (tail.slots == 0 && (KP & 3) == 0 && aligned16(pool_idx) && aligned16(token_ids)) {
        const int nv = KP >> 2;
        const int4 *src = reinterpret_cast<const int4 *>(pool_idx + (size_t)(req_ok ? b : 0) * P * KP);
        int4 *dst = reinterpret_cast<int4 *>(token_ids + (size_t)q * wout);
        for (int e = tid; e < K * nv; e += kTopkThreads) {
            const int j = e / nv, u = e - j * nv;
            dst[e] = j < nq ? __ldg(src + (size_t)slist[j] * nv + u) : make_int4(-1, -1, -1, -1);
        }
        return;
    }
    for (int e0 = 0; e0 < K * KP; e0 += 4 * kTopkThreads) {
        int32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + tid + u * kTopkThreads;
            const int j = e / KP, s = e - j * KP;
            v[u] = -1;
            if (e < K * KP && j < nq) v[u] = pool_idx[((size_t)b * P + slist[j]) * KP + s];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + tid + u * kTopkThreads;
            if (e < K * KP) token_ids[(size_t)q * wout + e] = v[u];
        }
    }
}

inline int topk_expand_launch(const float *scores, const uint8_t *cand, const int32_t *pool_idx,
                              const int32_t *q_req, int Q, int B, int max_pools, int kpool,
                              int select_k, const TailArgs &tail, int32_t *top_pools,
                              int32_t *token_ids, cudaStream_t stream) {
    if (Q < 0 || B < 0 || max_pools < 0 || kpool <= 0 || select_k < 0) return DSA_ERR_INVALID_ARG;
    if (kpool > DSA_MAX_KPOOL || select_k > DSA_MAX_SELECT) return DSA_ERR_UNSUPPORTED;
    if (Q == 0 || (select_k == 0 && tail.slots == 0)) return DSA_OK;
    if (!q_req || (select_k > 0 && !top_pools) || !token_ids ||
        (max_pools > 0 && (!scores || !cand || (B > 0 && !pool_idx))))
        return DSA_ERR_INVALID_ARG;
    if (tail.slots > 0 && (!tail.q_pos || (B > 0 && (!tail.first_valid || !tail.valid || !tail.req_start))))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(pool_idx, 4) || !aligned(q_req, 4) ||
        !aligned(top_pools, 4) || !aligned(token_ids, 4) || !aligned(tail.q_pos, 4) ||
        !aligned(tail.first_valid, 4) || !aligned(tail.req_start, 4))
        return DSA_ERR_ALIGNMENT;
    const int keys_in_smem = max_pools <= kTopkSmemKeys ? 1 : 0;
    const int smem = select_k * 4 + (keys_in_smem ? max_pools * 4 : 0);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(topk_expand_kernel), smem))
        return DSA_ERR_CUDA;
    if (launch_pdl(topk_expand_kernel, dim3(Q), dim3(kTopkThreads), smem, stream, scores, cand,
                   pool_idx, q_req, B, max_pools, kpool, select_k, keys_in_smem, tail, top_pools,
                   token_ids) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
