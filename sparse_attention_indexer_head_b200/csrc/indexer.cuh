// f3. The fused indexer: head gate, index scores, top-k pools and their
// expansion to token ids in one launch
// ("feat(glm53): indexer fp32 head-gate split-K": the FUSED_K_GATE arm that
// computes the head gate inside the indexer instead of as its own GEMM;
// "spark_model/layers/glm5next_dsa/mod.rs", "Shape of the pipeline", second
// to fourth arrows: [Q, P] scores with candidate validity, the top-k select,
// the expansion to a [Q, select_k * kpool] token-id row; trap 6).
//
// One thread-block cluster of C CTAs per query (C <= 8). CTA r of the cluster
//   1. sums its K-slice of the query's head gate (hidden[q] . w) before the
//      wait on the preceding kernel (both are step inputs the path never
//      writes); the C partials meet through distributed shared memory and are
//      added in rank order, so every CTA holds the same gate_w[q];
//   2. scores its share of the pools, 128-pool tiles of TMA-loaded pooled keys
//      on the tensor cores (D[128 pools x 16 heads] = keys . q_idx^T), one
//      thread per pool summing g_h * relu(dot_h) in head order, and writes
//      scores and cand;
//   3. takes part in an exact 8-bit MSB radix select of the n_q-th largest
//      candidate key over the whole cluster: each pass's 256-bin histograms
//      are added across the cluster through distributed shared memory; after
//      two passes, when at most 32 keys of the cluster share the answer's top
//      16 bits, one warp ranks them;
//   4. writes its selected pools in ascending id order at positions offset by
//      the lower-ranked CTAs' counts, expands them to token ids and writes its
//      stripe of the -1 tail.
// The selection is the one dsa_topk_expand makes (ties to the lowest pool id,
// -0 equal to +0, NaN as -inf), so results are deterministic.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma.cuh"
#include "topk_expand.cuh"

namespace dsa {

constexpr int kIxThreads = 256;
constexpr int kIxWarps = kIxThreads / 32;
constexpr int kIxTile = 128;                                // pools per MMA tile (M)
constexpr int kIxHeads = DSA_MAX_INDEX_HEADS;               // 16 (N)
constexpr int kIxMaxCluster = 8;
constexpr int kIxMaxTilesPerCta = 32;                       // 4096 pools a CTA: max_pools <= 32768
constexpr uint32_t kIxKeyAtom = kIxTile * 128;              // 16 KB: one 64-channel column
constexpr uint32_t kIxKeyTile = 2 * kIxKeyAtom;             // 32 KB
constexpr uint32_t kIxQAtom = kIxHeads * 128;               // 2 KB
constexpr uint32_t kIxOffQ = 2 * kIxKeyTile;                // after the two-stage key ring
constexpr uint32_t kIxOffKeys = kIxOffQ + 2 * kIxQAtom;     // radix keys of the CTA's pools
constexpr int kIxSmem = (int)kIxOffKeys + kIxMaxTilesPerCta * kIxTile * 4 + 1024;

struct IxCtl {
    uint64_t q_bar, load_full[2], mma_done[2], d_empty[2];
    uint32_t tmem_base;
    int hist[2][256];
    float red[64][kIxHeads];            // gate partials per row-part
    float gpart[kIxHeads];              // this CTA's gate partial (read by the cluster)
    float gate[kIxHeads];               // the query's gate weights
    int2 warp2[kIxWarps];
    int pick[3];                        // (digit, count above, count in it) of the current pass
    int ncand;                          // this CTA's candidates (read by the cluster)
    int nsmall;                         // this CTA's keys in the small bin (read by the cluster)
    uint32_t small[32];
    uint32_t tau;
    int req;
    int cnt[2];                         // this CTA's keys above / equal to tau (read by the cluster)
    int base[2];                        // the lower-ranked CTAs' keys above / equal to tau
    int tot[256];                       // the current pass's histogram summed over the cluster
    volatile int abort;
};

// Pools [p_lo, p_hi) of cluster rank r: whole 128-pool tiles, split evenly.
struct IxRange { int t0, t1, p_lo, p_hi; };
DSA_DEVINL IxRange ix_range(int r, int C, int P) {
    const int nt = (P + kIxTile - 1) / kIxTile;
    const int tpc = (nt + C - 1) / C;
    IxRange g;
    g.t0 = min(nt, r * tpc);
    g.t1 = min(nt, g.t0 + tpc);
    g.p_lo = min(P, g.t0 * kIxTile);
    g.p_hi = min(P, g.t1 * kIxTile);
    return g;
}

DSA_DEVINL bool ix_wait(IxCtl *c, uint64_t *bar, uint32_t parity) {
    if (c->abort) return false;
    if (!mbar_wait(bar, parity)) {
        c->abort = 1;
        return false;
    }
    return true;
}

DSA_DEVINL int ld_cluster_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
DSA_DEVINL uint32_t ld_cluster_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

// Exclusive prefix sums of (a, b) over the CTA's kIxThreads threads; *ta, *tb get the sums.
DSA_DEVINL int2 ix_excl_scan2(int a, int b, int2 *s_warp2, int *ta, int *tb) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = a, y = b;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, x, off);
        const int v = __shfl_up_sync(0xffffffffu, y, off);
        if (lane >= off) { x += u; y += v; }
    }
    if (lane == 31) s_warp2[warp] = make_int2(x, y);
    __syncthreads();
    int2 before = make_int2(0, 0), tot = make_int2(0, 0);
#pragma unroll
    for (int w2 = 0; w2 < kIxWarps; ++w2) {
        const int2 v = s_warp2[w2];
        if (w2 < warp) { before.x += v.x; before.y += v.y; }
        tot.x += v.x;
        tot.y += v.y;
    }
    *ta = tot.x;
    *tb = tot.y;
    return make_int2(before.x + x - a, before.y + y - b);
}

__global__ void __launch_bounds__(kIxThreads, 1)
indexer_kernel(const __grid_constant__ CUtensorMap key_map, const __grid_constant__ CUtensorMap q_map,
               const float *__restrict__ hidden, const float *__restrict__ w, int K, int H,
               const int32_t *__restrict__ q_req, const int32_t *__restrict__ q_pos,
               const uint8_t *__restrict__ pool_valid, const int32_t *__restrict__ first_valid,
               const int32_t *__restrict__ pool_idx, int B, int KP, int P, int SK,
               float *__restrict__ gate_w, float *__restrict__ scores, uint8_t *__restrict__ cand,
               int32_t *__restrict__ top_pools, int32_t *__restrict__ token_ids) {
    extern __shared__ uint8_t ix_smem_raw[];
    __shared__ IxCtl ctl_s;
    IxCtl *ctl = &ctl_s;
    const uint32_t raw = smem_u32(ix_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = ix_smem_raw + (base - raw);
    uint32_t *skeys = reinterpret_cast<uint32_t *>(gbase + kIxOffKeys);
    const uint32_t sQ = base + kIxOffQ;

    const int C = gridDim.x, r = blockIdx.x, q = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IxRange rg = ix_range(r, C, P);
    const int ntile = rg.t1 - rg.t0;

    if (warp == 0) {
        tc::tmem_alloc(&ctl->tmem_base, 32);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        mbar_init(&ctl->q_bar, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->load_full[i], 1);
            mbar_init(&ctl->mma_done[i], 1);
            mbar_init(&ctl->d_empty[i], kIxTile);
        }
        ctl->abort = 0;
        ctl->ncand = 0;
        ctl->nsmall = 0;
        fence_mbarrier_init();
        // the query's head rows are a step input: in flight before the wait
        mbar_arrive_expect_tx(&ctl->q_bar, 2 * kIxQAtom);
        tma_load_2d(sQ, &q_map, 0, q * H, &ctl->q_bar);
        tma_load_2d(sQ + kIxQAtom, &q_map, 64, q * H, &ctl->q_bar);
    }
    for (int i = tid; i < 2 * 256; i += kIxThreads) (&ctl->hist[0][0])[i] = 0;

    // ---- 1. this CTA's K-slice of the head gate (step inputs: before the wait).
    // Thread (kp, hq) takes rows k = kb + kp, kb + kp + 64, ... in order (all of a
    // batch's loads in flight first) for heads 4hq..4hq+3; the 64 row-parts are
    // then added in order, then the cluster's slices in rank order.
    {
        const int kp = tid >> 2, hq = tid & 3;
        const int per = (K + C - 1) / C;
        const int kb = min(K, r * per), ke = min(K, kb + per);
        const float *hrow = hidden + (size_t)q * K;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (H == kIxHeads && aligned16(w)) {
            for (int k0 = kb + kp; k0 < ke; k0 += 64 * 8) {
                float hv[8];
                float4 wv[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int k = k0 + 64 * j;
                    hv[j] = k < ke ? __ldg(hrow + k) : 0.f;
                    wv[j] = k < ke ? __ldg(reinterpret_cast<const float4 *>(w + (size_t)k * kIxHeads) + hq)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    acc[0] = fmaf(hv[j], wv[j].x, acc[0]);
                    acc[1] = fmaf(hv[j], wv[j].y, acc[1]);
                    acc[2] = fmaf(hv[j], wv[j].z, acc[2]);
                    acc[3] = fmaf(hv[j], wv[j].w, acc[3]);
                }
            }
        } else {
            for (int k = kb + kp; k < ke; k += 64) {
                const float hk = __ldg(hrow + k);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * hq + e < H) acc[e] = fmaf(hk, __ldg(w + (size_t)k * H + 4 * hq + e), acc[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) ctl->red[kp][4 * hq + e] = acc[e];
    }
    const int b = q_req[q];                       // a step input, like the query rows
    const bool req_ok = b >= 0 && b < B;
    const int qp = q_pos[q];
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid < kIxHeads) {
        float s = 0.f;
#pragma unroll
        for (int kp = 0; kp < 64; ++kp) s += ctl->red[kp][tid];
        ctl->gpart[tid] = s;
    }
    const uint32_t tmem = ctl->tmem_base;

    pdl_wait();                                   // pooled keys and flags come from compress
    pdl_launch_dependents();

    // ---- 2. tiles: a producer thread loads keys and issues the MMAs, warps 0-3 drain
    auto load = [&](int i) {
        const int s = i & 1;
        mbar_arrive_expect_tx(&ctl->load_full[s], kIxKeyTile);
        const int row = b * P + (rg.t0 + i) * kIxTile;
        const uint32_t dst = base + s * kIxKeyTile;
        tma_load_2d(dst, &key_map, 0, row, &ctl->load_full[s]);
        tma_load_2d(dst + kIxKeyAtom, &key_map, 64, row, &ctl->load_full[s]);
    };
    if (tid == 128 && req_ok) {
        if (ntile > 0) load(0);
        if (ntile > 1) load(1);
    }

    // every CTA's gate partial is in place: add them in rank order
    cluster_sync_all();
    if (tid < kIxHeads) {
        const uint32_t a = smem_u32(&ctl->gpart[tid]);
        float v[kIxMaxCluster];
#pragma unroll
        for (int c = 0; c < kIxMaxCluster; ++c) v[c] = c < C ? ld_cluster_f32(cluster_map(a, c)) : 0.f;
        float g = 0.f;
#pragma unroll
        for (int c = 0; c < kIxMaxCluster; ++c) g += v[c];      // rank order
        ctl->gate[tid] = tid < H ? g : 0.f;
        if (r == 0 && tid < H) gate_w[(size_t)q * H + tid] = g;
    }
    __syncthreads();

    if (tid == 128 && req_ok) {
        bool ok = ntile == 0 || ix_wait(ctl, &ctl->q_bar, 0);
        constexpr uint32_t idesc = tc::idesc_bf16(kIxTile, kIxHeads, false, false);
        for (int i = 0; ok && i < ntile; ++i) {
            const int s = i & 1;
            ok = ix_wait(ctl, &ctl->load_full[s], (i >> 1) & 1);
            if (ok && i >= 2) ok = ix_wait(ctl, &ctl->d_empty[s], ((i >> 1) - 1) & 1);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t sK = base + s * kIxKeyTile;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t off_k = (kk >> 2) * kIxKeyAtom + (kk & 3) * 32;
                const uint32_t off_q = (kk >> 2) * kIxQAtom + (kk & 3) * 32;
                tc::mma_bf16_ss(tmem + 16 * s, tc::desc_sw128(sK + off_k, 16, 1024),
                                tc::desc_sw128(sQ + off_q, 16, 1024), idesc, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(&ctl->mma_done[s]);
            if (i + 2 < ntile) {
                // the stage is free once this tile's MMAs have read it
                ok = ix_wait(ctl, &ctl->mma_done[s], (i >> 1) & 1);
                if (ok) load(i + 2);
            }
        }
        if (!ok) ctl->abort = 1;
    }

    int local_cand = 0;
    if (warp < 4) {
        float g[kIxHeads];
#pragma unroll
        for (int h = 0; h < kIxHeads; ++h) g[h] = ctl->gate[h];
        const long long f = req_ok ? (long long)first_valid[b] : 0;
        for (int i = 0; i < ntile; ++i) {
            const int s = i & 1;
            const int p = (rg.t0 + i) * kIxTile + tid;
            bool is_cand = false;
            if (req_ok && p < P) {
                const long long last = f + (long long)p * KP + KP - 1;
                is_cand = pool_valid[(size_t)b * P + p] != 0 && last <= (long long)qp;
            }
            float score = -INFINITY;
            const bool ok = req_ok && __all_sync(0xffffffffu, ix_wait(ctl, &ctl->mma_done[s], (i >> 1) & 1));
            if (ok) {
                tc::fence_after_sync();
                uint32_t d[kIxHeads];
                tc::tmem_ld16(tmem + 16 * s + ((uint32_t)(32 * warp) << 16), d);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                mbar_arrive(&ctl->d_empty[s]);
                float acc = 0.f;
#pragma unroll
                for (int h = 0; h < kIxHeads; ++h) acc = fmaf(g[h], fmaxf(__uint_as_float(d[h]), 0.f), acc);
                if (is_cand) score = acc;
            } else {
                is_cand = false;
            }
            if (p < P) {
                scores[(size_t)q * P + p] = is_cand ? score : -INFINITY;
                cand[(size_t)q * P + p] = is_cand ? 1 : 0;
            }
            const int lp = p - rg.p_lo;
            const uint32_t k = score_key(score, is_cand);
            if (p < P) skeys[lp] = k;
            local_cand += k != 0u;
            const uint32_t dgt = (p < P) ? (k >> 24) : 0x100u;
            const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
            if (dgt != 0x100u && lane == __ffs(peers) - 1) atomicAdd(&ctl->hist[0][dgt], __popc(peers));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local_cand += __shfl_xor_sync(0xffffffffu, local_cand, off);
    if (lane == 0 && local_cand) atomicAdd(&ctl->ncand, local_cand);

    // ---- 3. radix select over the cluster
    __syncthreads();
    cluster_sync_all();                           // histograms of pass 0 and candidate counts
    int ncand = 0;
    {
        int v[kIxMaxCluster];
#pragma unroll
        for (int c = 0; c < kIxMaxCluster; ++c)
            v[c] = c < C ? ld_cluster_s32(cluster_map(smem_u32(&ctl->ncand), c)) : 0;
#pragma unroll
        for (int c = 0; c < kIxMaxCluster; ++c) ncand += v[c];
    }
    const int nq = min(SK, ncand);
    const int nloc = rg.p_hi - rg.p_lo;
    uint32_t prefix = 0, pmask = 0;
    int remaining = nq;
    if (nq > 0) {
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass, hb = pass & 1;
            if (pass > 0) {
                for (int i = tid; i < nloc; i += kIxThreads) {
                    const uint32_t k = skeys[i];
                    if ((k & pmask) == prefix) atomicAdd(&ctl->hist[hb][(k >> shift) & 0xFF], 1);
                }
                cluster_sync_all();
            }
            {
                // thread t sums bin t over the cluster (all loads in flight at once)
                const uint32_t a = smem_u32(&ctl->hist[hb][tid]);
                int v[kIxMaxCluster];
#pragma unroll
                for (int c = 0; c < kIxMaxCluster; ++c) v[c] = c < C ? ld_cluster_s32(cluster_map(a, c)) : 0;
                int t = 0;
#pragma unroll
                for (int c = 0; c < kIxMaxCluster; ++c) t += v[c];
                ctl->tot[tid] = t;
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns bins 255-8l down to 248-8l
                int cbin[8], sum = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    cbin[i] = ctl->tot[255 - 8 * tid - i];
                    sum += cbin[i];
                }
                int above = sum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, above, off);
                    if (tid >= off) above += y;
                }
                int run = above - sum;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (run < remaining && remaining <= run + cbin[i]) {
                        ctl->pick[0] = 255 - 8 * tid - i;
                        ctl->pick[1] = run;
                        ctl->pick[2] = cbin[i];
                    }
                    run += cbin[i];
                }
            }
            __syncthreads();
            remaining -= ctl->pick[1];
            prefix |= (uint32_t)ctl->pick[0] << shift;
            pmask |= 0xFFu << shift;
            const int in_bin = ctl->pick[2];
            // the other histogram buffer was last read by the cluster before the
            // barrier above: clear it for the next pass
            for (int i = tid; i < 256; i += kIxThreads) ctl->hist[hb ^ 1][i] = 0;
            __syncthreads();
            if (pass == 1 && in_bin <= 32) {
                // At most 32 keys of the cluster share the answer's top 16 bits:
                // gather them and rank them on one warp instead of two more passes.
                for (int base0 = (tid & ~31); base0 < nloc; base0 += kIxThreads) {
                    const int i = base0 + lane;
                    const uint32_t k = i < nloc ? skeys[i] : 0u;
                    const bool m = i < nloc && (k & pmask) == prefix;
                    const uint32_t bal = __ballot_sync(0xffffffffu, m);
                    if (bal) {
                        int off = 0;
                        if (lane == 0) off = atomicAdd(&ctl->nsmall, __popc(bal));
                        off = __shfl_sync(0xffffffffu, off, 0);
                        if (m) ctl->small[off + __popc(bal & ((1u << lane) - 1u))] = k;
                    }
                }
                cluster_sync_all();
                if (tid < 32) {
                    // lane c < C reads CTA c's list length; lane tid then loads entry tid of
                    // the cluster's lists concatenated in rank order
                    const int nc = tid < C ? ld_cluster_s32(cluster_map(smem_u32(&ctl->nsmall), tid)) : 0;
                    int incl = nc;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, off);
                        if (tid >= off) incl += y;
                    }
                    const int n = __shfl_sync(0xffffffffu, incl, 31);
                    int owner = 0, start = 0;
#pragma unroll
                    for (int c = 0; c < kIxMaxCluster; ++c) {
                        const int e = __shfl_sync(0xffffffffu, incl, c);      // end of CTA c's list
                        const int b0 = e - __shfl_sync(0xffffffffu, nc, c);
                        if (c < C && tid >= b0 && tid < e) { owner = c; start = b0; }
                    }
                    const uint32_t mine =
                        tid < n ? ld_cluster_u32(cluster_map(smem_u32(&ctl->small[tid - start]), owner)) : 0u;
                    int gt = 0, ge = 0;
                    for (int j = 0; j < n; ++j) {
                        const uint32_t kj = __shfl_sync(0xffffffffu, mine, j);
                        gt += kj > mine;
                        ge += kj >= mine;
                    }
                    if (tid < n && gt < remaining && remaining <= ge) {
                        ctl->tau = mine;
                        ctl->req = remaining - gt;
                    }
                }
                __syncthreads();
                prefix = ctl->tau;
                remaining = ctl->req;
                break;
            }
        }
    }
    const uint32_t tau = prefix;     // the nq-th largest key of the query (when nq > 0)
    const int req_eq = remaining;    // keys equal to tau to take, lowest ids first

    // ---- 4. placement: this CTA's winners after those of the lower ranks
    const int chunk = (nloc + kIxThreads - 1) / kIxThreads;
    const int i_lo = min(nloc, tid * chunk), i_hi = min(nloc, i_lo + chunk);
    int gt = 0, eq = 0;
    if (nq > 0)
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = skeys[i];
            gt += k > tau;
            eq += k == tau;
        }
    int tot_gt, tot_eq;
    const int2 before = ix_excl_scan2(gt, eq, ctl->warp2, &tot_gt, &tot_eq);
    if (tid == 0) {
        ctl->cnt[0] = tot_gt;
        ctl->cnt[1] = tot_eq;
    }
    cluster_sync_all();
    if (tid < 32) {
        // counts of the lower-ranked CTAs, summed on one warp
        int g = 0, e = 0;
        if (tid < r) {
            g = ld_cluster_s32(cluster_map(smem_u32(&ctl->cnt[0]), tid));
            e = ld_cluster_s32(cluster_map(smem_u32(&ctl->cnt[1]), tid));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            g += __shfl_xor_sync(0xffffffffu, g, off);
            e += __shfl_xor_sync(0xffffffffu, e, off);
        }
        if (tid == 0) {
            ctl->base[0] = g;
            ctl->base[1] = e;
        }
    }
    __syncthreads();
    const int base_gt = ctl->base[0], base_eq = ctl->base[1];
    const size_t wrow = (size_t)SK * KP;
    if (nq > 0) {
        const int eq0 = base_eq + before.y;
        int pos = base_gt + before.x + min(eq0, req_eq);
        int eqr = eq0;
        for (int i = i_lo; i < i_hi; ++i) {
            const uint32_t k = skeys[i];
            bool take = false;
            if (k > tau) {
                take = true;
            } else if (k == tau) {
                take = eqr < req_eq;
                ++eqr;
            }
            if (take) {
                const int p = rg.p_lo + i;
                top_pools[(size_t)q * SK + pos] = p;
                const int32_t *src = pool_idx + ((size_t)b * P + p) * KP;
                int32_t *dst = token_ids + (size_t)q * wrow + (size_t)pos * KP;
                for (int s = 0; s < KP; ++s) dst[s] = __ldg(src + s);
                ++pos;
            }
        }
    }
    // the -1 tail: slots nq .. SK-1, striped over the cluster
    for (int j = nq + r * kIxThreads + tid; j < SK; j += C * kIxThreads) {
        top_pools[(size_t)q * SK + j] = -1;
        for (int s = 0; s < KP; ++s) token_ids[(size_t)q * wrow + (size_t)j * KP + s] = -1;
    }

    if (tid == 32) (void)mbar_wait(&ctl->q_bar, 0);   // the query rows' copy has landed
    tc::fence_before_sync();
    cluster_sync_all();                           // no CTA leaves while a peer still reads it
    if (warp == 0) tc::tmem_dealloc(tmem, 32);
}

// Cluster size: 8 CTAs whatever P (the gate's K-split uses every CTA; one with no
// pool tile only adds its gate slice and takes part in the select).
inline int indexer_cluster(int) { return kIxMaxCluster; }

inline int indexer_launch(const float *hidden, const float *w, int K, const void *q_idx,
                          const int32_t *q_req, const int32_t *q_pos, int Q, int H, int D,
                          const void *pool_keys, const uint8_t *pool_valid,
                          const int32_t *first_valid, const int32_t *pool_idx, int B, int kpool,
                          int max_pools, int select_k, float *gate_w, float *scores, uint8_t *cand,
                          int32_t *top_pools, int32_t *token_ids, cudaStream_t stream) {
    if (Q < 0 || K <= 0 || H <= 0 || D <= 0 || B < 0 || kpool <= 0 || max_pools < 0 || select_k < 0)
        return DSA_ERR_INVALID_ARG;
    if (D != kD || H > kIxHeads || kpool > DSA_MAX_KPOOL || select_k > DSA_MAX_SELECT)
        return DSA_ERR_UNSUPPORTED;
    if (max_pools > kIxMaxCluster * kIxMaxTilesPerCta * kIxTile) return DSA_ERR_UNSUPPORTED;
    if (Q == 0) return DSA_OK;
    if (Q > 65535 || (long long)B * max_pools >= (1ll << 31) || (long long)Q * H >= (1ll << 31))
        return DSA_ERR_UNSUPPORTED;
    if (!hidden || !w || !q_idx || !q_req || !q_pos || !gate_w ||
        (max_pools > 0 && (!scores || !cand)) || (select_k > 0 && (!top_pools || !token_ids)) ||
        (B > 0 && max_pools > 0 && (!pool_keys || !pool_valid || !first_valid || !pool_idx)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(hidden, 4) || !aligned(w, 4) || !aligned(q_idx, 16) || !aligned(q_req, 4) ||
        !aligned(q_pos, 4) || !aligned(pool_keys, 16) || !aligned(first_valid, 4) ||
        !aligned(pool_idx, 4) || !aligned(gate_w, 4) || !aligned(scores, 4) ||
        !aligned(top_pools, 4) || !aligned(token_ids, 4))
        return DSA_ERR_ALIGNMENT;
    CUtensorMap key_map, q_map;
    const void *kbase = (B > 0 && max_pools > 0) ? pool_keys : q_idx;
    const uint64_t krows = (B > 0 && max_pools > 0) ? (uint64_t)B * max_pools : (uint64_t)Q * H;
    if (!make_map_bf16_2d(&key_map, kbase, krows, kD, kD * 2, 64, kIxTile) ||
        !make_map_bf16_2d(&q_map, q_idx, (uint64_t)Q * H, kD, kD * 2, 64, kIxHeads))
        return DSA_ERR_CUDA;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(indexer_kernel), kIxSmem)) return DSA_ERR_CUDA;
    const int C = indexer_cluster(max_pools);
    if (launch_pdl_cluster(indexer_kernel, dim3(C, Q), dim3(kIxThreads), kIxSmem, stream, C, key_map,
                           q_map, hidden, w, K, H, q_req, q_pos, pool_valid, first_valid, pool_idx,
                           B, kpool, max_pools, select_k, gate_w, scores, cand, top_pools,
                           token_ids) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
