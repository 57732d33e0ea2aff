// f3. The fused indexer: head gate, index scores, top-k pools and their
// expansion to token ids in one launch
// ("feat(glm53): indexer fp32 head-gate split-K": the FUSED_K_GATE arm that
// computes the head gate inside the indexer instead of as its own GEMM;
// "spark_model/layers/glm5next_dsa/mod.rs", "Shape of the pipeline", second
// to fourth arrows: [Q, P] scores with candidate validity, the top-k select,
// the expansion to a [Q, select_k * kpool] token-id row; trap 6).
//
// One thread-block cluster of 8 CTAs per query. CTA r of the cluster
//   1. sums its K-slice of the query's head gate (hidden[q] . w) before the
//      wait on the preceding kernel (both are step inputs the path never
//      writes) and pushes the partial into every CTA's shared memory; each CTA
//      adds the 8 partials in rank order, so all hold the same gate_w[q];
//   2. scores its share of the pools, 128-pool tiles of TMA-loaded pooled keys
//      on the tensor cores (D[128 pools x 16 heads] = keys . q_idx^T), one
//      thread per pool summing g_h * relu(dot_h) in head order; it writes
//      scores and cand and pushes each pool's radix key into the shared
//      memory of the cluster's first CTA (the leader);
//   3. the leader selects: an exact 8-bit MSB radix select of the n_q-th
//      largest candidate key over the query's pools, with, after two passes,
//      a one-warp rank of the at most 32 keys that share the answer's top 16
//      bits; the winners are placed in ascending pool id (warps over
//      contiguous id ranges, ballot ranks) and expanded to token ids, and the
//      -1 tail is written.
// Pushes are distributed-shared-memory stores followed by a release arrive on
// the receiver's mbarrier, so the only cluster-wide rendezvous is the one that
// guarantees every CTA has started (its arrive is issued before the gate's
// loads). The selection is the one dsa_topk_expand makes (ties to the lowest
// pool id, -0 equal to +0, NaN as -inf), so results are deterministic.
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
constexpr int kIxCluster = 8;                               // CTAs per query
constexpr int kIxMaxPools = 32768;                          // keys the leader holds
constexpr uint32_t kIxKeyAtom = kIxTile * 128;              // 16 KB: one 64-channel column
constexpr uint32_t kIxKeyTile = 2 * kIxKeyAtom;             // 32 KB
constexpr uint32_t kIxQAtom = kIxHeads * 128;               // 2 KB
constexpr uint32_t kIxOffQ = 2 * kIxKeyTile;                // after the two-stage key ring
constexpr uint32_t kIxOffKeys = kIxOffQ + 2 * kIxQAtom;     // the query's radix keys (leader)

// Dynamic shared memory: the key ring (whose space also holds the leader's
// select_k selected ids once its tiles are done), the query rows and P radix
// keys (used by the leader, sized alike on every CTA).
inline int indexer_smem_bytes(int P) { return (int)kIxOffKeys + 4 * P + 1024; }
static_assert(4 * DSA_MAX_SELECT <= 2 * kIxKeyTile, "selected ids fit in the key ring");

struct IxCtl {
    uint64_t q_bar, load_full[2], mma_done[2], d_empty[2];
    uint64_t gate_bar;                  // the cluster's gate partials have arrived
    uint64_t keys_bar;                  // the cluster's radix keys have arrived (leader)
    uint32_t tmem_base;
    int hist[2][256];
    float red[64][kIxHeads];            // gate partials per row-part
    float gate_in[kIxCluster][kIxHeads];// the cluster's gate partials, by rank
    float gate[kIxHeads];               // the query's gate weights
    int ncand_in[kIxCluster];           // the cluster's candidate counts, by rank (leader)
    int hist_in[kIxCluster][256];       // the cluster's top-byte histograms, by rank (leader)
    int2 warp2[kIxWarps];
    int pick[3];                        // (digit, count above, count in it) of the current pass
    int ncand;                          // this CTA's candidates
    int nsmall;
    uint32_t small[32];
    uint32_t tau;
    int req;
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

// Bounded wait with cluster-scope acquire: writes that other CTAs of the cluster
// made before their release arrive on this (local) barrier are visible after it.
DSA_DEVINL bool mbar_wait_cluster(uint64_t *bar, uint32_t phase) {
    auto try_once = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(phase)
            : "memory");
        return ok != 0;
    };
    if (try_once()) return true;
    const long long t0 = clock64();
    for (;;) {
        if (try_once()) return true;
        if (clock64() - t0 > kWaitLimitCycles) break;
    }
    raise_device_error(kErrWaitTimeout);
    return false;
}

// Release arrive on the mbarrier at shared::cluster address `remote` (another
// CTA's, or this one's through its cluster address).
DSA_DEVINL void mbar_arrive_remote(uint32_t remote) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote)
                 : "memory");
}
DSA_DEVINL void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
DSA_DEVINL void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
DSA_DEVINL void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

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
    uint32_t *akeys = reinterpret_cast<uint32_t *>(gbase + kIxOffKeys);                 // [P]
    int32_t *slist = reinterpret_cast<int32_t *>(gbase);   // [SK], in the key ring (leader, at the end)
    const uint32_t sQ = base + kIxOffQ;

    const int C = gridDim.x, r = blockIdx.x, q = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IxRange rg = ix_range(r, C, P);
    const int ntile = rg.t1 - rg.t0;
    // the query's request and position are step inputs: their loads go out first
    const int b = q_req[q];
    const int qp = q_pos[q];

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
        mbar_init(&ctl->gate_bar, C);
        mbar_init(&ctl->keys_bar, C);
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
    // Every CTA of the cluster has started and initialised its barriers once the
    // cluster wait below returns; the arrive goes out now, so the rendezvous
    // overlaps the gate's loads.
    tc::fence_before_sync();
    __syncthreads();
    cluster_arrive_relaxed();

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
    const bool req_ok = b >= 0 && b < B;
    __syncthreads();
    if (tid < kIxHeads) {
        float gpart = 0.f;
        for (int kp = 0; kp < 64; ++kp) gpart += ctl->red[kp][tid];
        ctl->gate[tid] = gpart;                   // this CTA's partial, until the sum below
    }
    const uint32_t tmem = ctl->tmem_base;
    tc::fence_after_sync();
    __syncthreads();
    cluster_wait();
    // push: thread (c, h) of warps 0-3 writes this CTA's partial of head h into
    // slot r of CTA c; one thread per receiver then arrives on its barrier
    if (warp < 4) {
        const int c = tid >> 4, h = tid & 15;
        if (c < C) st_cluster_u32(cluster_map(smem_u32(&ctl->gate_in[r][h]), c), __float_as_uint(ctl->gate[h]));
    }
    __syncthreads();
    if (tid < C) {
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        mbar_arrive_remote(cluster_map(smem_u32(&ctl->gate_bar), tid));
    }

    pdl_wait();                                   // pooled keys and flags come from compress
    pdl_launch_dependents();

    // ---- 2. tiles: two issuing threads load keys and issue the MMAs, warps 0-3 drain
    auto load = [&](int i) {
        const int s = i & 1;
        mbar_arrive_expect_tx(&ctl->load_full[s], kIxKeyTile);
        const int row = b * P + (rg.t0 + i) * kIxTile;
        const uint32_t dst = base + s * kIxKeyTile;
        tma_load_2d(dst, &key_map, 0, row, &ctl->load_full[s]);
        tma_load_2d(dst + kIxKeyAtom, &key_map, 64, row, &ctl->load_full[s]);
    };
    // tiles i = 0, 2, 4 ... go through stage 0 and the issuer in warp 4, tiles
    // 1, 3, 5 ... through stage 1 and the issuer in warp 5 (a single thread
    // starts about one MMA per 128 cycles; two in separate warps run in parallel)
    const bool issuer = (tid == 128 || tid == 160) && req_ok;
    const int my_s = (tid - 128) >> 5;
    if (issuer && my_s < ntile) load(my_s);
    // the cluster's gate partials, added in rank order
    if (tid < kIxHeads) {
        float g = 0.f;
        if (mbar_wait_cluster(&ctl->gate_bar, 0)) {
            for (int c = 0; c < C; ++c) g += ctl->gate_in[c][tid];
        } else {
            ctl->abort = 1;
        }
        ctl->gate[tid] = tid < H ? g : 0.f;
        if (r == 0 && tid < H) gate_w[(size_t)q * H + tid] = g;
    }
    __syncthreads();

    if (issuer) {
        bool ok = my_s >= ntile || ix_wait(ctl, &ctl->q_bar, 0);
        constexpr uint32_t idesc = tc::idesc_bf16(kIxTile, kIxHeads, false, false);
        for (int i = my_s; ok && i < ntile; i += 2) {
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

    const uint32_t lead_keys = cluster_map(smem_u32(akeys), 0);   // the leader's key array
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
                const uint32_t k = score_key(score, is_cand);
                st_cluster_u32(lead_keys + 4u * (uint32_t)p, k);
                local_cand += k != 0u;
            }
            // this CTA's share of the first radix pass: the top bytes of its keys
            const uint32_t dgt = p < P ? (score_key(score, is_cand) >> 24) : 0x100u;
            const uint32_t peers = __match_any_sync(0xffffffffu, dgt);
            if (dgt != 0x100u && lane == __ffs(peers) - 1) atomicAdd(&ctl->hist[0][dgt], __popc(peers));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local_cand += __shfl_xor_sync(0xffffffffu, local_cand, off);
    if (lane == 0 && local_cand) atomicAdd(&ctl->ncand, local_cand);
    __syncthreads();
    // this CTA's histogram and candidate count to the leader, then its release
    // arrive (after every key this CTA pushed: the CTA barrier orders them before it)
    st_cluster_u32(cluster_map(smem_u32(&ctl->hist_in[r][tid]), 0), (uint32_t)ctl->hist[0][tid]);
    __syncthreads();
    if (tid == 0) {
        st_cluster_u32(cluster_map(smem_u32(&ctl->ncand_in[r]), 0), (uint32_t)ctl->ncand);
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        mbar_arrive_remote(cluster_map(smem_u32(&ctl->keys_bar), 0));
    }

    if (r == 0) {
        // ---- 3. the leader selects over the query's P keys
        if (tid == 0) {
            int n = 0;
            if (mbar_wait_cluster(&ctl->keys_bar, 0)) {
                for (int c = 0; c < C; ++c) n += ctl->ncand_in[c];
            } else {
                ctl->abort = 1;
            }
            ctl->req = ctl->abort ? 0 : n;
        }
        __syncthreads();
        const int nq = min(SK, ctl->req);

        uint32_t prefix = 0, pmask = 0;
        int remaining = nq;
        if (nq > 0) {
            // pass 0's histogram: the cluster's top-byte histograms added up
            {
                int t = 0;
                for (int c = 0; c < C; ++c) t += ctl->hist_in[c][tid];
                __syncthreads();
                ctl->hist[0][tid] = t;
            }
            __syncthreads();
#pragma unroll 1
            for (int pass = 0; pass < 4; ++pass) {
                const int shift = 24 - 8 * pass, hb = pass & 1;
                if (pass > 0) {
                    for (int p = tid; p < P; p += kIxThreads) {
                        const uint32_t k = akeys[p];
                        if ((k & pmask) == prefix) atomicAdd(&ctl->hist[hb][(k >> shift) & 0xFF], 1);
                    }
                    __syncthreads();
                }
                if (tid < 32) {
                    // lane l owns bins 255-8l down to 248-8l
                    int cbin[8], sum = 0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        cbin[i] = ctl->hist[hb][255 - 8 * tid - i];
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
                for (int i = tid; i < 256; i += kIxThreads) ctl->hist[hb ^ 1][i] = 0;
                __syncthreads();
                if (pass == 1 && in_bin <= 32) {
                    // At most 32 keys share the answer's top 16 bits: gather them and
                    // rank them on one warp instead of two more passes.
                    for (int base0 = (tid & ~31); base0 < P; base0 += kIxThreads) {
                        const int p = base0 + lane;
                        const uint32_t k = p < P ? akeys[p] : 0u;
                        const bool m = p < P && (k & pmask) == prefix;
                        const uint32_t bal = __ballot_sync(0xffffffffu, m);
                        if (bal) {
                            int off = 0;
                            if (lane == 0) off = atomicAdd(&ctl->nsmall, __popc(bal));
                            off = __shfl_sync(0xffffffffu, off, 0);
                            if (m) ctl->small[off + __popc(bal & ((1u << lane) - 1u))] = k;
                        }
                    }
                    __syncthreads();
                    if (tid < 32) {
                        const int n = ctl->nsmall;
                        const uint32_t mine = tid < n ? ctl->small[tid] : 0u;
                        int gt = 0, ge = 0;
                        for (int j = 0; j < n; ++j) {
                            const uint32_t kj = ctl->small[j];
                            gt += kj > mine;
                            ge += kj >= mine;
                        }
                        if (tid < n && gt < remaining && remaining <= ge) {
                            ctl->tau = mine;
                            ctl->pick[0] = remaining - gt;
                        }
                    }
                    __syncthreads();
                    prefix = ctl->tau;
                    remaining = ctl->pick[0];
                    break;
                }
            }
        }
        const uint32_t tau = prefix;     // the nq-th largest key (when nq > 0)
        const int req_eq = remaining;    // keys equal to tau to take, lowest ids first

        // ---- 4. winners in ascending pool id: every key above tau, then the
        // req_eq lowest-id keys equal to it. Warp w places the keys of a contiguous
        // range, 32 consecutive keys a step (conflict-free reads, ballot ranks).
        const int span = (((P + kIxWarps - 1) / kIxWarps) + 31) & ~31;
        const int wlo = min(P, warp * span), whi = min(P, wlo + span);
        const uint32_t below = (1u << lane) - 1u;
        int wgt = 0, weq = 0;
        if (nq > 0)
            for (int p0 = wlo; p0 < whi; p0 += 32) {
                const int p = p0 + lane;
                const uint32_t k = p < whi ? akeys[p] : 0u;
                wgt += __popc(__ballot_sync(0xffffffffu, p < whi && k > tau));
                weq += __popc(__ballot_sync(0xffffffffu, p < whi && k == tau));
            }
        if (lane == 0) ctl->warp2[warp] = make_int2(wgt, weq);
        __syncthreads();
        int gt_before = 0, eq_before = 0;
        for (int w2 = 0; w2 < warp; ++w2) {
            gt_before += ctl->warp2[w2].x;
            eq_before += ctl->warp2[w2].y;
        }
        if (nq > 0) {
            int pos = gt_before + min(eq_before, req_eq), eqs = eq_before;
            for (int p0 = wlo; p0 < whi; p0 += 32) {
                const int p = p0 + lane;
                const uint32_t k = p < whi ? akeys[p] : 0u;
                const bool g = p < whi && k > tau, e = p < whi && k == tau;
                const uint32_t be = __ballot_sync(0xffffffffu, e);
                const bool take = g || (e && eqs + __popc(be & below) < req_eq);
                const uint32_t bt = __ballot_sync(0xffffffffu, take);
                if (take) slist[pos + __popc(bt & below)] = p;
                pos += __popc(bt);
                eqs += __popc(be);
            }
        }
        __syncthreads();
        const size_t wrow = (size_t)SK * KP;
        for (int j = tid; j < SK; j += kIxThreads) top_pools[(size_t)q * SK + j] = j < nq ? slist[j] : -1;
        // expansion: with kpool a multiple of 4 and 16-byte aligned rows, a
        // selected pool's ids move as kpool/4 vector loads and stores; otherwise
        // four scalar gathers in flight per thread before the stores
        if ((KP & 3) == 0 && aligned16(pool_idx) && aligned16(token_ids)) {
            const int nv = KP >> 2;                         // 16-byte pieces a pool
            const int4 *src = reinterpret_cast<const int4 *>(pool_idx + (size_t)b * P * KP);
            int4 *dst = reinterpret_cast<int4 *>(token_ids + (size_t)q * wrow);
            for (int e = tid; e < SK * nv; e += kIxThreads) {
                const int j = e / nv, u = e - j * nv;
                dst[e] = j < nq ? __ldg(src + (size_t)slist[j] * nv + u) : make_int4(-1, -1, -1, -1);
            }
        } else {
            for (int e0 = 0; e0 < SK * KP; e0 += 4 * kIxThreads) {
                int32_t v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + tid + u * kIxThreads;
                    const int j = e / KP, s = e - j * KP;
                    v[u] = -1;
                    if (e < SK * KP && j < nq) v[u] = __ldg(pool_idx + ((size_t)b * P + slist[j]) * KP + s);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int e = e0 + tid + u * kIxThreads;
                    if (e < SK * KP) token_ids[(size_t)q * wrow + e] = v[u];
                }
            }
        }
    }

    if (tid == 32) (void)mbar_wait(&ctl->q_bar, 0);   // the query rows' copy has landed
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 32);
}

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
    if (max_pools > kIxMaxPools) return DSA_ERR_UNSUPPORTED;
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
    const int smem = indexer_smem_bytes(max_pools);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(indexer_kernel), smem)) return DSA_ERR_CUDA;
    if (launch_pdl_cluster(indexer_kernel, dim3(kIxCluster, Q), dim3(kIxThreads), smem, stream,
                           kIxCluster, key_map, q_map, hidden, w, K, H, q_req, q_pos, pool_valid,
                           first_valid, pool_idx, B, kpool, max_pools, select_k, gate_w, scores,
                           cand, top_pools, token_ids) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
