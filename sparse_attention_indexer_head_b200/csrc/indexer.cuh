// f3. The fused indexer: head gate, index scores, top-k pools and their
// expansion to token ids in one launch
// ("feat(glm53): indexer fp32 head-gate split-K": the FUSED_K_GATE arm that
// computes the head gate inside the indexer instead of as its own GEMM;
// "spark_model/layers/glm5next_dsa/mod.rs", "Shape of the pipeline", second
// to fourth arrows: [Q, P] scores with candidate validity, the top-k select,
// the expansion to a [Q, select_k * kpool] token-id row; trap 6).
//
// One thread-block cluster per query: 8 CTAs, or 16 where few queries leave
// most of the device idle. CTA r of the cluster
//   1. sums its K-slice of the query's head gate (hidden[q] . w) before the
//      wait on the preceding kernel (both are step inputs the path never
//      writes) and pushes the partial into every CTA's shared memory; each CTA
//      adds the C partials in rank order, so all hold the same gate_w[q];
//   2. scores its contiguous range of pools, 128-pool tiles of TMA-loaded
//      pooled keys on the tensor cores (D[128 pools x 16 heads] = keys .
//      q_idx^T), one thread per pool summing g_h * relu(dot_h) in head order;
//      it writes scores and cand and keeps each pool's radix key in its own
//      shared memory;
//   3. the cluster selects together: an exact 8-bit MSB radix select of the
//      n_q-th largest candidate key. Each pass every CTA counts the digit over
//      its own keys and sends the 256 counts to every CTA, so all CTAs add the
//      same histogram and take the same digit; after two passes, when at most
//      32 keys share the answer's top 16 bits, those keys are exchanged and
//      ranked on one warp instead of two more passes;
//   4. every CTA counts its keys above the answer and equal to it, exchanges
//      the counts, and writes its winners at their places in ascending pool id
//      (ties to the lowest ids) with their token ids; the -1 tail is shared out.
// An exchange is a set of asynchronous distributed-shared-memory stores into
// slot r of every CTA's buffer, each completing its bytes on that CTA's
// mbarrier (which expects the C ranks' bytes); two buffers alternate, so a CTA
// never receives the next exchange into a buffer it is still reading. The selection is the one dsa_topk_expand makes (ties to the
// lowest pool id, -0 equal to +0, NaN as -inf), so results are deterministic.
#pragma once

#include <atomic>

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
constexpr int kIxMaxCluster = 16;                           // with few queries
constexpr int kIxMaxPools = 32768;
constexpr int kIxXWords = 260;                              // exchange: 256 counts + 4
constexpr uint32_t kIxXBytes = 4 * kIxXWords;               // 65 16-byte pieces
constexpr uint32_t kIxKeyAtom = kIxTile * 128;              // 16 KB: one 64-channel column
constexpr uint32_t kIxKeyTile = 2 * kIxKeyAtom;             // 32 KB
constexpr uint32_t kIxQAtom = kIxHeads * 128;               // 2 KB
constexpr int kIxStages = 5;                                // deepest key ring (tiles in flight)
constexpr uint32_t kIxTmemCols = 128;                       // up to kIxStages D[128 x 16]
static_assert(kIxHeads * kIxStages <= (int)kIxTmemCols, "tensor memory columns");
// Dynamic shared memory of a ring of ns stages: the ring, the query rows, the
// radix keys of this CTA's pools (whole tiles).
__host__ __device__ inline uint32_t ix_off_q(int ns) { return (uint32_t)ns * kIxKeyTile; }
__host__ __device__ inline uint32_t ix_off_keys(int ns) { return ix_off_q(ns) + 2 * kIxQAtom; }

// Dynamic shared memory: the key ring, the query rows and the radix keys of
// this CTA's pools (whole tiles).
inline int indexer_smem_bytes(int P, int C, int ns) {
    const int tiles = (P + kIxTile - 1) / kIxTile;
    return (int)ix_off_keys(ns) + 5 * kIxTile * ((tiles + C - 1) / C) + 1024;   // keys, valid bytes
}

struct IxCtl {
    uint64_t q_bar, load_full[kIxStages], mma_done[kIxStages], d_empty[kIxStages];
    uint64_t gate_bar;                  // the cluster's gate partials have arrived
    uint64_t xbar[2];                   // an exchange into buffer i has fully arrived
    uint32_t tmem_base;
    int hloc[256];                      // this CTA's counts of the current digit
    float red[64][kIxHeads];            // gate partials per row-part
    float gate_in[kIxMaxCluster][kIxHeads];   // the cluster's gate partials, by rank
    float gate[kIxHeads];               // the query's gate weights
    alignas(16) int xin[2][kIxMaxCluster][kIxXWords];   // exchange buffers: rank c's words
    alignas(16) int xout[kIxXWords];    // this CTA's words of the current exchange
    int2 warp2[kIxWarps];
    int pick[3];                        // (digit, count above, count in it) of the current pass
    int ncand;                          // this CTA's candidates
    int nsmall;
    uint32_t small[32];                 // this CTA's keys sharing the answer's top 16 bits
    uint32_t tau;
    int req;
    int gt16;                           // this CTA's keys above the answer's top 16 bits
    int rank_gt, rank_eq;               // keys above / equal to tau on the lower ranks
    volatile int abort;
};
static_assert(sizeof(IxCtl) <= 46 * 1024, "static shared memory");

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
// 16 bytes into another CTA's shared memory (shared::cluster address), their
// arrival completing 16 bytes of the transaction count of the mbarrier at
// `remote_bar` (in the same CTA as the destination).
DSA_DEVINL void st_async_b32(uint32_t remote, uint32_t v, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote),
                 "r"(v), "r"(remote_bar)
                 : "memory");
}
DSA_DEVINL void st_async_v4(uint32_t remote, int4 v, uint32_t remote_bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.s32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
            remote),
        "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(remote_bar)
        : "memory");
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
               int32_t *__restrict__ top_pools, int32_t *__restrict__ token_ids, int NS) {
    extern __shared__ uint8_t ix_smem_raw[];
    __shared__ IxCtl ctl_s;
    IxCtl *ctl = &ctl_s;
    const uint32_t raw = smem_u32(ix_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *gbase = ix_smem_raw + (base - raw);
    uint32_t *akeys = reinterpret_cast<uint32_t *>(gbase + ix_off_keys(NS));   // this CTA's pools
    uint8_t *svalid;                     // their pool_valid bytes (after the keys)
    const uint32_t sQ = base + ix_off_q(NS);

    const int C = gridDim.x, r = blockIdx.x, q = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IxRange rg = ix_range(r, C, P);
    const int ntile = rg.t1 - rg.t0;
    svalid = reinterpret_cast<uint8_t *>(akeys + (size_t)kIxTile * ((((P + kIxTile - 1) / kIxTile) + C - 1) / C));
    // the query's request and position are step inputs: their loads go out first
    const int b = q_req[q];
    const int qp = q_pos[q];

    if (warp == 0) {
        tc::tmem_alloc(&ctl->tmem_base, kIxTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        mbar_init(&ctl->q_bar, 1);
        for (int i = 0; i < kIxStages; ++i) {
            mbar_init(&ctl->load_full[i], 1);
            mbar_init(&ctl->mma_done[i], 1);
            mbar_init(&ctl->d_empty[i], kIxTile);
        }
        mbar_init(&ctl->gate_bar, 1);
        // the other ranks' partials arrive as asynchronous stores counted in bytes
        mbar_arrive_expect_tx(&ctl->gate_bar, (uint32_t)(C - 1) * kIxHeads * 4);
        mbar_init(&ctl->xbar[0], 1);       // own expect_tx; the other ranks' bytes complete it
        mbar_init(&ctl->xbar[1], 1);
        ctl->abort = 0;
        ctl->ncand = 0;
        ctl->nsmall = 0;
        fence_mbarrier_init();
        // the query's head rows are a step input: in flight before the wait
        mbar_arrive_expect_tx(&ctl->q_bar, 2 * kIxQAtom);
        tma_load_2d(sQ, &q_map, 0, q * H, &ctl->q_bar);
        tma_load_2d(sQ + kIxQAtom, &q_map, 64, q * H, &ctl->q_bar);
    }
    for (int i = tid; i < 256; i += kIxThreads) ctl->hloc[i] = 0;
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
    // push: thread (c, h) stores this CTA's partial of head h into slot r of CTA
    // c, completing 4 bytes on that CTA's barrier (its own slot: a plain store)
    {
        const int c = tid >> 4, h = tid & 15;
        const uint32_t v = __float_as_uint(ctl->gate[h]);
        if (c == r)
            ctl->gate_in[r][h] = ctl->gate[h];
        else if (c < C)
            st_async_b32(cluster_map(smem_u32(&ctl->gate_in[r][h]), c), v,
                         cluster_map(smem_u32(&ctl->gate_bar), c));
    }
    __syncthreads();

    pdl_wait();                                   // pooled keys and flags come from compress
    pdl_launch_dependents();

    // ---- 2. tiles: a producer thread loads keys into an NS-deep ring, two
    // issuing threads issue the MMAs (tile i into stage and accumulator i % NS),
    // warps 0-3 drain the accumulators
    auto load = [&](int i) {
        const int s = i % NS;
        mbar_arrive_expect_tx(&ctl->load_full[s], kIxKeyTile);
        const int row = b * P + (rg.t0 + i) * kIxTile;
        const uint32_t dst = base + s * kIxKeyTile;
        tma_load_2d(dst, &key_map, 0, row, &ctl->load_full[s]);
        tma_load_2d(dst + kIxKeyAtom, &key_map, 64, row, &ctl->load_full[s]);
    };
    // tiles i = 0, 2, 4 ... go to the issuer in warp 4, tiles 1, 3, 5 ... to the
    // issuer in warp 5 (a single thread starts about one MMA per 128 cycles; two
    // in separate warps run in parallel)
    const bool issuer = (tid == 128 || tid == 160) && req_ok;
    const bool producer = tid == 192 && req_ok;
    const int my_s = (tid - 128) >> 5;
    if (producer)
        for (int i = 0; i < min(ntile, NS); ++i) load(i);
    // this CTA's pool_valid bytes, all loads in flight at once (seen by the
    // epilogue after the barrier below)
    if (req_ok) {
        const uint8_t *vsrc = pool_valid + (size_t)b * P + rg.p_lo;
        const int nv = max(0, rg.p_hi - rg.p_lo);
        for (int i0 = 0; i0 < nv; i0 += 4 * kIxThreads) {
            uint8_t v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kIxThreads + tid;
                v[u] = i < nv ? __ldg(vsrc + i) : (uint8_t)0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * kIxThreads + tid;
                if (i < nv) svalid[i] = v[u];
            }
        }
    }
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
            const int s = i % NS, ph = (i / NS) & 1;
            ok = ix_wait(ctl, &ctl->load_full[s], ph);
            if (ok && i >= NS) ok = ix_wait(ctl, &ctl->d_empty[s], ph ^ 1);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t sK = base + s * kIxKeyTile;
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t off_k = (kk >> 2) * kIxKeyAtom + (kk & 3) * 32;
                const uint32_t off_q = (kk >> 2) * kIxQAtom + (kk & 3) * 32;
                tc::mma_bf16_ss(tmem + kIxHeads * s, tc::desc_sw128(sK + off_k, 16, 1024),
                                tc::desc_sw128(sQ + off_q, 16, 1024), idesc, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(&ctl->mma_done[s]);
        }
        if (!ok) ctl->abort = 1;
    } else if (producer) {
        // tile i reuses stage i % NS once the MMAs of tile i - NS have read it
        bool ok = true;
        for (int i = NS; ok && i < ntile; ++i) {
            const int s = i % NS;
            ok = ix_wait(ctl, &ctl->mma_done[s], ((i / NS) - 1) & 1);
            if (ok) load(i);
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
            const int s = i % NS;
            const int p = (rg.t0 + i) * kIxTile + tid;
            bool is_cand = false;
            if (req_ok && p < P) {
                const long long last = f + (long long)p * KP + KP - 1;
                is_cand = svalid[p - rg.p_lo] != 0 && last <= (long long)qp;
            }
            float score = -INFINITY;
            const bool ok = req_ok && __all_sync(0xffffffffu, ix_wait(ctl, &ctl->mma_done[s], (i / NS) & 1));
            if (ok) {
                tc::fence_after_sync();
                uint32_t d[kIxHeads];
                tc::tmem_ld16(tmem + kIxHeads * s + ((uint32_t)(32 * warp) << 16), d);
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
                akeys[p - rg.p_lo] = k;
                local_cand += k != 0u;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local_cand += __shfl_xor_sync(0xffffffffu, local_cand, off);
    if (lane == 0 && local_cand) atomicAdd(&ctl->ncand, local_cand);
    __syncthreads();

    // ---- 3. the cluster selects
    // Exchange: word t (thread t) and words 256, 257 go into slot r of
    // every CTA's buffer xi & 1; returns the buffer once all C slots of this
    // CTA's copy have arrived. Every CTA makes the same exchanges in the same
    // order (each decision below is taken on exchanged data alike everywhere).
    int xi = 0;
    auto exchange = [&](int v, int extra, int extra2) -> int {
        const int bf = xi & 1;
        ctl->xout[tid] = v;
        if (tid < kIxXWords - 256) ctl->xout[256 + tid] = tid == 0 ? extra : tid == 1 ? extra2 : 0;
        if (tid == 0) mbar_arrive_expect_tx(&ctl->xbar[bf], (uint32_t)(C - 1) * kIxXBytes);
        __syncthreads();
        // thread t sends 16-byte piece t % 65 to rank t / 65; this CTA's own slot
        // is a plain copy (seen by the CTA after the barrier below)
        const uint32_t dst0 = smem_u32(&ctl->xin[bf][r][0]), bar0 = smem_u32(&ctl->xbar[bf]);
        for (int t = tid; t < (int)(kIxXBytes / 16) * C; t += kIxThreads) {
            const int c = t / (kIxXBytes / 16), u = t - c * (kIxXBytes / 16);
            const int4 val = reinterpret_cast<const int4 *>(ctl->xout)[u];
            if (c == r)
                reinterpret_cast<int4 *>(&ctl->xin[bf][r][0])[u] = val;
            else
                st_async_v4(cluster_map(dst0 + 16u * (uint32_t)u, c), val, cluster_map(bar0, c));
        }
        if (tid == 0 && !mbar_wait_cluster(&ctl->xbar[bf], (xi >> 1) & 1)) ctl->abort = 1;
        ++xi;
        __syncthreads();
        return bf;
    };
    const int nloc = max(0, rg.p_hi - rg.p_lo);
    uint32_t prefix = 0, pmask = 0;
    int remaining = 0, nq = 0;
    bool counts_known = false;           // the lower ranks' counts came with the small list
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        {
            // this CTA's counts of the digit over its keys that match the prefix
            ctl->hloc[tid] = 0;
            __syncthreads();
            for (int i0 = warp * 32; i0 < nloc; i0 += kIxThreads) {
                const int i = i0 + lane;
                const uint32_t k = i < nloc ? akeys[i] : 0u;
                const bool m = i < nloc && (k & pmask) == prefix;
                hist_add_warp(ctl->hloc, m ? (k >> shift) & 0xFFu : 0x100u);
            }
            __syncthreads();
        }
        const int bf = exchange(ctl->hloc[tid], pass == 0 ? ctl->ncand : 0, 0);
        // the cluster's histogram (integer counts: the sum is the same everywhere)
        int t = 0;
        for (int c = 0; c < C; ++c) t += ctl->xin[bf][c][tid];
        ctl->hloc[tid] = t;
        if (pass == 0 && tid == 0) {
            int n = 0;
            for (int c = 0; c < C; ++c) n += ctl->xin[bf][c][256];
            ctl->req = ctl->abort ? 0 : n;
        }
        __syncthreads();
        if (pass == 0) {
            nq = min(SK, ctl->req);
            remaining = nq;
            if (nq == 0) break;
        }
        if (tid < 32) {
            // lane l owns bins 255-8l down to 248-8l
            int cbin[8], sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cbin[i] = ctl->hloc[255 - 8 * tid - i];
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
        if (pass == 1 && ctl->pick[2] <= 32) {
            // At most 32 keys share the answer's top 16 bits: every CTA sends its
            // own (at most 32) with its count of keys above those 16 bits, and all
            // rank the same list on one warp; the lists and counts also give every
            // rank's keys above and equal to the answer, so no further exchange.
            if (tid == 0) {
                ctl->nsmall = 0;
                ctl->gt16 = 0;
            }
            __syncthreads();
            int above16 = 0;
            for (int i0 = warp * 32; i0 < nloc; i0 += kIxThreads) {
                const int i = i0 + lane;
                const uint32_t k = i < nloc ? akeys[i] : 0u;
                const bool m = i < nloc && (k & pmask) == prefix;
                above16 += __popc(__ballot_sync(0xffffffffu, i < nloc && (k & pmask) > prefix));
                const uint32_t bal = __ballot_sync(0xffffffffu, m);
                if (bal) {
                    int off = 0;
                    if (lane == 0) off = atomicAdd(&ctl->nsmall, __popc(bal));
                    off = __shfl_sync(0xffffffffu, off, 0);
                    if (m) ctl->small[off + __popc(bal & ((1u << lane) - 1u))] = k;
                }
            }
            if (lane == 0 && above16) atomicAdd(&ctl->gt16, above16);
            __syncthreads();
            const int ns = min(ctl->nsmall, 32);
            const int bs = exchange(tid < ns ? (int)ctl->small[tid] : 0, ns, ctl->gt16);
            if (tid < 32) {
                // lane l takes the l-th key of the ranks' lists laid end to end
                uint32_t mine = 0u;
                int n = 0;
                for (int c = 0; c < C; ++c) {
                    const int nc = min(ctl->xin[bs][c][256], 32);
                    if (tid >= n && tid < n + nc) mine = (uint32_t)ctl->xin[bs][c][tid - n];
                    n += nc;
                }
                n = min(n, 32);
                int gt = 0, ge = 0;
                for (int j = 0; j < n; ++j) {
                    const uint32_t kj = __shfl_sync(0xffffffffu, mine, j);
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
            if (tid == 0) {
                int g = 0, e = 0;
                for (int c = 0; c < r; ++c) {
                    const int nc = min(ctl->xin[bs][c][256], 32);
                    g += ctl->xin[bs][c][257];
                    for (int j = 0; j < nc; ++j) {
                        const uint32_t kj = (uint32_t)ctl->xin[bs][c][j];
                        g += kj > prefix;
                        e += kj == prefix;
                    }
                }
                ctl->rank_gt = g;
                ctl->rank_eq = e;
            }
            __syncthreads();
            counts_known = true;
            break;
        }
    }
    const uint32_t tau = prefix;     // the nq-th largest key (when nq > 0)
    const int req_eq = remaining;    // keys equal to tau to take, lowest ids first

    // ---- 4. winners in ascending pool id: every key above tau, then the req_eq
    // lowest-id keys equal to it. Warp w of CTA r takes a contiguous range of the
    // CTA's pools, 32 consecutive keys a step (ballot ranks); the places before it
    // are the counts of the lower ranks and of the lower warps. The CTA's winners
    // go to a list in the idle key ring, then their token ids are gathered with
    // every row's loads in flight at once.
    const size_t wrow = (size_t)SK * KP;
    const bool vec = (KP & 3) == 0 && aligned16(pool_idx) && aligned16(token_ids);
    if (nq > 0) {
        const int span = (((nloc + kIxWarps - 1) / kIxWarps) + 31) & ~31;
        const int wlo = min(nloc, warp * span), whi = min(nloc, wlo + span);
        const uint32_t below = (1u << lane) - 1u;
        int wgt = 0, weq = 0;
        for (int p0 = wlo; p0 < whi; p0 += 32) {
            const int i = p0 + lane;
            const uint32_t k = i < whi ? akeys[i] : 0u;
            wgt += __popc(__ballot_sync(0xffffffffu, i < whi && k > tau));
            weq += __popc(__ballot_sync(0xffffffffu, i < whi && k == tau));
        }
        if (lane == 0) ctl->warp2[warp] = make_int2(wgt, weq);
        __syncthreads();
        int cgt = 0, ceq = 0, gtw = 0, eqw = 0;
        for (int w2 = 0; w2 < kIxWarps; ++w2) {
            const int2 v = ctl->warp2[w2];
            cgt += v.x;
            ceq += v.y;
            if (w2 < warp) { gtw += v.x; eqw += v.y; }
        }
        int gtr = 0, eqr = 0;
        if (counts_known) {
            gtr = ctl->rank_gt;
            eqr = ctl->rank_eq;
        } else {
            const int bc = exchange(tid == 0 ? cgt : tid == 1 ? ceq : 0, 0, 0);
            for (int c = 0; c < r; ++c) {
                gtr += ctl->xin[bc][c][0];
                eqr += ctl->xin[bc][c][1];
            }
        }
        int eqs = eqr + eqw;
        int pos = gtr + gtw + min(eqs, req_eq);
        const int c_start = gtr + min(eqr, req_eq);                 // this CTA's places
        const int c_end = gtr + cgt + min(eqr + ceq, req_eq);
        int32_t *tlist = reinterpret_cast<int32_t *>(gbase);        // at most SK ids
        const int32_t *prow = pool_idx + (size_t)b * P * KP;
        for (int p0 = wlo; p0 < whi; p0 += 32) {
            const int i = p0 + lane;
            const uint32_t k = i < whi ? akeys[i] : 0u;
            const bool g = i < whi && k > tau, e = i < whi && k == tau;
            const uint32_t be = __ballot_sync(0xffffffffu, e);
            const bool take = g || (e && eqs + __popc(be & below) < req_eq);
            const uint32_t bt = __ballot_sync(0xffffffffu, take);
            if (take) {
                const int j = pos + __popc(bt & below);
                const int pid = rg.p_lo + i;
                top_pools[(size_t)q * SK + j] = pid;
                tlist[j - c_start] = pid;
            }
            pos += __popc(bt);
            eqs += __popc(be);
        }
        __syncthreads();
        const int nt = c_end - c_start;
        if (vec) {
            const int nv = KP >> 2;                         // 16-byte pieces a pool
            const int4 *src = reinterpret_cast<const int4 *>(prow);
            int4 *dst = reinterpret_cast<int4 *>(token_ids + (size_t)q * wrow) + (size_t)c_start * nv;
            for (int e = tid; e < nt * nv; e += kIxThreads) {
                const int jj = e / nv, u = e - jj * nv;
                dst[e] = __ldg(src + (size_t)tlist[jj] * nv + u);
            }
        } else {
            int32_t *dst = token_ids + (size_t)q * wrow + (size_t)c_start * KP;
            for (int e = tid; e < nt * KP; e += kIxThreads) {
                const int jj = e / KP, u = e - jj * KP;
                dst[e] = __ldg(prow + (size_t)tlist[jj] * KP + u);
            }
        }
    }
    // the -1 tail, slots [nq, SK), shared out over the cluster
    for (int j = nq + r * kIxThreads + tid; j < SK; j += C * kIxThreads) {
        top_pools[(size_t)q * SK + j] = -1;
        for (int u = 0; u < KP; ++u) token_ids[(size_t)q * wrow + (size_t)j * KP + u] = -1;
    }

    if (tid == 32) (void)mbar_wait(&ctl->q_bar, 0);   // the query rows' copy has landed
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kIxTmemCols);
}

// Clusters of 16 CTAs the device holds at once with the largest shared-memory
// size the kernel takes (asked once per device); 0 when none or unknown.
inline int indexer_max_clusters16() {
    static std::atomic<int> known[64];   // count + 1; 0 = not asked
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    const int k = known[dev].load(std::memory_order_relaxed);
    if (k != 0) return k - 1;
    const void *f = reinterpret_cast<const void *>(indexer_kernel);
    const int smem = indexer_smem_bytes(kIxMaxPools, kIxMaxCluster, kIxStages);
    int n = 0;
    if (ensure_smem_attr(f, smem) &&
        cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kIxMaxCluster, 1, 1);
        cfg.blockDim = dim3(kIxThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kIxMaxCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, indexer_kernel, &cfg) != cudaSuccess) n = 0;
    }
    (void)cudaGetLastError();
    known[dev].store(n + 1, std::memory_order_relaxed);
    return n;
}

// CTAs a query: 16 where clusters of 8 would leave most of the device idle (16
// CTAs a query still fit in one wave), every CTA gets at least two tiles and
// the device holds all Q clusters of 16 at once; 8 otherwise.
inline int indexer_cluster_size(int Q, int P) {
    const int tiles = (P + kIxTile - 1) / kIxTile;
    if ((long long)Q * kIxMaxCluster > sm_count() || tiles < 2 * kIxMaxCluster) return kIxCluster;
    return indexer_max_clusters16() >= Q ? kIxMaxCluster : kIxCluster;
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
    const int C = indexer_cluster_size(Q, max_pools);
    // ring depth: deep where the clusters fill at most one wave (each CTA then
    // streams many tiles), two stages otherwise, so two CTAs share an SM
    const int tpc = ceil_div(ceil_div(max_pools, kIxTile), C);
    int NS = (long long)Q * C <= sm_count() ? std::max(2, std::min(kIxStages, tpc)) : 2;
    // as deep as the block's shared-memory limit allows
    cudaFuncAttributes fa;
    int dev = 0, optin = 0;
    if (cudaFuncGetAttributes(&fa, indexer_kernel) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return DSA_ERR_CUDA;
    while (NS > 2 && (long long)fa.sharedSizeBytes + indexer_smem_bytes(max_pools, C, NS) > optin) --NS;
    const int smem = indexer_smem_bytes(max_pools, C, NS);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(indexer_kernel), smem)) return DSA_ERR_CUDA;
    if (launch_pdl_cluster(indexer_kernel, dim3(C, Q), dim3(kIxThreads), smem, stream, C, key_map, q_map, hidden, w, K, H, q_req, q_pos, pool_valid,
                           first_valid, pool_idx, B, kpool, max_pools, select_k, gate_w, scores,
                           cand, top_pools, token_ids, NS) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
