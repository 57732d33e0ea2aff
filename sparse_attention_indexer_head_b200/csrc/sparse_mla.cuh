// a7. NoPE MLA restricted to the selected tokens
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" last
// arrow; MASKED_ATTN_MAX_KEYS doc: the reference is dense attention under a
// set-membership mask, so gathering the selected rows is exact; trap 5: NoPE,
// the 512-wide latent row is both key and value).
//
// Split-KV decode on the 5th-generation tensor cores: a query's W selected ids
// are cut into S contiguous splits; one CTA per (split, query, 64-head group)
// gathers its latent rows and runs an online softmax for every head.
// The S partials (O, running max m, running sum l) of a (query, head group)
// are merged in split order, so results do not depend on scheduling: with
// S == 1 the CTA normalises and writes bf16 out and the lse itself; otherwise
// the partials go to the workspace and a combine kernel merges them.
#pragma once

#include "common.cuh"
#include "tc_ptx.cuh"

namespace dsa {

constexpr int kL = DSA_KV_LORA;      // 512
// Split partials in the workspace: the unnormalised O rows as bf16
// [Q][S][Hm][512] (1 KB a row), then (m, l) as float2 [Q][S][Hm]. O is rounded
// to bf16 once, like the P weights of the PV product: each rounding moves an
// output by at most 2^-9 of the largest selected value in its channel.
constexpr size_t kPartRowBytes = kL * 2 + 8;

// ---------------------------------------------------------------------------------------
// tcgen05 split-KV kernel. One CTA per (split, query, group of 64 heads).
//
// Per chunk of 48 selected tokens:
//   S[64 heads x 48 tokens]   = Q[64 x 512] . KV[48 x 512]^T   (M=64, N=48, 32 K-steps,
//                               as four K-quarters into four accumulators)
//   softmax over the chunk's tokens, per head row (two threads a head)
//   O^T[512 x 64 heads]      += KV^T[512 x 48] . P^T[48 x 64]  (4 x M=128, N=64, 3 K-steps)
// The latent row is both key and value (NoPE), so one 128B-swizzled shared tile
// of the gathered rows serves as the K-major B operand of S and as the MN-major A
// operand of O^T. Accumulators live in tensor memory: O^T in columns [0,256)
// (all 128 lanes), the four S parts in columns [256,448) (lanes 0-15 of each
// 32-lane quadrant, the M=64 layout).
//
// Warp roles (512 threads): warp 0 allocates tensor memory; lane 0 of each of
// warps 0-3 issues MMAs in an event loop over the barriers (its K-quarter of S
// as soon as the chunk has landed and the softmax has read the previous S, its
// 128-latent block of PV as soon as the chunk's P is ready); warps 8-15 gather,
// two groups of four warps filling alternate 48-token slots of a 3-slot ring
// with 16-byte cp.async pieces straight into the 128B-swizzled layout (a zero
// fill for ids that are -1 or outside the request). The copies' landing is
// tracked by the slot's mbarrier (cp.async.mbarrier.arrive), so no gather warp
// waits for its own copies. (Per-row TMA copies -- tile::gather4 or a 1-D bulk
// copy per 1 KB row -- move only 12-20 GB/s per SM here, bounded by their
// per-instruction cost; cp.async reaches about 37 GB/s per SM once a slot is
// spread over four warps.) Warps 4-7 load Q, run the softmax, rescale O^T when
// a head's running max grows by more than 2^8 (lazy rescaling); all sixteen
// warps write the epilogue.
// ---------------------------------------------------------------------------------------
constexpr int kTcThreads = 512;
constexpr int kTcChunk = 48;                        // tokens per chunk (one S tile, one PV pass)
constexpr int kTcSlots = 3;                         // ring slots, one chunk each
constexpr int kTcHeads = 64;
constexpr uint32_t kOffQ = 0;                       // 64 KB: 8 atoms x [64 rows x 128 B]
constexpr uint32_t kOffKV = 64 * 1024;              // 144 KB: 8 atoms x [144 rows x 128 B]
constexpr uint32_t kAtomKV = kTcSlots * kTcChunk * 128;   // 18 KB: one 64-latent column of the ring
constexpr uint32_t kSlotRows = kTcChunk * 128;      // 6 KB: a slot's rows within an atom
constexpr uint32_t kOffP = kOffKV + 8 * kAtomKV;    // 2 buffers x 8 KB: [64 heads x 128 B], 128B swizzle
constexpr uint32_t kStageP = 8 * 1024;
constexpr uint32_t kOffCtl = kOffP + 2 * kStageP;
constexpr uint32_t kTmemCols = 512;
// MMAs are issued by one thread in each of warps 0-3: a single issuing thread
// starts about one tcgen05.mma every 128 cycles whatever the tile, and issuers
// in different warps proceed in parallel. Each of the four issues one K-quarter
// of S into its own accumulator (the softmax adds the four) and the PV of one
// 128-latent block of O^T. The four S parts fill the columns O^T leaves, so S
// has one buffer: S(c+1) waits only for the softmax to have read S(c).
constexpr int kIssuers = 4;
constexpr int kSParts = 4;
constexpr int kSBufs = 1;
constexpr uint32_t kSCol = 256;                     // S: [256, 256 + kSBufs * kSParts * chunk)
static_assert(kSCol + kSBufs * kSParts * kTcChunk <= kTmemCols, "tensor memory columns");
static_assert(kSParts <= kIssuers && kSParts % 2 == 0, "S parts: one issuer each, read in pairs");
constexpr float kLazyRescale = 8.0f;                // log2 units
constexpr int kSmTarget = 148;                      // CTAs of one full wave (one CTA per SM)
constexpr int kMinSplitChunks = 4;                  // chunks a split holds, where there are enough
static_assert(kOffP % 1024 == 0, "P buffers hold 128B-swizzle atoms");

struct TcCtl {
    uint64_t kv_full[kTcSlots], kv_empty[kTcSlots];
    uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2];
    uint64_t o_done, o_final, q_full, fin;
    uint16_t vmask[kTcSlots][4];          // validity of a slot's rows, 12 rows per gather warp
    float alpha[kTcHeads];
    float lsum[kTcHeads];
    float mfin[kTcHeads];
    uint32_t tmem_base;
    int have_o;                           // the epilogue reads O^T (set by the softmax warps)
    volatile int abort;
};
constexpr int kTcSmemBytes = (int)kOffCtl + (int)sizeof(TcCtl) + 1024;   // + alignment slack
static_assert(kTcSmemBytes <= 232448, "shared memory per block");

struct MlaGeom {
    int S;         // splits per (query, head group)
    int per;       // selected-id slots per split (a multiple of the chunk)
};

// The split plan, the same on every device: as many splits as keep the grid
// within one wave of CTAs, no split holding more chunks than needed for that,
// but at least kMinSplitChunks chunks a split (half the row's chunks when it
// has fewer): each CTA's first gather and its epilogue cost about as much as a
// few chunks, so more splits of fewer chunks end later. Every split then holds
// at least one id. Splits merge through global partials and the combine kernel
// (a merge inside thread-block clusters, measured at the same split counts,
// was slower on every workload).
inline MlaGeom mla_plan(int Q, int Hm, int W) {
    MlaGeom g{1, kTcChunk};
    if (Q <= 0 || W <= 0) return g;
    const long long ctas = (long long)Q * ((Hm + kTcHeads - 1) / kTcHeads);
    const int chunks = ceil_div(W, kTcChunk);
    int per_chunks = chunks;
    if (ctas < kSmTarget) {
        per_chunks = ceil_div(chunks, (int)(kSmTarget / ctas));
        per_chunks = std::max(per_chunks, std::min(kMinSplitChunks, ceil_div(chunks, 2)));
    }
    g.per = per_chunks * kTcChunk;
    g.S = ceil_div(chunks, per_chunks);
    return g;
}

inline size_t mla_workspace_bytes(int Q, int Hm, int W) {
    if (Q <= 0 || Hm <= 0) return 0;
    const MlaGeom g = mla_plan(Q, Hm, W);
    if (g.S == 1) return 0;
    return (size_t)Q * g.S * Hm * kPartRowBytes;
}

DSA_DEVINL bool tc_wait(TcCtl *ctl, uint64_t *bar, uint32_t parity) {
    if (ctl->abort) return false;
    if (!mbar_wait(bar, parity)) {
        ctl->abort = 1;
        return false;
    }
    return true;
}

// Two E4M3 values (low byte first) widened to a bf16 pair: through f16, exact
// for every E4M3 value (at most 4 significant bits, exponents 2^-9 .. 2^8).
DSA_DEVINL uint32_t e4m3x2_to_bf16x2(uint16_t v) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
    float lo, hi;
    asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return pack_bf16x2(lo, hi);
}

// Where a request's logical token t lives in the latent cache. Contiguous:
// row req_start[b] + t, t < T_b = req_start[b+1] - req_start[b]. Paged (a
// block table, block_table != nullptr): row block_table[b][t / page] * page +
// t % page, t < T_b = seq_len[b]; a negative block number or a block index past
// max_blocks makes the token invalid. Either way a row at or past kv_rows is
// never read (the token counts as invalid).
struct KvMap {
    const int32_t *req_start;
    const int32_t *block_table;   // [B, max_blocks] or nullptr
    const int32_t *seq_len;       // [B] (paged)
    int max_blocks, page;
};

// kv: the latent cache, kv_rows rows of 512 bf16, or of 512 E4M3 bytes (kFp8:
// the MMA takes them widened to bf16, which is exact; the cache-wide scale is
// folded into scale_log2 and out_scale).
template <bool kPaged, bool kFp8>
__global__ void __launch_bounds__(kTcThreads, 1)
mla_tc_kernel(const __nv_bfloat16 *__restrict__ qm, const void *__restrict__ kv_raw,
              const KvMap map, const int32_t *__restrict__ q_req,
              const int32_t *__restrict__ token_ids, int B, int kv_rows, int Hm, int W, int S,
              int per, float scale_log2, float out_scale, uint8_t *__restrict__ part,
              __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    extern __shared__ uint8_t mla_smem_raw[];
    const uint32_t raw = smem_u32(mla_smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;           // 128B-swizzle atoms need 1 KB
    uint8_t *gbase = mla_smem_raw + (base - raw);
    TcCtl *ctl = reinterpret_cast<TcCtl *>(gbase + kOffCtl);
    const uint32_t sQ = base + kOffQ;
    const uint32_t sKV = base + kOffKV;                      // stage s: rows [32s, 32s+32) of each atom
    const uint32_t sP = base + kOffP;                        // buffer b at sP + b * kStageP

    const int split = blockIdx.x, qi = blockIdx.y, hg = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j0 = min(W, split * per), j1 = min(W, j0 + per);
    const int ntok = j1 - j0;
    const int nch = (ntok + kTcChunk - 1) / kTcChunk;
    const int h0 = hg * kTcHeads, nh = min(kTcHeads, Hm - h0);
    // Request geometry is a step input: its loads go out before the set-up and are
    // used after the wait on the predecessor.
    const int b = q_req[qi];
    const bool req_ok = b >= 0 && b < B;
    int rs = 0, T = 0;
    if (req_ok) {
        if constexpr (kPaged) {
            T = max(0, map.seq_len[b]);
        } else {
            rs = map.req_start[b];
            T = max(0, map.req_start[b + 1] - rs);
        }
    }

    if (warp >= 4 && warp < 8) {
        // Q tile (a step input): 64 rows x 64 16-byte chunks into the swizzled
        // K-major layout, issued before the predecessor grid finishes.
        for (int x = tid - 128; x < kTcHeads * 64; x += 128) {
            const int h = x >> 6, cc = x & 63;
            const uint32_t dst = sQ + (cc >> 3) * 8192 + h * 128 + (((cc & 7) ^ (h & 7)) << 4);
            if (h < nh)
                tc::cp_async16(dst, qm + ((size_t)qi * Hm + h0 + h) * kL + cc * 8);
            else
                tc::st_shared_zero16(dst);
        }
    }

    if (warp == 0) {
        tc::tmem_alloc(&ctl->tmem_base, kTmemCols);
        tc::tmem_relinquish();
    }
    if (tid == 32) {
        for (int i = 0; i < kTcSlots; ++i) {
            mbar_init(&ctl->kv_full[i], 4 * 32 + 4);   // four warps' lanes' copies + their masks' arrives
            mbar_init(&ctl->kv_empty[i], kIssuers);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->s_full[i], kSParts);
            mbar_init(&ctl->s_empty[i], 128);
            mbar_init(&ctl->p_full[i], 128);
            mbar_init(&ctl->p_empty[i], kIssuers);
        }
        mbar_init(&ctl->o_done, kIssuers);
        mbar_init(&ctl->o_final, kIssuers);
        mbar_init(&ctl->q_full, 128);
        mbar_init(&ctl->fin, kIssuers);
        ctl->abort = 0;
        fence_mbarrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    pdl_wait();                       // token ids come from the predecessor grid
    pdl_launch_dependents();

    if (warp < kIssuers) {
        // ------------------------------------------------------------------ MMA issuers
        // Lane 0 of warp w issues the PV of latent block w and the K-quarter w of
        // every S.
        if (lane == 0 && nch > 0) {
            const int w = warp;
            const bool s_issuer = w < kSParts;
            constexpr uint32_t idS = tc::idesc_bf16(64, kTcChunk, false, false);
            constexpr uint32_t idPV = tc::idesc_bf16(128, 64, true, false);
            // Chunk c lives in ring slot c % 3: rows [48 slot, 48 slot + 48) of every
            // 144-row column atom.
            // PV(cp), block w: O^T[128w .. 128w+127] += V^T P^T over the chunk's 48
            // tokens (three K-steps).
            auto issue_pv = [&](int cp) {
                const int slot = cp % kTcSlots, pb = cp & 1;
                tc::fence_after_sync();
                tc::fence_proxy_async_smem();     // the slot was written by cp.async
#pragma unroll
                for (int ks = 0; ks < kTcChunk / 16; ++ks) {
                    // V^T: MN-major, 64-latent atoms kAtomKV apart, 8-token groups 1 KB apart
                    const uint64_t a = tc::desc_sw128(sKV + w * 2 * kAtomKV + slot * kSlotRows + ks * 2048,
                                                      kAtomKV, 1024);
                    // P^T: K-major, 128-byte rows (48 of 64 tokens used), 8-head groups 1 KB apart
                    const uint64_t bd = tc::desc_sw128(sP + pb * kStageP + ks * 32, 16, 1024);
                    tc::mma_bf16_ss(tmem + w * 64, a, bd, idPV, (cp > 0 || ks > 0) ? 1u : 0u);
                }
                tc::mma_commit(&ctl->kv_empty[slot]);
                tc::mma_commit(&ctl->p_empty[pb]);
                tc::mma_commit(&ctl->o_done);
            };
            // S(c), K-quarter w = Q K^T over latent [128w, 128w + 128) of chunk c's
            // 48 tokens, into part w of the S buffer.
            auto issue_s = [&](int c) {
                const int slot = c % kTcSlots, sb = c % kSBufs;
                tc::fence_after_sync();
                tc::fence_proxy_async_smem();     // the slot was written by cp.async
                const uint32_t d = tmem + kSCol + (uint32_t)((sb * kSParts + w) * kTcChunk);
                constexpr int kPart = kL / 16 / kSParts;
#pragma unroll
                for (int k2 = 0; k2 < kPart; ++k2) {
                    const int kk = w * kPart + k2;
                    const uint32_t qo = (kk >> 2) * 8192 + (kk & 3) * 32;
                    const uint32_t ko = (kk >> 2) * kAtomKV + slot * kSlotRows + (kk & 3) * 32;
                    tc::mma_bf16_ss(d, tc::desc_sw128(sQ + qo, 16, 1024),
                                    tc::desc_sw128(sKV + ko, 16, 1024), idS, k2 > 0 ? 1u : 0u);
                }
                tc::mma_commit(&ctl->s_full[sb]);
            };
            // Event loop: issue whichever product is ready, PV first (it frees a
            // slot for the gathers); give up after the wait bound without progress.
            bool ok = tc_wait(ctl, &ctl->q_full, 0);
            int ns = s_issuer ? 0 : nch, np = 0;
            long long t_last = clock64();
            while (ok && np < nch) {
                if ((np < ns || !s_issuer) && mbar_test(&ctl->p_full[np & 1], (np >> 1) & 1)) {
                    // the softmax of chunk np waited for its rows: they have landed
                    issue_pv(np++);
                    t_last = clock64();
                    continue;
                }
                if (s_issuer && ns < nch) {
                    const bool ready = mbar_test(&ctl->kv_full[ns % kTcSlots], (ns / kTcSlots) & 1) &&
                                       (ns < kSBufs ||
                                        mbar_test(&ctl->s_empty[ns % kSBufs], ((ns / kSBufs) - 1) & 1));
                    if (ready) {
                        issue_s(ns++);
                        t_last = clock64();
                        continue;
                    }
                }
                if (ctl->abort) { ok = false; break; }
                if (clock64() - t_last > kWaitLimitCycles) {
                    raise_device_error(kErrWaitTimeout);
                    ctl->abort = 1;
                    ok = false;
                }
            }
            // o_final is single-use: once it completes every PV of this CTA has landed
            // (a parity wait on o_done cannot tell the last two PVs apart).
            if (ok) tc::mma_commit(&ctl->o_final);
            // every MMA of this issuer has completed before tensor memory is released
            tc::mma_commit(&ctl->fin);
        }
        __syncwarp();
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ gather warps
        // Two groups of four warps (warps 8-11, 12-15) fill alternate chunks
        // (group p: chunks p, p+2, ...); warp i of a group copies rows 12i..12i+11
        // of the chunk's slot as 16-byte cp.async pieces straight into the swizzled
        // layout (zero-filled for invalid ids) and records their validity. Each
        // lane's copies arrive on the slot's barrier as they land, so no warp waits
        // for its own copies.
        const int grp = (warp - 8) >> 2, sub = (warp - 8) & 3;
        auto load_id = [&](int c) -> int {         // lane l < 12: row 12 sub + l of chunk c
            const int j = c * kTcChunk + 12 * sub + lane;
            return (lane < 12 && c < nch && j < ntok) ? __ldg(token_ids + (size_t)qi * W + j0 + j) : -1;
        };
        // cache row of a logical id, -1 when the id is not a valid token
        auto resolve = [&](int id) -> int {
            if (id < 0 || id >= T) return -1;
            long long r;
            if constexpr (kPaged) {
                const int bi = id / map.page;
                if (bi >= map.max_blocks) return -1;
                const int blk = __ldg(map.block_table + (size_t)b * map.max_blocks + bi);
                if (blk < 0) return -1;
                r = (long long)blk * map.page + (id - bi * map.page);
            } else {
                r = (long long)rs + id;
            }
            return r < (long long)kv_rows ? (int)r : -1;
        };
        auto gather_chunk = [&](int c, int myrow) -> bool {
            const int slot = c % kTcSlots;
            bool ok = true;
            if (c >= kTcSlots) ok = tc_wait(ctl, &ctl->kv_empty[slot], ((c / kTcSlots) - 1) & 1);
            if (!__all_sync(0xffffffffu, ok)) return false;
            const uint32_t vm = __ballot_sync(0xffffffffu, myrow >= 0);   // bits 0..11
            const uint32_t dst0 = sKV + slot * kSlotRows;
            if constexpr (!kFp8) {
                const auto *kv = reinterpret_cast<const __nv_bfloat16 *>(kv_raw);
#pragma unroll
                for (int rr = 0; rr < 12; ++rr) {
                    const int r = 12 * sub + rr;                 // row within the chunk
                    const int row = __shfl_sync(0xffffffffu, myrow, rr);
                    const __nv_bfloat16 *src = row >= 0 ? kv + (size_t)row * kL : qm;   // qm: never read
                    const uint32_t nb = row >= 0 ? 16u : 0u;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int cc = lane + 32 * hh;         // 16-byte piece of the 1 KB row
                        const uint32_t dst = dst0 + (cc >> 3) * kAtomKV + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
                        tc::cp_async16_zfill(dst, row >= 0 ? src + cc * 8 : src, nb);
                    }
                }
                if (lane == 0) {
                    ctl->vmask[slot][sub] = (uint16_t)vm;
                    mbar_arrive(&ctl->kv_full[slot]);          // releases this warp's mask
                }
                tc::cp_async_arrive_noinc(&ctl->kv_full[slot]);
            } else {
                // E4M3 rows of 512 bytes: lane l loads channels 16l..16l+15 of each of
                // the warp's 12 rows (all loads in flight first), widens them to bf16
                // exactly and stores the two 16-byte pieces into the swizzled layout.
                const auto *kv8 = reinterpret_cast<const uint8_t *>(kv_raw);
                uint4 raw[12];
#pragma unroll
                for (int rr = 0; rr < 12; ++rr) {
                    const int row = __shfl_sync(0xffffffffu, myrow, rr);
                    raw[rr] = row >= 0 ? ldg_nc_v4(kv8 + (size_t)row * kL + 16 * lane)
                                       : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int rr = 0; rr < 12; ++rr) {
                    const int r = 12 * sub + rr;
                    const uint32_t w[4] = {raw[rr].x, raw[rr].y, raw[rr].z, raw[rr].w};
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int cc = 2 * lane + hh;          // 16-byte piece of the bf16 row
                        const uint32_t dst = dst0 + (cc >> 3) * kAtomKV + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
                        const uint32_t a = w[2 * hh], bword = w[2 * hh + 1];
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                     "r"(e4m3x2_to_bf16x2((uint16_t)(a & 0xFFFFu))),
                                     "r"(e4m3x2_to_bf16x2((uint16_t)(a >> 16))),
                                     "r"(e4m3x2_to_bf16x2((uint16_t)(bword & 0xFFFFu))),
                                     "r"(e4m3x2_to_bf16x2((uint16_t)(bword >> 16)))
                                     : "memory");
                    }
                }
                tc::fence_proxy_async_smem();               // generic stores -> tensor-core reads
                if (lane == 0) {
                    ctl->vmask[slot][sub] = (uint16_t)vm;
                    mbar_arrive(&ctl->kv_full[slot]);
                }
                mbar_arrive(&ctl->kv_full[slot]);            // this lane's rows are in place
            }
            return true;
        };
        bool go = true;
        if constexpr (!kPaged) {
            // ids of the group's next two chunks are in flight (static queue slots)
            int idq[2] = {load_id(grp), load_id(grp + 2)};
            for (int c0 = grp; go && c0 < nch; c0 += 4) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c0 + 2 * u;
                    if (!go || c >= nch) break;
                    const int id = idq[u];
                    idq[u] = load_id(c + 4);
                    go = gather_chunk(c, resolve(id));
                }
            }
        } else {
            // The block-table lookup is a second dependent load: rows are resolved
            // two of the group's chunks ahead, ids loaded four ahead.
            int rq[2] = {resolve(load_id(grp)), resolve(load_id(grp + 2))};
            int idq[2] = {load_id(grp + 4), load_id(grp + 6)};
            for (int c0 = grp; go && c0 < nch; c0 += 4) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c = c0 + 2 * u;
                    if (!go || c >= nch) break;
                    const int row = rq[u];
                    rq[u] = resolve(idq[u]);
                    idq[u] = load_id(c + 8);
                    go = gather_chunk(c, row);
                }
            }
        }
        tc::cp_async_wait_all();          // nothing of this warp in flight past here
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ softmax (warps 4-7)
        // S is read with the 16x64b tensor-memory shape, so every lane works:
        // thread t of warp 4+w holds head row hh = 16w + (t>>2) + 8(t&1) and the
        // chunk's tokens of parity par = (t>>1)&1; its partner t^2 holds the
        // other parity of the same head. Row max and sum take one exchange.
        const int wq = warp - 4;
        const int hh = 16 * wq + (lane >> 2) + 8 * (lane & 1);
        const int par = (lane >> 1) & 1;
        const bool owner = par == 0;          // writes the head's per-row values
        tc::cp_async_wait_all();          // this thread's Q copies (issued at entry)
        tc::fence_proxy_async_smem();
        mbar_arrive(&ctl->q_full);

        const uint32_t tl = tmem + ((uint32_t)(32 * wq) << 16);
        float m_used = -INFINITY, l = 0.f;
        bool failed = false;
        for (int c = 0; c < nch; ++c) {
            const int slot = c % kTcSlots, sb = c & 1, sbuf = c % kSBufs;
            bool bad = !tc_wait(ctl, &ctl->kv_full[slot], (c / kTcSlots) & 1);
            bad = bad || !tc_wait(ctl, &ctl->s_full[sbuf], (c / kSBufs) & 1);
            tc::fence_after_sync();
            // 48 columns of each S part: this thread's 24 tokens par + 2i, i < 24;
            // the parts are read two at a time and summed pairwise, (p0+p1)+(p2+p3)
            float sacc[24];
            const uint32_t sc0 = tl + kSCol + (uint32_t)(sbuf * kSParts * kTcChunk);
#pragma unroll
            for (int pp = 0; pp < kSParts; pp += 2) {
                uint32_t r[24], r2[24];
                const uint32_t a0 = sc0 + (uint32_t)(pp * kTcChunk);
                tc::tmem_ld16x64b_x16(a0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                tc::tmem_ld16x64b_x8(a0 + 32, *reinterpret_cast<uint32_t(*)[8]>(&r[16]));
                tc::tmem_ld16x64b_x16(a0 + kTcChunk, *reinterpret_cast<uint32_t(*)[16]>(&r2[0]));
                tc::tmem_ld16x64b_x8(a0 + kTcChunk + 32, *reinterpret_cast<uint32_t(*)[8]>(&r2[16]));
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 24; ++i) {
                    const float t2 = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
                    sacc[i] = pp == 0 ? t2 : sacc[i] + t2;
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&ctl->s_empty[sbuf]);

            // validity of the chunk's 48 rows (12 per gather warp), then bit 2i: token par + 2i
            const uint64_t vm48 = (uint64_t)ctl->vmask[slot][0] | ((uint64_t)ctl->vmask[slot][1] << 12) |
                                  ((uint64_t)ctl->vmask[slot][2] << 24) | ((uint64_t)ctl->vmask[slot][3] << 36);
            const uint64_t vmp = vm48 >> par;
            float z[24];
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 24; ++i) {
                z[i] = ((vmp >> (2 * i)) & 1) ? sacc[i] * scale_log2 : -INFINITY;
                mx = fmaxf(mx, z[i]);
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            float alpha = 1.f;
            if (mx > m_used + kLazyRescale) {
                alpha = ex2(m_used - mx);
                m_used = mx;
            }
            float pv[24];
            float psum = 0.f;
#pragma unroll
            for (int i = 0; i < 24; ++i) {
                pv[i] = z[i] == -INFINITY ? 0.f : ex2(z[i] - m_used);
                psum += pv[i];       // fp32 weights: the row sum and lse stay exact to fp32
            }
            psum += __shfl_xor_sync(0xffffffffu, psum, 2);
            l = fmaf(l, alpha, psum);
            if (owner) ctl->alpha[hh] = alpha;
            // bf16 P row of the head: this thread packs tokens 24par .. 24par+23,
            // taking the other parity from its partner.
            uint32_t pk[12];
#pragma unroll
            for (int k = 0; k < 12; ++k) {
                const float recv = __shfl_xor_sync(0xffffffffu, par ? pv[k] : pv[k + 12], 2);
                pk[k] = par ? pack_bf16x2(recv, pv[k + 12]) : pack_bf16x2(pv[k], recv);
            }

            bad = bad || (c >= 2 && !tc_wait(ctl, &ctl->p_empty[sb], ((c >> 1) - 1) & 1));
            // One barrier per chunk; a second only when some head rescales or a wait failed.
            bool need = false;
            if (tc::named_bar_or(2, 128, bad || (owner && c >= 1 && alpha != 1.f))) {
                if (tc::named_bar_or(2, 128, bad)) { failed = true; break; }
                need = true;
            }
#pragma unroll
            for (int q3 = 0; q3 < 3; ++q3) {
                const int c16 = 3 * par + q3;     // 16-byte piece of the 128-byte row (pieces 6, 7 unused)
                const uint32_t dst = sP + sb * kStageP + hh * 128 + ((c16 ^ (hh & 7)) << 4);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                             "r"(pk[4 * q3]), "r"(pk[4 * q3 + 1]), "r"(pk[4 * q3 + 2]),
                             "r"(pk[4 * q3 + 3])
                             : "memory");
            }
            if (need) {
                // O^T columns of rescaled heads times alpha, after PV(c-1) has landed.
                bad = !tc_wait(ctl, &ctl->o_done, (c - 1) & 1);
                if (tc::named_bar_or(2, 128, bad)) { failed = true; break; }
                tc::fence_after_sync();
#pragma unroll 1
                for (int blk = 0; blk < 8; ++blk) {
                    uint32_t o[32];
                    const uint32_t ta = tl + (blk >> 1) * 64 + (blk & 1) * 32;
                    tc::tmem_ld32(ta, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        o[j] = __float_as_uint(__uint_as_float(o[j]) * ctl->alpha[(blk & 1) * 32 + j]);
                    tc::tmem_st32(ta, o);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
            }
            tc::fence_proxy_async_smem();
            mbar_arrive(&ctl->p_full[sb]);
        }

        // ------------------------------------------------------------------ epilogue
        bool have_o = !failed && nch > 0;
        if (have_o) {
            const bool bad = !tc_wait(ctl, &ctl->o_final, 0);
            have_o = !tc::named_bar_or(2, 128, bad);
        }
        if (owner) ctl->lsum[hh] = l;
        tc::named_bar_sync(2, 128);
        // O^T is written after the CTA barrier below, by all sixteen warps.
        if (owner) ctl->mfin[hh] = have_o ? m_used : -INFINITY;
        if (tid == 128) ctl->have_o = have_o ? 1 : 0;
        if (S == 1 && lse && owner && hh < nh)
            lse[(size_t)qi * Hm + h0 + hh] =
                (have_o && l > 0.f) ? (m_used + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }

    // Every MMA of this CTA has completed before tensor memory is released.
    if (warp == 0 && lane == 0 && nch > 0) (void)mbar_wait(&ctl->fin, 0);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    {
        // O^T out of tensor memory by all sixteen warps: warp w reads the lane
        // quarter w % 4 (32 latent rows of each 128-row block) for two of the
        // eight (latent block, 32-head half) pieces; each store writes 32
        // consecutive latent values of one head (128 bytes).
        const int quarter = warp & 3;
        const uint32_t tq = tmem + ((uint32_t)(32 * quarter) << 16);
        const bool have_o = ctl->have_o != 0;
        if (S > 1) {
            const size_t row0 = (size_t)(qi * S + split) * Hm + h0;
            __nv_bfloat16 *po = reinterpret_cast<__nv_bfloat16 *>(part) + row0 * kL;
            float2 *pml = reinterpret_cast<float2 *>(part + (size_t)gridDim.y * S * Hm * kL * 2) + row0;
            if (have_o) {
                // Lanes 2i and 2i+1 hold latent columns L, L+1: the even lane
                // writes both columns of heads j, the odd lane of heads j+1.
                const bool odd = lane & 1;
#pragma unroll 1
                for (int bi = 0; bi < 2; ++bi) {
                    const int blk = 2 * (warp >> 2) + bi;
                    uint32_t o[32];
                    tc::tmem_ld32(tq + (blk >> 1) * 64 + (blk & 1) * 32, o);
                    tc::tmem_wait_ld();
                    const int L2 = (blk >> 1) * 128 + 32 * quarter + (lane & ~1);
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float x = __shfl_xor_sync(0xffffffffu, __uint_as_float(odd ? o[j] : o[j + 1]), 1);
                        const int h = (blk & 1) * 32 + j + (odd ? 1 : 0);
                        const uint32_t v = odd ? pack_bf16x2(x, __uint_as_float(o[j + 1]))
                                               : pack_bf16x2(__uint_as_float(o[j]), x);
                        if (h < nh) *reinterpret_cast<uint32_t *>(po + (size_t)h * kL + L2) = v;
                    }
                }
            }
            if (tid < kTcHeads && tid < nh)
                pml[tid] = make_float2(ctl->mfin[tid], have_o ? ctl->lsum[tid] : 0.f);
        } else {
            // single split: normalise here and write bf16 out directly
            __nv_bfloat16 *ob = out + ((size_t)qi * Hm + h0) * kL;
#pragma unroll 1
            for (int bi = 0; bi < 2; ++bi) {
                const int blk = 2 * (warp >> 2) + bi;
                uint32_t o[32];
                if (have_o) {
                    tc::tmem_ld32(tq + (blk >> 1) * 64 + (blk & 1) * 32, o);
                    tc::tmem_wait_ld();
                }
                const int L = (blk >> 1) * 128 + 32 * quarter + lane;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int h = (blk & 1) * 32 + j;
                    const float lh = ctl->lsum[h];
                    const float v = (have_o && lh > 0.f) ? __uint_as_float(o[j]) / lh * out_scale : 0.f;
                    if (h < nh) ob[(size_t)h * kL + L] = __float2bfloat16_rn(v);
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();              // every tensor-memory read is done before the release
    }
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// One CTA per (head, query); 128 threads x 4 channels. Up to 16 splits are
// merged from one round of loads (every split's m, l and row in flight at once);
// more splits take a first round for the maxima. Splits are merged in split
// order (deterministic).
__global__ void __launch_bounds__(128)
mla_combine_kernel(const uint8_t *__restrict__ part, int Hm, int S, float out_scale,
                   __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    constexpr int kRound = 16;
    const int h = blockIdx.x, q = blockIdx.y, tid = threadIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    const size_t row0 = (size_t)q * S * Hm + h;                  // split u: row0 + u * Hm
    const __nv_bfloat16 *po = reinterpret_cast<const __nv_bfloat16 *>(part) + row0 * kL + 4 * tid;
    const float2 *pml = reinterpret_cast<const float2 *>(part + (size_t)gridDim.y * S * Hm * kL * 2) + row0;
    const size_t sstride = (size_t)Hm * kL;
    float M = -INFINITY;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    float lsum = 0.f;
    auto accum = [&](float m, float l, uint2 v) {
        if (m == -INFINITY) return;
        const float w = ex2(m - M);
        lsum = fmaf(l, w, lsum);
        o[0] = fmaf(bf16lo(v.x), w, o[0]);
        o[1] = fmaf(bf16hi(v.x), w, o[1]);
        o[2] = fmaf(bf16lo(v.y), w, o[2]);
        o[3] = fmaf(bf16hi(v.y), w, o[3]);
    };
    if (S <= kRound) {
        float2 ml[kRound];
        uint2 v[kRound];
#pragma unroll
        for (int u = 0; u < kRound; ++u) {
            const bool in = u < S;
            ml[u] = in ? __ldg(pml + (size_t)u * Hm) : make_float2(-INFINITY, 0.f);
            v[u] = in ? __ldg(reinterpret_cast<const uint2 *>(po + u * sstride)) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kRound; ++u) M = fmaxf(M, ml[u].x);
        if (M != -INFINITY) {
#pragma unroll
            for (int u = 0; u < kRound; ++u) accum(ml[u].x, ml[u].y, v[u]);
        }
    } else {
        for (int s0 = 0; s0 < S; s0 += 8) {
            float mv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) mv[u] = s0 + u < S ? __ldg(pml + (size_t)(s0 + u) * Hm).x : -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) M = fmaxf(M, mv[u]);
        }
        if (M != -INFINITY) {
            for (int s0 = 0; s0 < S; s0 += 8) {
                float2 ml[8];
                uint2 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const bool in = s0 + u < S;
                    ml[u] = in ? __ldg(pml + (size_t)(s0 + u) * Hm) : make_float2(-INFINITY, 0.f);
                    v[u] = in ? __ldg(reinterpret_cast<const uint2 *>(po + (s0 + u) * sstride))
                              : make_uint2(0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) accum(ml[u].x, ml[u].y, v[u]);
            }
        }
    }
    const float inv = lsum > 0.f ? out_scale / lsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(o[0] * inv, o[1] * inv);
    packed.y = pack_bf16x2(o[2] * inv, o[3] * inv);
    *reinterpret_cast<uint2 *>(out + ((size_t)q * Hm + h) * kL + 4 * tid) = packed;
    if (lse && tid == 0)
        lse[(size_t)q * Hm + h] = lsum > 0.f ? (M + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
}

// Kernels sparse_mla_launch runs for this shape: the split kernel, plus the
// combine when a query's ids are split.
inline int sparse_mla_launch_count(int Q, int Hm, int W) {
    if (Q <= 0 || Hm <= 0 || W < 0) return 0;
    return mla_plan(Q, Hm, W).S > 1 ? 2 : 1;
}

template <bool kPaged, bool kFp8>
inline int sparse_mla_launch_map(const void *q, const void *kv, int64_t kv_rows, const KvMap &map,
                                 float kv_scale, const int32_t *q_req, const int32_t *token_ids,
                                 int Q, int B, int Hm, int W, int kv_lora, int rope_dim,
                                 float sm_scale, void *out, float *lse, void *ws, size_t ws_bytes,
                                 cudaStream_t stream) {
    if (Q < 0 || B < 0 || Hm <= 0 || W < 0 || kv_lora <= 0 || rope_dim < 0 || kv_rows < 0)
        return DSA_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || sm_scale == INFINITY || sm_scale == -INFINITY)
        return DSA_ERR_INVALID_ARG;
    if (kPaged && (map.page <= 0 || map.max_blocks < 0)) return DSA_ERR_INVALID_ARG;
    if (kFp8 && !(kv_scale > 0.f && kv_scale < INFINITY)) return DSA_ERR_INVALID_ARG;
    if (kv_lora != kL || rope_dim != 0 || Hm % 16 != 0 || Hm > DSA_MAX_MLA_HEADS)
        return DSA_ERR_UNSUPPORTED;
    if (kv_rows > (int64_t)INT32_MAX) return DSA_ERR_UNSUPPORTED;   // rows are 32-bit indices
    if (Q == 0) return DSA_OK;
    if (Q > 65535) return DSA_ERR_UNSUPPORTED;
    if (!q || !q_req || !out || (W > 0 && !token_ids) || (kv_rows > 0 && !kv))
        return DSA_ERR_INVALID_ARG;
    if (B > 0 && (kPaged ? (!map.seq_len || (map.max_blocks > 0 && !map.block_table)) : !map.req_start))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(map.req_start, 4) ||
        !aligned(map.block_table, 4) || !aligned(map.seq_len, 4) || !aligned(q_req, 4) ||
        !aligned(token_ids, 4) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(ws, 16))
        return DSA_ERR_ALIGNMENT;
    const size_t need = mla_workspace_bytes(Q, Hm, W);
    if (need > 0 && (!ws || ws_bytes < need)) return DSA_ERR_WORKSPACE;
    if (!ensure_smem_attr(reinterpret_cast<const void *>(mla_tc_kernel<kPaged, kFp8>), kTcSmemBytes))
        return DSA_ERR_CUDA;
    const MlaGeom g = mla_plan(Q, Hm, W);
    // fp8: S = sm_scale * q . (s k8) = (sm_scale * s) q . k8, and O = s * (P V8)
    const float out_scale = kFp8 ? kv_scale : 1.0f;
    const float scale_log2 = (kFp8 ? sm_scale * kv_scale : sm_scale) * 1.4426950408889634f;
    const int groups = (Hm + kTcHeads - 1) / kTcHeads;
    auto *part = reinterpret_cast<uint8_t *>(ws);
    const auto *qb = reinterpret_cast<const __nv_bfloat16 *>(q);
    auto *ob = reinterpret_cast<__nv_bfloat16 *>(out);
    const dim3 grid(g.S, Q, groups);
    if (launch_pdl(mla_tc_kernel<kPaged, kFp8>, grid, dim3(kTcThreads), kTcSmemBytes,
                   stream, qb, kv, map, q_req, token_ids, B, (int)kv_rows, Hm, W, g.S, g.per,
                   scale_log2, out_scale, part, ob, lse) != cudaSuccess)
        return DSA_ERR_CUDA;
    int st = launch_status();
    if (st != DSA_OK || g.S == 1) return st;
    if (launch_pdl(mla_combine_kernel, dim3(Hm, Q), dim3(128), 0, stream, part, Hm, g.S,
                   out_scale, ob, lse) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

inline int sparse_mla_launch(const void *q, const void *kv, int64_t kv_rows,
                             const int32_t *req_start, const int32_t *q_req,
                             const int32_t *token_ids, int Q, int B, int Hm, int W, int kv_lora,
                             int rope_dim, float sm_scale, void *out, float *lse, void *ws,
                             size_t ws_bytes, cudaStream_t stream) {
    const KvMap map{req_start, nullptr, nullptr, 0, 1};
    return sparse_mla_launch_map<false, false>(q, kv, kv_rows, map, 1.0f, q_req, token_ids, Q, B,
                                               Hm, W, kv_lora, rope_dim, sm_scale, out, lse, ws,
                                               ws_bytes, stream);
}

inline int sparse_mla_launch_paged(const void *q, const void *kv, int64_t kv_rows,
                                   const int32_t *block_table, int max_blocks, int page_size,
                                   const int32_t *seq_len, const int32_t *q_req,
                                   const int32_t *token_ids, int Q, int B, int Hm, int W,
                                   int kv_lora, int rope_dim, float sm_scale, void *out, float *lse,
                                   void *ws, size_t ws_bytes, cudaStream_t stream) {
    const KvMap map{nullptr, block_table, seq_len, max_blocks, page_size};
    return sparse_mla_launch_map<true, false>(q, kv, kv_rows, map, 1.0f, q_req, token_ids, Q, B,
                                              Hm, W, kv_lora, rope_dim, sm_scale, out, lse, ws,
                                              ws_bytes, stream);
}

inline int sparse_mla_launch_paged_fp8(const void *q, const void *kv8, float kv_scale,
                                       int64_t kv_rows, const int32_t *block_table, int max_blocks,
                                       int page_size, const int32_t *seq_len, const int32_t *q_req,
                                       const int32_t *token_ids, int Q, int B, int Hm, int W,
                                       int kv_lora, int rope_dim, float sm_scale, void *out,
                                       float *lse, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const KvMap map{nullptr, block_table, seq_len, max_blocks, page_size};
    return sparse_mla_launch_map<true, true>(q, kv8, kv_rows, map, kv_scale, q_req, token_ids, Q,
                                             B, Hm, W, kv_lora, rope_dim, sm_scale, out, lse, ws,
                                             ws_bytes, stream);
}

}  // namespace dsa
