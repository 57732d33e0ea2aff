// a2+a3. kpool_compress with the k_norm LayerNorm fused in
// ("spark_model/layers/glm5next_dsa/mod.rs": "Shape of the pipeline" first
// arrow; traps 1-4; KERNEL_MAX_KPOOL).
//
// B200 design. The op streams the k and gate caches once (256 B per token row
// each) and writes one 256 B key per pool: it is HBM-bound, so the kernel is a
// TMA-fed stream with all arithmetic in registers:
//   * a persistent CTA (one an SM) owns a range of tiles; a tile is TP
//     consecutive pools of one request, i.e. up to 128 contiguous token rows
//     of k and of gate. Where the requests' pool counts differ by more than a
//     tile (and there are at most 2048 requests, 1152 above kpool 4) the CTAs
//     first find every request's first valid token and split the tiles that
//     hold pools evenly among themselves (pool slots past a request's span are
//     then written apart, without a trip through the pipeline); otherwise each
//     takes a contiguous range of every request's tile grid;
//   * a producer warp moves each tile with 1-D bulk copies (cp.async.bulk) into
//     a shared-memory ring -- the k rows, the gate rows and the 16-byte-aligned
//     span of validity bytes covering them -- all completing on one mbarrier,
//     so no consumer waits on a global load;
//   * statistics warps take each landed tile's LayerNorm statistics, one thread
//     a token row, and hand them to the pool warps by mbarrier;
//   * a half-warp of a pool warp handles one pool; lane l owns channels
//     8l..8l+7 (one 16-byte vector of each row); the per-channel softmax over
//     the kpool slots runs in one pass in packed fp32x2, shifted by slot 0's
//     logit (exp2 with log2(e) folded into the logits; a second pass shifted by
//     the slots' maximum where a weight overflows);
//   * the first valid token of a request is found from its validity bytes
//     (16-byte loads, a ballot scan).
#pragma once

#include "common.cuh"

namespace dsa {

// Geometry per kpool. kpool <= 4: 12 pool warps (a half-warp a pool, so 24 pools,
// 96 token rows at kpool 4, a tile) and 3 statistics warps (a thread a row);
// with the producer four warps per scheduler, so up to 128 registers a thread.
// Larger pools (more live registers): 6 pool warps (12 pools) and 2 statistics
// warps. A stage holds the tile's k rows then its gate rows; three or four
// stages in the ring.
template <int KP> struct CmpCfg {
    static constexpr int kPoolWarps = KP <= 4 ? 12 : 6;         // a half-warp per pool
    static constexpr int kStatWarps = KP <= 4 ? 3 : 2;          // LayerNorm statistics, a tile ahead
    static constexpr int kWarps = kPoolWarps + kStatWarps;      // consumer warps
    static constexpr int kConsumers = kWarps * 32;
    static constexpr int kThreads = kConsumers + 32;            // + 1 producer warp
    static constexpr int kTP = 2 * kPoolWarps;                  // pools per tile
    static constexpr int kTileTokens = kTP * KP;
    static constexpr int kStages = 4;                           // most ring stages (3 or 4 run)
    static constexpr int kStageBytes = 2 * kTileTokens * 128 * 2;
};
constexpr int kD = DSA_INDEX_DIM;   // 128 channels
// Requests the balanced partition handles (4 int32 a request in shared memory);
// each thread of the CTA owns kCmpReqPerThread consecutive requests.
constexpr int kCmpReqPerThread = 4;
constexpr float kLog2e = 1.4426950408889634f;

// Bit i of the result is set iff byte i of w is nonzero: (low seven bits + 0x7F)
// carries into a byte's top bit iff those bits are not all zero, and the OR adds
// the byte's own top bit; no carry crosses into the next byte.
DSA_DEVINL uint32_t nonzero_bytes(uint32_t w) {
    const uint32_t h = (((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w) & 0x80808080u;
    return ((h >> 7) & 1u) | ((h >> 14) & 2u) | ((h >> 21) & 4u) | ((h >> 28) & 8u);
}

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

// One pool on a half-warp: lane l owns channels 8l..8l+7 of the kpool slot rows
// at krow/grow (shared memory), held as four fp32 pairs so the arithmetic runs
// as packed fp32x2 (FFMA2 / FADD2 / FMUL2) instructions.
DSA_DEVINL void unpack8x2(const uint4 &v, float2 (&x)[4]) {
    x[0] = make_float2(bf16lo(v.x), bf16hi(v.x));
    x[1] = make_float2(bf16lo(v.y), bf16hi(v.y));
    x[2] = make_float2(bf16lo(v.z), bf16hi(v.z));
    x[3] = make_float2(bf16lo(v.w), bf16hi(v.w));
}

// Round a pair to bf16 (nearest even) and widen it back: the stored k_norm value.
DSA_DEVINL float2 round_bf16x2(float2 y) {
    const uint32_t p = pack_bf16x2(y.x, y.y);
    return make_float2(bf16lo(p), bf16hi(p));
}

// LayerNorm statistics of one token row on one thread. The row's sixteen
// 16-byte pieces are read in the order j ^ rot (j = 0..15, rot in 0..7), so the
// eight rows of consecutive rot that one shared-memory phase serves touch eight
// distinct bank groups. The moments are shifted by a sample of the row (the
// first element read, element 8 * rot), which lies within a few standard
// deviations of the mean, so their difference does not cancel. Sums are
// pairwise: within a piece, over four pieces, over the four groups. Returns
// (rstd, -mu * rstd). The order is fixed, so every kernel that calls it gets
// the same bits for the same row and rot.
DSA_DEVINL float2 row_stats(const __nv_bfloat16 *row, int rot, float eps) {
    float2 g1[4], g2[4];
    float x0 = 0.f;
    float2 nx0 = make_float2(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * q + i;
            v[i] = *reinterpret_cast<const uint4 *>(row + 8 * ((j & 8) | ((j & 7) ^ rot)));
        }
        if (q == 0) {
            x0 = bf16lo(v[0].x);
            nx0 = make_float2(-x0, -x0);
        }
        float2 p1[4], p2[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 x[4], d[4];
            unpack8x2(v[i], x);
#pragma unroll
            for (int c = 0; c < 4; ++c) d[c] = __fadd2_rn(x[c], nx0);
            p1[i] = __fadd2_rn(__fadd2_rn(d[0], d[1]), __fadd2_rn(d[2], d[3]));
            p2[i] = __fadd2_rn(__ffma2_rn(d[1], d[1], __fmul2_rn(d[0], d[0])),
                               __ffma2_rn(d[3], d[3], __fmul2_rn(d[2], d[2])));
        }
        g1[q] = __fadd2_rn(__fadd2_rn(p1[0], p1[1]), __fadd2_rn(p1[2], p1[3]));
        g2[q] = __fadd2_rn(__fadd2_rn(p2[0], p2[1]), __fadd2_rn(p2[2], p2[3]));
    }
    const float2 s1 = __fadd2_rn(__fadd2_rn(g1[0], g1[1]), __fadd2_rn(g1[2], g1[3]));
    const float2 s2 = __fadd2_rn(__fadd2_rn(g2[0], g2[1]), __fadd2_rn(g2[2], g2[3]));
    const float a1 = __fadd_rn(s1.x, s1.y), a2 = __fadd_rn(s2.x, s2.y);
    const float dm = __fmul_rn(a1, 1.0f / kD);
    const float var = fmaxf(fmaf(-dm, dm, __fmul_rn(a2, 1.0f / kD)), 0.f);
    const float mu = __fadd_rn(x0, dm);
    const float r = rsqrt_approx(__fadd_rn(var, eps));
    return make_float2(r, __fmul_rn(-mu, r));
}

// The statistics as the pool warps read them: (rstd, rstd, -mu * rstd,
// -mu * rstd), each value already paired for the packed fp32x2 arithmetic.
DSA_DEVINL float4 stat_pairs(float2 st) { return make_float4(st.x, st.x, st.y, st.y); }

// LayerNorm statistics of a tile's token rows, one thread a row, the row's
// read order keyed by its index in the tile (rot = index mod 8). Every thread
// of the statistics group calls it.
DSA_DEVINL void token_stats(const __nv_bfloat16 *sk, int ntok, float eps, float4 *stat, int ctid,
                            int nthreads) {
    for (int tok = ctid; tok < ntok; tok += nthreads)
        stat[tok] = stat_pairs(row_stats(sk + (size_t)tok * kD, tok & 7, eps));
}

// The pooled key chunk of lane l (channels 8l..8l+7) from the pool's kpool
// k rows and gate rows, with the rows' LayerNorm statistics st[s] (as paired
// by stat_pairs). s_ape holds
// ape * log2(e) laid out [slot][half][lane][4] so a half-warp's loads are
// contiguous. Returns the packed bf16 chunk (zero when the pool is invalid).
//
// One pass over the slots: the per-channel softmax is shifted by slot 0's
// logit instead of the slots' maximum (the same quotient), so each slot's
// exp2 weight and weighted k_norm row are formed as the row streams by, with
// no max pass and no logits held between passes; slot 0's own weight is
// exactly 1 (0 + 1, so a non-finite logit still carries through as NaN), with
// no exp2. A weight that overflows
// (logits more than 2^7 apart in log2 units) leaves a non-finite denominator;
// the warp then redoes its pools shifted by the slots' maximum.
template <int KP>
DSA_DEVINL uint4 compress_pool(const __nv_bfloat16 *krow, const __nv_bfloat16 *grow,
                               const float4 *st, const float *s_ape, const float2 (&lw)[4],
                               const float2 (&lb)[4], int l, bool ok) {
    const float2 log2e2 = make_float2(kLog2e, kLog2e);
    auto knorm = [&](int s, float2 (&kn)[4]) {
        const float4 rs = st[s];
        const float2 r2 = make_float2(rs.x, rs.y), n2 = make_float2(rs.z, rs.w);
        float2 x[4];
        unpack8x2(*reinterpret_cast<const uint4 *>(krow + s * kD), x);
#pragma unroll
        for (int c = 0; c < 4; ++c)
            kn[c] = round_bf16x2(__ffma2_rn(__ffma2_rn(x[c], r2, n2), lw[c], lb[c]));
    };
    auto logits = [&](int s, float2 (&lg)[4]) {
        float2 g[4];
        unpack8x2(*reinterpret_cast<const uint4 *>(grow + s * kD), g);
        const float4 a0 = *reinterpret_cast<const float4 *>(s_ape + (s * 2) * 64 + 4 * l);
        const float4 a1 = *reinterpret_cast<const float4 *>(s_ape + (s * 2 + 1) * 64 + 4 * l);
        lg[0] = __ffma2_rn(g[0], log2e2, make_float2(a0.x, a0.y));
        lg[1] = __ffma2_rn(g[1], log2e2, make_float2(a0.z, a0.w));
        lg[2] = __ffma2_rn(g[2], log2e2, make_float2(a1.x, a1.y));
        lg[3] = __ffma2_rn(g[3], log2e2, make_float2(a1.z, a1.w));
    };
    // slots a step (measured: unrolled fully the loop spills; one slot a step
    // is fastest at kpool <= 4, two above)
    constexpr int kSlotUnroll = KP <= 4 ? 1 : 2;
    float2 nsh[4], den[4], acc[4];
    {
        float2 lg[4];
        logits(0, lg);
#pragma unroll
        for (int c = 0; c < 4; ++c) nsh[c] = make_float2(-lg[c].x, -lg[c].y);
    }
#pragma unroll 1
    for (int attempt = 0;; ++attempt) {
        int s_first = 0;
        if (attempt == 0) {
            // slot 0 is the shift: its weight is (-nsh + nsh) + 1, i.e. 1, or NaN
            // where its logit is not finite, as exp2 of the difference would give
            float2 kn[4];
            knorm(0, kn);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 z0 = __ffma2_rn(nsh[c], make_float2(-1.f, -1.f), nsh[c]);
                den[c] = __fadd2_rn(z0, make_float2(1.f, 1.f));
                acc[c] = __ffma2_rn(den[c], kn[c], make_float2(0.f, 0.f));
            }
            s_first = 1;
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                den[c] = make_float2(0.f, 0.f);
                acc[c] = make_float2(0.f, 0.f);
            }
        }
#pragma unroll kSlotUnroll
        for (int s = s_first; s < KP; ++s) {
            float2 kn[4], lg[4];
            logits(s, lg);
            knorm(s, kn);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 z = __fadd2_rn(lg[c], nsh[c]);
                const float2 e = make_float2(ex2(z.x), ex2(z.y));
                den[c] = __fadd2_rn(den[c], e);
                acc[c] = __ffma2_rn(e, kn[c], acc[c]);
            }
        }
        float dsum = 0.f;     // finite iff every denominator is (a NaN or inf carries through)
#pragma unroll
        for (int c = 0; c < 4; ++c) dsum += den[c].x + den[c].y;
        if (attempt == 1 || !__any_sync(0xffffffffu, !(dsum < INFINITY))) break;
        // overflow somewhere in the warp: shift by the slots' maximum instead
        float2 mx[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) mx[c] = make_float2(-INFINITY, -INFINITY);
#pragma unroll
        for (int s = 0; s < KP; ++s) {
            float2 lg[4];
            logits(s, lg);
#pragma unroll
            for (int c = 0; c < 4; ++c) mx[c] = make_float2(fmaxf(mx[c].x, lg[c].x), fmaxf(mx[c].y, lg[c].y));
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) nsh[c] = make_float2(-mx[c].x, -mx[c].y);
    }
    uint4 o = make_uint4(0, 0, 0, 0);
    if (ok) {
        uint32_t w[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 inv = make_float2(rcp_approx(den[c].x), rcp_approx(den[c].y));
            const float2 v = __fmul2_rn(acc[c], inv);
            w[c] = pack_bf16x2(v.x, v.y);
        }
        o = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return o;
}

// A tile's description, read by every consumer thread as two 16-byte loads.
struct __align__(16) CmpMeta {
    int b, p0, p1, n_in, f, rs;
    int voff;             // validity byte of the tile's first row in the stage's byte window
    int pad;
};
DSA_DEVINL CmpMeta load_meta(const CmpMeta *m) {
    const int4 a = reinterpret_cast<const int4 *>(m)[0], c = reinterpret_cast<const int4 *>(m)[1];
    return CmpMeta{a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
}
// A stage's validity window: the 16-byte-aligned span of validity bytes that
// covers the tile's rows (at most 128 rows + 2 x 15 bytes of alignment).
constexpr int kCmpValidWindow = 160;

// Persistent kernel: CTA c owns a contiguous range of (request, pool-tile) work
// items. The last warp is the producer: it finds each request's first valid
// token (a warp ballot scan, cached across the request's tiles) and streams each
// tile's k rows, gate rows and validity bytes into the shared-memory ring. The
// other warps consume: a half-warp per pool.
template <int KP>
__global__ void __launch_bounds__(CmpCfg<KP>::kThreads, 1)
kpool_compress_kernel(const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ gate,
                      const uint8_t *__restrict__ valid, const int32_t *__restrict__ req_start,
                      int B, int max_pools, int tiles_per_req, int n_tiles, int balance_ok, int ns,
                      const float *__restrict__ ape, const __nv_bfloat16 *__restrict__ ln_w,
                      const __nv_bfloat16 *__restrict__ ln_b, float eps,
                      __nv_bfloat16 *__restrict__ pool_keys, int32_t *__restrict__ pool_idx,
                      uint8_t *__restrict__ pool_valid, int32_t *__restrict__ first_valid) {
    using C = CmpCfg<KP>;
    constexpr int TP = C::kTP;
    constexpr int kCmpStages = C::kStages;       // static arrays; ns stages are used
    constexpr int kCmpStageBytes = C::kStageBytes;
    constexpr int kCmpTileTokens = C::kTileTokens;
    constexpr int kCmpConsumers = C::kConsumers;
    constexpr int kCmpThreads = C::kThreads;
    extern __shared__ __align__(128) uint8_t cmp_smem[];
    __shared__ __align__(16) float s_ape[KP * kD];   // ape * log2(e), [slot][half][lane][4]
    __shared__ __align__(16) float4 s_stat[kCmpStages][kCmpTileTokens];   // stat_pairs
    __shared__ __align__(8) uint64_t full[kCmpStages], empty[kCmpStages], stat_full[kCmpStages];
    __shared__ CmpMeta meta[kCmpStages];
    __shared__ __align__(16) uint8_t s_valid[kCmpStages][kCmpValidWindow];
    __shared__ int s_np_lo, s_np_hi;      // fewest and most pools a request holds

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    // Unbalanced (many requests): contiguous ranges of every request's tile grid.
    int t_begin = (int)((long long)blockIdx.x * n_tiles / G);
    int t_end = (int)((long long)(blockIdx.x + 1) * n_tiles / G);
    // Balanced: per request its first valid token, and prefix sums over the requests
    // of the tiles holding pools in its span and of the pool slots past the span.
    int32_t *s_f = reinterpret_cast<int32_t *>(cmp_smem + ns * kCmpStageBytes);
    int32_t *s_pre = s_f + B;
    int32_t *s_epre = s_pre + (B + 1);
    int32_t *s_rs = s_epre + (B + 1);                // req_start, B + 1 entries

    if (tid == 0) {
        for (int s = 0; s < kCmpStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::kPoolWarps);
            mbar_init(&stat_full[s], C::kStatWarps);
        }
        fence_mbarrier_init();
        s_np_lo = INT_MAX;
        s_np_hi = 0;
    }
    // Step inputs the path never writes, all read in one round trip before the
    // wait on the preceding kernel: ape, the request offsets the partition
    // choice needs, and the producer's first request (contiguous ranges).
    constexpr int kApePerThread = (KP * kD + kCmpThreads - 1) / kCmpThreads;
    float apev[kApePerThread];
#pragma unroll
    for (int u = 0; u < kApePerThread; ++u) {
        const int i = tid + u * kCmpThreads;
        apev[u] = i < KP * kD ? ape[i] : 0.f;
    }
    // The balanced partition pays only where the requests' pool counts differ by
    // more than a tile; otherwise every request's tile grid holds about as many
    // real tiles and contiguous ranges of the grids are even already.
    int np_lo = INT_MAX, np_hi = 0;
    if (balance_ok) {
        for (int b = tid; b < B; b += kCmpThreads) {
            const int rs = req_start[b], re = req_start[b + 1];
            s_rs[b] = rs;
            if (b == B - 1) s_rs[B] = re;
            const int np = min(max_pools, max(0, re - rs) / KP);
            np_lo = min(np_lo, np);
            np_hi = max(np_hi, np);
        }
        np_lo = __reduce_min_sync(0xffffffffu, np_lo);
        np_hi = __reduce_max_sync(0xffffffffu, np_hi);
    }
    long long total = 0;
    int first_rs = 0, first_re = 0;
    if (warp == kCmpConsumers / 32 && t_begin < t_end) {
        const int b0 = t_begin / tiles_per_req;
        total = req_start[B];                       // rows of the validity array
        first_rs = req_start[b0];
        first_re = req_start[b0 + 1];
    }
    __syncthreads();                                // barrier and counter initialisation
#pragma unroll
    for (int u = 0; u < kApePerThread; ++u) {
        const int i = tid + u * kCmpThreads, sl = i / kD, c = i % kD;
        if (i < KP * kD) s_ape[(sl * 2 + ((c >> 2) & 1)) * 64 + 4 * (c >> 3) + (c & 3)] = apev[u] * kLog2e;
    }
    if (balance_ok && lane == 0) {
        atomicMin(&s_np_lo, np_lo);
        atomicMax(&s_np_hi, np_hi);
    }
    __syncthreads();                                // s_ape, s_rs and the pool-count range
    const bool balanced = balance_ok && s_np_hi - s_np_lo > TP;
    int g_lo = 0, g_hi = 0, e_lo = 0, e_hi = 0;
    if (balanced) {
        total = s_rs[B];
        // ---- each request's first valid token, a thread a request: the first 64
        // validity bytes from the request's first row (four 16-byte loads, a
        // nonzero-byte mask) settle almost every request; a warp scans the rest
#pragma unroll 1
        for (int b = tid; b < B; b += kCmpThreads) {
            const long long rs = s_rs[b], re = s_rs[b + 1];
            const long long c0 = rs & ~15ll;
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const long long c = c0 + 16 * j;
                v[j] = c < re && c + 16 <= total ? __ldg(reinterpret_cast<const uint4 *>(valid + c))
                                                 : make_uint4(0u, 0u, 0u, 0u);
            }
            uint64_t m = 0;             // bit i: validity byte c0 + i is nonzero
#pragma unroll
            for (int j = 0; j < 4; ++j)
                m |= (uint64_t)(nonzero_bytes(v[j].x) | nonzero_bytes(v[j].y) << 4 |
                                nonzero_bytes(v[j].z) << 8 | nonzero_bytes(v[j].w) << 12) << (16 * j);
            const long long wend = min(re, c0 + 64);      // the window's end within the request
            m &= ~0ull << (int)(rs - c0);
            if (wend - c0 < 64) m &= (1ull << (int)max(0ll, wend - c0)) - 1ull;
            const int T = (int)max(0ll, re - rs);
            const bool covered = wend <= (total & ~15ll);  // every chunk of the window was loaded
            int f;
            if (T == 0) f = 0;
            else if (!covered) f = -1;
            else if (m) f = (int)(c0 + __ffsll((long long)m) - 1 - rs);
            else f = wend == re ? T : -1;
            s_f[b] = f;
        }
        __syncthreads();
        for (int b = warp; b < B; b += kCmpThreads / 32) {
            if (s_f[b] >= 0) continue;                     // warp-uniform
            const int rs = s_rs[b];
            const int T = max(0, s_rs[b + 1] - rs);
            const int f = first_valid_scan(valid, rs, T);
            if (lane == 0) s_f[b] = f;
        }
        __syncthreads();
        // ---- per request: tiles of pools in its span, pool slots past it; prefix
        // sums (thread t owns requests kCmpReqPerThread t, ... + kCmpReqPerThread)
        const int rb0 = tid * kCmpReqPerThread;
        int tl[kCmpReqPerThread], em[kCmpReqPerThread], st = 0, se = 0;
#pragma unroll
        for (int u = 0; u < kCmpReqPerThread; ++u) {
            const int b = rb0 + u;
            tl[u] = em[u] = 0;
            if (b < B) {
                const int T = max(0, s_rs[b + 1] - s_rs[b]);
                const int n_span = max(0, min(max_pools, (T - s_f[b]) / KP));
                tl[u] = (n_span + TP - 1) / TP;
                em[u] = max_pools - n_span;
            }
            st += tl[u];
            se += em[u];
        }
        __shared__ int2 s_w2[kCmpThreads / 32];
        int x = st, y = se;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, x, off), c = __shfl_up_sync(0xffffffffu, y, off);
            if (lane >= off) { x += a; y += c; }
        }
        if (lane == 31) s_w2[warp] = make_int2(x, y);
        __syncthreads();
        int bx = 0, by = 0, R = 0, E = 0;
        for (int w2 = 0; w2 < kCmpThreads / 32; ++w2) {
            const int2 v = s_w2[w2];
            if (w2 < warp) { bx += v.x; by += v.y; }
            R += v.x;
            E += v.y;
        }
        int px = bx + x - st, py = by + y - se;
#pragma unroll
        for (int u = 0; u < kCmpReqPerThread; ++u) {
            const int b = rb0 + u;
            if (b < B) {
                s_pre[b] = px;
                s_epre[b] = py;
                if (b == B - 1) { s_pre[B] = px + tl[u]; s_epre[B] = py + em[u]; }
            }
            px += tl[u];
            py += em[u];
        }
        __syncthreads();
        g_lo = (int)((long long)blockIdx.x * R / G);
        g_hi = (int)((long long)(blockIdx.x + 1) * R / G);
        e_lo = (int)((long long)blockIdx.x * E / G);
        e_hi = (int)((long long)(blockIdx.x + 1) * E / G);
        t_begin = 0;
        t_end = g_hi - g_lo;                       // this CTA's tiles, in order
    }
    // k, gate and the validity bytes are step inputs too: the producer streams
    // tiles before the wait on the preceding kernel; a thread waits for it before
    // its first write to an output (the pool warps, and the producer's stores of
    // the slots past the spans).
    pdl_launch_dependents();

    if (warp == kCmpConsumers / 32) {
        // ---------------------------------------------------------------- producer warp
        int cur_b = -1, cur_f = 0, cur_rs = 0, cur_T = 0;
        // balanced: the first request holding real tile g_lo (s_pre is non-decreasing)
        int bb = 0;
        if (balanced) {
            int lo = 0, hi = B - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_pre[mid] <= g_lo) lo = mid; else hi = mid - 1;
            }
            bb = lo;
        }
        // ring position: stage s of pass ph (tile i uses stage i mod ns in pass i / ns)
        for (int t = t_begin, i = 0, s = 0, ph = 0; t < t_end;
             ++t, ++i, ph ^= (s + 1 == ns), s = (s + 1 == ns) ? 0 : s + 1) {
            bool ok = true;
            if (i >= ns) ok = mbar_wait(&empty[s], ph ^ 1);
            if (!__all_sync(0xffffffffu, ok)) break;
            int b, j;
            if (balanced) {
                const int g = g_lo + t;
                while (s_pre[bb + 1] <= g) ++bb;
                b = bb;
                j = g - s_pre[bb];
            } else {
                b = t / tiles_per_req;
                j = t - b * tiles_per_req;
            }
            if (b != cur_b) {
                const bool first = i == 0 && !balanced;
                cur_rs = balanced ? s_rs[b] : first ? first_rs : req_start[b];
                cur_T = max(0, (balanced ? s_rs[b + 1] : first ? first_re : req_start[b + 1]) - cur_rs);
                cur_f = balanced ? s_f[b] : first_valid_scan(valid, cur_rs, cur_T);
                cur_b = b;
            }
            const int p0 = j * TP;
            const int n_span = min(max_pools, (cur_T - cur_f) / KP);
            // balanced tiles end at the span (the slots past it are written apart)
            const int p1 = balanced ? min(p0 + TP, n_span) : min(p0 + TP, max_pools);
            const int n_in = max(0, min(p1, n_span) - p0);
            // The tile's rows of k and gate, and the 16-byte-aligned span of
            // validity bytes covering them, arrive together by bulk copy; the
            // span stops at the last whole 16-byte chunk of the array and any
            // rows past that (the array's last few bytes) are read by plain loads.
            const long long row0 = (long long)cur_rs + cur_f + (long long)p0 * KP;
            const long long row1 = row0 + (long long)n_in * KP;
            const long long vs = row0 & ~15ll;
            const long long ve = min((row1 + 15) & ~15ll, max(vs, total & ~15ll));
            const uint32_t vbytes = n_in > 0 ? (uint32_t)(ve - vs) : 0u;
            if (n_in > 0)
                for (long long r = max(ve, row0) + lane; r < row1; r += 32)
                    s_valid[s][r - vs] = valid[r];
            __syncwarp();
            if (lane == 0) {
                meta[s] = CmpMeta{b, p0, p1, n_in, cur_f, cur_rs, (int)(row0 - vs), 0};
                if (n_in > 0) {
                    const uint32_t bytes = (uint32_t)(n_in * KP * kD * 2);
                    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(cmp_smem + s * kCmpStageBytes);
                    mbar_arrive_expect_tx(&full[s], 2 * bytes + vbytes);
                    bulk_g2s(sk, k + row0 * kD, bytes, &full[s]);
                    bulk_g2s(sk + kCmpTileTokens * kD, gate + row0 * kD, bytes, &full[s]);
                    if (vbytes > 0) bulk_g2s(&s_valid[s][0], valid + vs, vbytes, &full[s]);
                } else {
                    mbar_arrive(&full[s]);
                }
            }
            __syncwarp();
        }
        pdl_wait();
        if (balanced) {
            // pool slots past each request's span: index -1, invalid (the key rows
            // there are not written); this CTA's share of them, request by request
            int b = 0;
            {
                int lo = 0, hi = B - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_epre[mid] <= e_lo) lo = mid; else hi = mid - 1;
                }
                b = lo;
            }
            for (int e = e_lo; e < e_hi && b < B;) {
                while (b < B && s_epre[b + 1] <= e) ++b;
                if (b >= B) break;
                const int first_p = max_pools - (s_epre[b + 1] - s_epre[b]);    // = n_span
                const int p_a = first_p + (e - s_epre[b]);
                const int cnt = min(e_hi, s_epre[b + 1]) - e;
                const size_t pb = (size_t)b * max_pools;
                for (int x = lane; x < cnt * KP; x += 32) pool_idx[(pb + p_a) * KP + x] = -1;
                for (int x = lane; x < cnt; x += 32) pool_valid[pb + p_a + x] = 0;
                e += cnt;
            }
        }
        return;
    }

    // -------------------------------------------------------------------- consumer warps
    // Warp-specialised: kStatWarps warps take each tile's LayerNorm statistics as
    // soon as it lands (a tile ahead of the pools), kPoolWarps warps compress its
    // pools once the statistics are in; mbarriers hand the tiles over, so no
    // barrier spans all consumers.
    if (warp >= C::kPoolWarps) {
        const int stid = tid - C::kPoolWarps * 32;
        for (int t = t_begin, s = 0, ph = 0; t < t_end; ++t, ph ^= (s + 1 == ns), s = (s + 1 == ns) ? 0 : s + 1) {
            const bool ok = mbar_wait(&full[s], ph);
            if (!__all_sync(0xffffffffu, ok)) break;
            const __nv_bfloat16 *sk = reinterpret_cast<const __nv_bfloat16 *>(cmp_smem + s * kCmpStageBytes);
            token_stats(sk, meta[s].n_in * KP, eps, &s_stat[s][0], stid, C::kStatWarps * 32);
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_full[s]);
        }
        return;
    }
    const int hw = tid >> 4;     // half-warp: one pool at a time
    const int l = tid & 15;      // channels 8l .. 8l+7
    float2 lw[4], lb[4];
    unpack8x2(ldg_nc_v4(ln_w + 8 * l), lw);
    unpack8x2(ldg_nc_v4(ln_b + 8 * l), lb);
    constexpr int kPoolThreads = C::kPoolWarps * 32;
    pdl_wait();
    if (balanced) {
        // first_valid: this CTA's share of the requests
        const int b_lo = (int)((long long)blockIdx.x * B / G), b_hi = (int)((long long)(blockIdx.x + 1) * B / G);
        for (int b = b_lo + tid; b < b_hi; b += kPoolThreads) first_valid[b] = s_f[b];
    }
    for (int t = t_begin, s = 0, ph = 0; t < t_end; ++t, ph ^= (s + 1 == ns), s = (s + 1 == ns) ? 0 : s + 1) {
        const bool ok = mbar_wait(&stat_full[s], ph);
        if (!__all_sync(0xffffffffu, ok)) break;
        const CmpMeta m = load_meta(&meta[s]);
        const __nv_bfloat16 *sk = reinterpret_cast<const __nv_bfloat16 *>(cmp_smem + s * kCmpStageBytes);
        const __nv_bfloat16 *sg = sk + kCmpTileTokens * kD;
        const size_t pool_base = (size_t)m.b * max_pools;
        if (!balanced && m.p0 == 0 && tid == 0) first_valid[m.b] = m.f;

        // Pools of this tile past the request's span: no key, index -1, invalid.
        for (int x = m.n_in * KP + tid; x < (m.p1 - m.p0) * KP; x += kPoolThreads)
            pool_idx[(pool_base + m.p0) * KP + x] = -1;
        for (int x = m.n_in + tid; x < m.p1 - m.p0; x += kPoolThreads)
            pool_valid[pool_base + m.p0 + x] = 0;

        // Warp-uniform loop: the two half-warps of a warp take pools ii and ii+1;
        // a half-warp past the tile computes on a loaded row and stores nothing.
        for (int ii = 2 * warp; ii < m.n_in; ii += kPoolThreads / 16) {
            const bool active = ii + (hw & 1) < m.n_in;
            const int pi = active ? ii + (hw & 1) : ii;
            const int p = m.p0 + pi;
            // the pool is valid iff its KP validity bytes are all nonzero: lane l < KP
            // of the half-warp tests byte l, one ballot gathers them
            const bool vb = l >= KP || s_valid[s][m.voff + pi * KP + l] != 0;
            const uint32_t vbits = (__ballot_sync(0xffffffffu, vb) >> (16 * (hw & 1))) & 0xFFFFu;
            const bool okp = vbits == 0xFFFFu;
            const uint4 o = compress_pool<KP>(sk + (size_t)pi * KP * kD + 8 * l,
                                              sg + (size_t)pi * KP * kD + 8 * l,
                                              &s_stat[s][pi * KP], s_ape, lw, lb, l, okp);
            if (!active) continue;
            *reinterpret_cast<uint4 *>(pool_keys + (pool_base + p) * kD + 8 * l) = o;
            if (l < KP) pool_idx[(pool_base + p) * KP + l] = okp ? m.f + p * KP + l : -1;
            if (l == 0) pool_valid[pool_base + p] = okp ? 1 : 0;
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
    using C = CmpCfg<KP>;
    constexpr int TP = C::kTP;
    // Up to kCmpReqPerThread requests a thread, the CTA may split the tiles that
    // hold pools evenly (balanced, where request lengths differ); beyond, always
    // contiguous ranges of every request's tile grid.
    const int balance_ok = B <= kCmpReqPerThread * C::kThreads ? 1 : 0;
    // Ring depth: each stage turns over in its load latency plus the consumers'
    // time on it, so a fourth stage (more bytes in flight, less of the ring idle
    // while a tile is worked on) where the block's shared memory has room for it
    // next to the balanced partition's per-request arrays.
    const void *f = reinterpret_cast<const void *>(kpool_compress_kernel<KP>);
    cudaFuncAttributes fa;
    int dev = 0, optin = 0;
    if (cudaFuncGetAttributes(&fa, f) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return DSA_ERR_CUDA;
    const int extra = balance_ok ? 4 * (4 * B + 3) : 0;
    int ns = C::kStages;
    while (ns > 3 && (long long)fa.sharedSizeBytes + ns * C::kStageBytes + extra > optin) --ns;
    const int smem = ns * C::kStageBytes + extra;
    if (!ensure_smem_attr(f, smem)) return DSA_ERR_CUDA;
    const int tiles_per_req = max(1, ceil_div(max_pools, TP));
    const long long n_tiles = (long long)tiles_per_req * B;
    if (n_tiles > (1ll << 30)) return DSA_ERR_UNSUPPORTED;
    const int grid = (int)std::min<long long>(n_tiles, sm_count());
    if (launch_pdl(kpool_compress_kernel<KP>, dim3(grid), dim3(C::kThreads), smem, stream, k, gate,
                   valid, req_start, B, max_pools, tiles_per_req, (int)n_tiles, balance_ok, ns, ape, ln_w,
                   ln_b, eps, keys, idx, pv, fv) != cudaSuccess)
        return DSA_ERR_CUDA;
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
