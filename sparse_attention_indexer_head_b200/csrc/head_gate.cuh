// a1. Indexer head gate: out[M,N] = hidden[M,K] @ w[K,N], fp32
// ("feat(glm53): indexer fp32 head-gate split-K", PR description: the fp32
// [M,4096]x[4096,16] product that cuBLAS served with two CTAs).
//
// B200 design: K is split across a thread-block cluster of 8 CTAs; each CTA
// owns 16 rows and a K/8 slice, staged in shared memory with all global loads
// in flight at once. 16 warps sweep the slice with a bank-conflict-free lane
// mapping, their partials are folded in a fixed order, and the 8 CTAs'
// partials are summed through distributed shared memory in rank order. One
// launch, no atomics, no workspace, deterministic.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kGateRows = 16;      // rows of hidden per CTA
constexpr int kGateSplit = 8;      // CTAs per cluster (K split)
constexpr int kGateThreads = 512;  // 16 warps
constexpr int kGateWarps = kGateThreads / 32;
constexpr int kGateMaxN = 16;
constexpr int kGateSlice = 512;    // k rows staged per pass
constexpr int kGateHStride = kGateSlice + 1;   // padded hidden rows: conflict-free column reads
constexpr int kGateSmem = (kGateRows * kGateHStride + kGateSlice * kGateMaxN +
                           kGateWarps * kGateRows * kGateMaxN + kGateRows * kGateMaxN) * 4;

// Lane mapping inside a warp: lane = 2*m + half, so a lane owns row m and
// columns 8*half .. 8*half+7. For each k the 16 rows read 16 different
// hidden values (padded row stride: distinct banks) and the 32 lanes read only
// two distinct 32-byte pieces of the w row (broadcast), so shared memory is
// conflict-free. Warp w covers k rows w, w+16, w+32, ... of the slice.
__global__ void __cluster_dims__(1, kGateSplit, 1) __launch_bounds__(kGateThreads)
head_gate_kernel(const float *__restrict__ hidden, const float *__restrict__ w,
                 float *__restrict__ out, int M, int K, int N) {
    extern __shared__ __align__(16) float gate_smem[];
    float *hs = gate_smem;                                   // [16][513]
    float *ws = hs + kGateRows * kGateHStride;               // [512][16], zero-padded columns
    float *red = ws + kGateSlice * kGateMaxN;                // [16 warps][16][16]
    float *part = red + kGateWarps * kGateRows * kGateMaxN;  // [16][16] this CTA's partial

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = blockIdx.y;       // == cluster CTA rank (cluster dims 1 x 8)
    const int m0 = blockIdx.x * kGateRows;
    const int rows = min(kGateRows, M - m0);

    const int k4 = K >> 2;
    const int per = (k4 + kGateSplit - 1) / kGateSplit;
    const int kb = min(K, rank * per * 4);
    const int ke = min(K, (rank + 1) * per * 4);

    const int m = lane >> 1, n0 = (lane & 1) * 8;
    float acc[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) acc[n] = 0.f;

    const bool w_vec = N == kGateMaxN && aligned16(w);
    for (int k0 = kb; k0 < ke; k0 += kGateSlice) {
        const int len = min(kGateSlice, ke - k0);
        // -- stage: every load of the pass is issued before the first store
        constexpr int HV = kGateRows * kGateSlice / 4 / kGateThreads;    // 4 float4 of hidden
        constexpr int WV = kGateSlice * kGateMaxN / 4 / kGateThreads;    // 4 float4 of w
        float4 hv[HV], wv[WV];
#pragma unroll
        for (int u = 0; u < HV; ++u) {
            const int i = tid + u * kGateThreads;          // i = r * 128 + c4
            const int r = i >> 7, c4 = (i & 127) * 4;
            hv[u] = (r < rows && c4 < len)
                        ? __ldg(reinterpret_cast<const float4 *>(hidden + (size_t)(m0 + r) * K + k0 + c4))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (w_vec) {
            const float4 *src = reinterpret_cast<const float4 *>(w + (size_t)k0 * kGateMaxN);
#pragma unroll
            for (int u = 0; u < WV; ++u) {
                const int i = tid + u * kGateThreads;
                wv[u] = i < len * 4 ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
#pragma unroll
            for (int u = 0; u < WV; ++u) {
                const int i = tid + u * kGateThreads;      // float4 index: row i/4, cols 4(i%4)..
                const int kk = i >> 2, c = (i & 3) * 4;
                float t[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    t[e] = (kk < len && c + e < N) ? __ldg(w + (size_t)(k0 + kk) * N + c + e) : 0.f;
                wv[u] = make_float4(t[0], t[1], t[2], t[3]);
            }
        }
        __syncthreads();   // the previous pass is done with hs / ws
#pragma unroll
        for (int u = 0; u < HV; ++u) {
            const int i = tid + u * kGateThreads;
            const int r = i >> 7, c4 = (i & 127) * 4;
            float *d = hs + r * kGateHStride + c4;
            d[0] = hv[u].x; d[1] = hv[u].y; d[2] = hv[u].z; d[3] = hv[u].w;
        }
#pragma unroll
        for (int u = 0; u < WV; ++u)
            reinterpret_cast<float4 *>(ws)[tid + u * kGateThreads] = wv[u];
        __syncthreads();
        // -- 8 independent accumulators per lane; 32 k rows per warp per pass
        const float *hrow = hs + m * kGateHStride;
#pragma unroll 4
        for (int kk = warp; kk < len; kk += kGateWarps) {
            const float h = hrow[kk];
            const float4 wa = *reinterpret_cast<const float4 *>(ws + kk * kGateMaxN + n0);
            const float4 wb = *reinterpret_cast<const float4 *>(ws + kk * kGateMaxN + n0 + 4);
            acc[0] = fmaf(h, wa.x, acc[0]); acc[1] = fmaf(h, wa.y, acc[1]);
            acc[2] = fmaf(h, wa.z, acc[2]); acc[3] = fmaf(h, wa.w, acc[3]);
            acc[4] = fmaf(h, wb.x, acc[4]); acc[5] = fmaf(h, wb.y, acc[5]);
            acc[6] = fmaf(h, wb.z, acc[6]); acc[7] = fmaf(h, wb.w, acc[7]);
        }
    }

    // Loads and arithmetic above touch only the step's inputs; from here on the
    // CTA writes shared state and then the output, after the predecessor grid.
    pdl_wait();
    pdl_launch_dependents();

    // Fold the 16 warps (fixed order), then the 8 cluster ranks (rank order).
#pragma unroll
    for (int n = 0; n < 8; ++n) red[(warp * kGateRows + m) * kGateMaxN + n0 + n] = acc[n];
    __syncthreads();
    if (tid < kGateRows * kGateMaxN) {
        float sum = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kGateWarps; ++w2) sum += red[w2 * kGateRows * kGateMaxN + tid];
        part[tid] = sum;
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
    if (tid < 2 * kGateMaxN) {
        const int rr = rank + (tid >= kGateMaxN ? kGateSplit : 0);
        const int n = tid % kGateMaxN;
        const uint32_t local = smem_u32(&part[rr * kGateMaxN + n]);
        float v[kGateSplit];
#pragma unroll
        for (int c = 0; c < kGateSplit; ++c) {   // all remote loads in flight at once
            uint32_t remote;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(c));
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v[c]) : "r"(remote) : "memory");
        }
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < kGateSplit; ++c) s += v[c];
        if (rr < rows && n < N) out[(size_t)(m0 + rr) * N + n] = s;
    }
    // Keep this CTA's shared memory alive until every rank has read it.
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// Many rows (chunked prefill): the row blocks alone fill the device, so a CTA
// takes its 16 rows over the whole of K, with no cluster: the same staging,
// lane mapping and fixed-order warp fold as above, the next slice's loads in
// flight (registers) while the current slice is summed. Deterministic; the
// order of the sum differs from the split kernel's only in where the K slices
// meet.
__global__ void __launch_bounds__(kGateThreads, 1)
head_gate_rows_kernel(const float *__restrict__ hidden, const float *__restrict__ w,
                      float *__restrict__ out, int M, int K, int N) {
    extern __shared__ __align__(16) float gate_smem[];
    float *hs = gate_smem;                                   // [16][513]
    float *ws = hs + kGateRows * kGateHStride;               // [512][16], zero-padded columns
    float *red = ws + kGateSlice * kGateMaxN;                // [16 warps][16][16]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * kGateRows;
    const int rows = min(kGateRows, M - m0);
    const int m = lane >> 1, n0 = (lane & 1) * 8;
    const bool w_vec = N == kGateMaxN && aligned16(w);
    constexpr int HV = kGateRows * kGateSlice / 4 / kGateThreads;    // 4 float4 of hidden
    constexpr int WV = kGateSlice * kGateMaxN / 4 / kGateThreads;    // 4 float4 of w
    float4 hv[HV], wv[WV];
    auto load = [&](int k0) {
        const int len = min(kGateSlice, K - k0);
#pragma unroll
        for (int u = 0; u < HV; ++u) {
            const int i = tid + u * kGateThreads;          // i = r * 128 + c4
            const int r = i >> 7, c4 = (i & 127) * 4;
            hv[u] = (r < rows && c4 < len)
                        ? __ldg(reinterpret_cast<const float4 *>(hidden + (size_t)(m0 + r) * K + k0 + c4))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (w_vec) {
            const float4 *src = reinterpret_cast<const float4 *>(w + (size_t)k0 * kGateMaxN);
#pragma unroll
            for (int u = 0; u < WV; ++u) {
                const int i = tid + u * kGateThreads;
                wv[u] = i < len * 4 ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        } else {
#pragma unroll
            for (int u = 0; u < WV; ++u) {
                const int i = tid + u * kGateThreads;      // float4 index: row i/4, cols 4(i%4)..
                const int kk = i >> 2, c = (i & 3) * 4;
                float t[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    t[e] = (kk < len && c + e < N) ? __ldg(w + (size_t)(k0 + kk) * N + c + e) : 0.f;
                wv[u] = make_float4(t[0], t[1], t[2], t[3]);
            }
        }
    };
    float acc[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) acc[n] = 0.f;
    load(0);
    for (int k0 = 0; k0 < K; k0 += kGateSlice) {
        const int len = min(kGateSlice, K - k0);
        __syncthreads();   // the previous slice is done with hs / ws
#pragma unroll
        for (int u = 0; u < HV; ++u) {
            const int i = tid + u * kGateThreads;
            const int r = i >> 7, c4 = (i & 127) * 4;
            float *d = hs + r * kGateHStride + c4;
            d[0] = hv[u].x; d[1] = hv[u].y; d[2] = hv[u].z; d[3] = hv[u].w;
        }
#pragma unroll
        for (int u = 0; u < WV; ++u)
            reinterpret_cast<float4 *>(ws)[tid + u * kGateThreads] = wv[u];
        __syncthreads();
        if (k0 + kGateSlice < K) load(k0 + kGateSlice);   // in flight while this slice is summed
        const float *hrow = hs + m * kGateHStride;
#pragma unroll 4
        for (int kk = warp; kk < len; kk += kGateWarps) {
            const float h = hrow[kk];
            const float4 wa = *reinterpret_cast<const float4 *>(ws + kk * kGateMaxN + n0);
            const float4 wb = *reinterpret_cast<const float4 *>(ws + kk * kGateMaxN + n0 + 4);
            acc[0] = fmaf(h, wa.x, acc[0]); acc[1] = fmaf(h, wa.y, acc[1]);
            acc[2] = fmaf(h, wa.z, acc[2]); acc[3] = fmaf(h, wa.w, acc[3]);
            acc[4] = fmaf(h, wb.x, acc[4]); acc[5] = fmaf(h, wb.y, acc[5]);
            acc[6] = fmaf(h, wb.z, acc[6]); acc[7] = fmaf(h, wb.w, acc[7]);
        }
    }
    // Loads and arithmetic above touch only the step's inputs; the output is
    // written after the predecessor grid.
    pdl_wait();
    pdl_launch_dependents();
#pragma unroll
    for (int n = 0; n < 8; ++n) red[(warp * kGateRows + m) * kGateMaxN + n0 + n] = acc[n];
    __syncthreads();
    if (tid < kGateRows * kGateMaxN) {
        const int r = tid / kGateMaxN, n = tid % kGateMaxN;
        float sum = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kGateWarps; ++w2) sum += red[w2 * kGateRows * kGateMaxN + tid];
        if (r < rows && n < N) out[(size_t)(m0 + r) * N + n] = sum;
    }
}

// The size checks of head_gate_launch, on their own (no pointer is looked at).
inline int head_gate_shape_status(int M, int K, int N) {
    if (M < 0 || K <= 0 || N <= 0) return DSA_ERR_INVALID_ARG;
    if (N > kGateMaxN || (K & 3) != 0) return DSA_ERR_UNSUPPORTED;
    if (ceil_div(M, kGateRows) > 65535 * 16) return DSA_ERR_UNSUPPORTED;
    return DSA_OK;
}

inline int head_gate_launch(const float *hidden, const float *w, float *out, int M, int K, int N,
                            cudaStream_t stream) {
    const int st = head_gate_shape_status(M, K, N);
    if (st != DSA_OK) return st;
    if (M == 0) return DSA_OK;
    if (!hidden || !w || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(w, 4) || !aligned(out, 4)) return DSA_ERR_ALIGNMENT;
    const int row_blocks = ceil_div(M, kGateRows);
    if (row_blocks > 65535 * 16) return DSA_ERR_UNSUPPORTED;
    // Where the split clusters would take more than two waves of the device,
    // the row blocks alone fill it: one CTA a row block over the whole of K.
    if ((long long)row_blocks * kGateSplit > 2ll * sm_count()) {
        if (!ensure_smem_attr(reinterpret_cast<const void *>(head_gate_rows_kernel), kGateSmem))
            return DSA_ERR_CUDA;
        if (launch_pdl(head_gate_rows_kernel, dim3(row_blocks), dim3(kGateThreads), kGateSmem, stream,
                       hidden, w, out, M, K, N) != cudaSuccess)
            return DSA_ERR_CUDA;
        return launch_status();
    }
    dim3 grid(row_blocks, kGateSplit);
    if (!ensure_smem_attr(reinterpret_cast<const void *>(head_gate_kernel), kGateSmem))
        return DSA_ERR_CUDA;
    if (launch_pdl(head_gate_kernel, grid, dim3(kGateThreads), kGateSmem, stream, hidden, w, out,
                   M, K, N) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
