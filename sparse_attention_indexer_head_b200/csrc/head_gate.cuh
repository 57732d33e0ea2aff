// a1. Indexer head gate: out[M,N] = hidden[M,K] @ w[K,N], fp32
// ("feat(glm53): indexer fp32 head-gate split-K", PR description: the fp32
// [M,4096]x[4096,16] product that cuBLAS served with two CTAs).
//
// B200 design: K is split across a thread-block cluster of 8 CTAs; each CTA
// owns 16 rows and a K/8 slice. A CTA stages its slice of w in shared memory,
// 16 lanes per row sweep the slice with 16-byte loads of hidden, the 16
// partial sums per row are folded with half-warp shuffles, and the 8 CTAs'
// partials are summed through distributed shared memory in rank order. One
// launch, no atomics, no workspace, deterministic.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kGateRows = 16;      // rows of hidden per CTA
constexpr int kGateSplit = 8;      // CTAs per cluster (K split)
constexpr int kGateThreads = 256;  // 16 rows x 16 k-lanes
constexpr int kGateMaxN = 16;
constexpr int kGateMaxSlice = 512; // K-slice rows staged per pass

__global__ void __cluster_dims__(1, kGateSplit, 1) __launch_bounds__(kGateThreads)
head_gate_kernel(const float *__restrict__ hidden, const float *__restrict__ w,
                 float *__restrict__ out, int M, int K, int N) {
    __shared__ __align__(16) float ws[kGateMaxSlice * kGateMaxN];  // w slice, zero-padded to 16 cols
    __shared__ float part[kGateRows * kGateMaxN];                   // this CTA's partial sums

    const int tid = threadIdx.x;
    const int j = tid & 15;            // k-lane within the row
    const int r = tid >> 4;            // row within the CTA
    const int rank = blockIdx.y;       // == cluster CTA rank (cluster dims 1 x 8)
    const int m = blockIdx.x * kGateRows + r;

    // This CTA's K range, in multiples of 4 (16-byte vectors of hidden).
    const int k4 = K >> 2;
    const int per = (k4 + kGateSplit - 1) / kGateSplit;
    const int kb = min(K, rank * per * 4);
    const int ke = min(K, (rank + 1) * per * 4);

    float acc[kGateMaxN];
#pragma unroll
    for (int n = 0; n < kGateMaxN; ++n) acc[n] = 0.f;

    // Each pass stages up to 512 rows of w and this thread's 8 vectors of hidden.
    // All loads of a pass are issued before the first use, so one memory
    // latency covers the pass instead of one per load.
    const bool w_vec = N == kGateMaxN && aligned16(w);
    for (int k0 = kb; k0 < ke; k0 += kGateMaxSlice) {
        const int len = min(kGateMaxSlice, ke - k0);
        float4 hv[kGateMaxSlice / 64];
#pragma unroll
        for (int u = 0; u < kGateMaxSlice / 64; ++u) {
            const int kk = 4 * j + 64 * u;
            hv[u] = (m < M && kk < len)
                        ? __ldg(reinterpret_cast<const float4 *>(hidden + (size_t)m * K + k0 + kk))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();   // the previous pass is done with ws
        if (w_vec) {
            const float4 *src = reinterpret_cast<const float4 *>(w + (size_t)k0 * kGateMaxN);
            float4 tmp[kGateMaxSlice * kGateMaxN / 4 / kGateThreads];
#pragma unroll
            for (int u = 0; u < kGateMaxSlice * kGateMaxN / 4 / kGateThreads; ++u) {
                const int i = tid + u * kGateThreads;
                tmp[u] = i < len * 4 ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < kGateMaxSlice * kGateMaxN / 4 / kGateThreads; ++u) {
                const int i = tid + u * kGateThreads;
                if (i < len * 4) reinterpret_cast<float4 *>(ws)[i] = tmp[u];
            }
        } else {
            for (int i0 = 0; i0 < len * kGateMaxN; i0 += 8 * kGateThreads) {
                float tmp[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + tid + u * kGateThreads;
                    const int kk = i / kGateMaxN, n = i % kGateMaxN;
                    tmp[u] = (i < len * kGateMaxN && n < N) ? __ldg(w + (size_t)(k0 + kk) * N + n)
                                                            : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + tid + u * kGateThreads;
                    if (i < len * kGateMaxN) ws[i] = tmp[u];
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kGateMaxSlice / 64; ++u) {
            const int kk = 4 * j + 64 * u;
            if (kk >= len) break;
            const float hvu[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 *wr = reinterpret_cast<const float4 *>(ws + (kk + e) * kGateMaxN);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 wv = wr[q];
                    acc[4 * q + 0] = fmaf(hvu[e], wv.x, acc[4 * q + 0]);
                    acc[4 * q + 1] = fmaf(hvu[e], wv.y, acc[4 * q + 1]);
                    acc[4 * q + 2] = fmaf(hvu[e], wv.z, acc[4 * q + 2]);
                    acc[4 * q + 3] = fmaf(hvu[e], wv.w, acc[4 * q + 3]);
                }
            }
        }
    }

    // Fold the 16 k-lanes of each row (a fixed butterfly order).
#pragma unroll
    for (int off = 8; off > 0; off >>= 1)
#pragma unroll
        for (int n = 0; n < kGateMaxN; ++n) acc[n] += __shfl_xor_sync(0xffffffffu, acc[n], off);
    if (j == 0) {
#pragma unroll
        for (int n = 0; n < kGateMaxN; ++n) part[r * kGateMaxN + n] = acc[n];
    }

    // Cluster-wide: every CTA's partials visible, then rank c sums rows c and
    // c + 8 over the 8 ranks in rank order.
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
    if (tid < 2 * kGateMaxN) {
        const int rr = rank + (tid >= kGateMaxN ? kGateSplit : 0);
        const int n = tid % kGateMaxN;
        const int mm = blockIdx.x * kGateRows + rr;
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
        if (mm < M && n < N) out[(size_t)mm * N + n] = s;
    }
    // Keep this CTA's shared memory alive until every rank has read it.
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

inline int head_gate_launch(const float *hidden, const float *w, float *out, int M, int K, int N,
                            cudaStream_t stream) {
    if (M < 0 || K <= 0 || N <= 0) return DSA_ERR_INVALID_ARG;
    if (N > kGateMaxN || (K & 3) != 0) return DSA_ERR_UNSUPPORTED;
    if (M == 0) return DSA_OK;
    if (!hidden || !w || !out) return DSA_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(w, 4) || !aligned(out, 4)) return DSA_ERR_ALIGNMENT;
    const int row_blocks = ceil_div(M, kGateRows);
    if (row_blocks > 65535 * 16) return DSA_ERR_UNSUPPORTED;
    dim3 grid(row_blocks, kGateSplit);
    head_gate_kernel<<<grid, kGateThreads, 0, stream>>>(hidden, w, out, M, K, N);
    return launch_status();
}

}  // namespace dsa
