// f1. Indexer-cache store: a step's new tokens' k and gate rows and validity
// bytes into the per-request caches ("spark_model/layers/glm5next_dsa/mod.rs",
// Glm5NextDsaKernels::indexer_store: a staged indexer row placed at a
// device-side position and marked valid).
//
// One warp per new token: lanes 0-15 copy its 256-byte k row, lanes 16-31 its
// 256-byte gate row (one 16-byte vector each); lane 0 writes the validity byte.
// The destination row, req_start[b] + pos, is resolved on the device, so a
// captured graph replays over live positions; a token whose request or
// position is out of range is skipped.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kStoreWarps = 8;

__global__ void __launch_bounds__(kStoreWarps * 32)
indexer_store_kernel(const __nv_bfloat16 *__restrict__ k_new, const __nv_bfloat16 *__restrict__ gate_new,
                     const uint8_t *__restrict__ valid_new, const int32_t *__restrict__ tok_req,
                     const int32_t *__restrict__ tok_pos, int n, const int32_t *__restrict__ req_start,
                     int B, __nv_bfloat16 *__restrict__ k, __nv_bfloat16 *__restrict__ gate,
                     uint8_t *__restrict__ valid) {
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * kStoreWarps + (threadIdx.x >> 5);
    pdl_wait();
    pdl_launch_dependents();
    if (i >= n) return;
    const int b = tok_req[i], pos = tok_pos[i];
    if (b < 0 || b >= B) return;
    const int rs = req_start[b], T = req_start[b + 1] - rs;
    if (pos < 0 || pos >= T) return;
    const size_t row = (size_t)rs + pos;
    const int c = lane & 15;                         // 16-byte piece of the 256-byte row
    const __nv_bfloat16 *src = (lane < 16 ? k_new : gate_new) + (size_t)i * DSA_INDEX_DIM + 8 * c;
    __nv_bfloat16 *dst = (lane < 16 ? k : gate) + row * DSA_INDEX_DIM + 8 * c;
    *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
    if (lane == 0) valid[row] = valid_new ? (valid_new[i] != 0 ? 1 : 0) : 1;
}

inline int indexer_store_launch(const void *k_new, const void *gate_new, const uint8_t *valid_new,
                                const int32_t *tok_req, const int32_t *tok_pos, int n, int D,
                                const int32_t *req_start, int B, void *k, void *gate,
                                uint8_t *valid, cudaStream_t stream) {
    if (n < 0 || D <= 0 || B < 0) return DSA_ERR_INVALID_ARG;
    if (D != DSA_INDEX_DIM) return DSA_ERR_UNSUPPORTED;
    if (n == 0) return DSA_OK;
    if (!k_new || !gate_new || !tok_req || !tok_pos || (B > 0 && (!req_start || !k || !gate || !valid)))
        return DSA_ERR_INVALID_ARG;
    if (!aligned(k_new, 16) || !aligned(gate_new, 16) || !aligned(tok_req, 4) ||
        !aligned(tok_pos, 4) || !aligned(req_start, 4) || !aligned(k, 16) || !aligned(gate, 16))
        return DSA_ERR_ALIGNMENT;
    if (B == 0) return DSA_OK;
    const int grid = ceil_div(n, kStoreWarps);
    if (launch_pdl(indexer_store_kernel, dim3(grid), dim3(kStoreWarps * 32), 0, stream,
                   reinterpret_cast<const __nv_bfloat16 *>(k_new),
                   reinterpret_cast<const __nv_bfloat16 *>(gate_new), valid_new, tok_req, tok_pos, n,
                   req_start, B, reinterpret_cast<__nv_bfloat16 *>(k),
                   reinterpret_cast<__nv_bfloat16 *>(gate), valid) != cudaSuccess)
        return DSA_ERR_CUDA;
    return launch_status();
}

}  // namespace dsa
