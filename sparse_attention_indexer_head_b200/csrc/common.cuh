// Shared device helpers of the sm_100a DSA kernels: bf16 packing, mbarrier and
// bulk-copy PTX wrappers with bounded waits, and host-side argument checks.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/dsa.h"

#define DSA_DEVINL __device__ __forceinline__

namespace dsa {

// ---------------------------------------------------------------- device error flag
// Sticky flag a kernel sets when a bounded wait gives up (it then returns early
// instead of spinning forever). Read and cleared by dsa_device_status(). The
// library is a single translation unit (csrc/dsa_abi.cu), so it is defined here.
__device__ int g_device_error = 0;

enum : int { kErrWaitTimeout = 1 };

DSA_DEVINL void raise_device_error(int code) { atomicOr(&g_device_error, code); }

// ---------------------------------------------------------------- bf16 helpers
DSA_DEVINL float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
DSA_DEVINL float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Round two floats to bf16 (nearest even) and pack lo | hi << 16.
DSA_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

DSA_DEVINL float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

DSA_DEVINL void unpack8(const uint4 &v, float (&x)[8]) {
    x[0] = bf16lo(v.x); x[1] = bf16hi(v.x);
    x[2] = bf16lo(v.y); x[3] = bf16hi(v.y);
    x[4] = bf16lo(v.z); x[5] = bf16hi(v.z);
    x[6] = bf16lo(v.w); x[7] = bf16hi(v.w);
}

// ---------------------------------------------------------------- shared-memory addressing
DSA_DEVINL uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
DSA_DEVINL void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

DSA_DEVINL void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

DSA_DEVINL void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

DSA_DEVINL void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

DSA_DEVINL bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete. Gives up once about two
// seconds of SM clock cycles have passed (each try_wait may itself suspend for
// a while, so the bound is on elapsed cycles, not on the number of polls),
// raises the device error flag and returns false.
constexpr long long kWaitLimitCycles = 4000000000ll;
// Non-blocking probe: has the phase with this parity completed?
DSA_DEVINL bool mbar_test(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase)
        : "memory");
    return ok != 0;
}

DSA_DEVINL bool mbar_wait(uint64_t *bar, uint32_t phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, phase)) return true;
        if (clock64() - t0 > kWaitLimitCycles) break;
    }
    raise_device_error(kErrWaitTimeout);
    return false;
}

// ---------------------------------------------------------------- bulk async copy (TMA, 1-D)
// Global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) completing on `bar` via the transaction count.
DSA_DEVINL void bulk_g2s(void *smem_dst, const void *gmem_src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------- misc
DSA_DEVINL float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// MUFU reciprocal / reciprocal square root (relative error about 2^-23); used
// where the result is rounded to bf16 afterwards.
DSA_DEVINL float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
DSA_DEVINL float rsqrt_approx(float x) {
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T>
DSA_DEVINL T ldg_nc(const T *p) { return __ldg(p); }

DSA_DEVINL bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

DSA_DEVINL uint4 ldg_nc_v4(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel of the path is launched with programmatic stream serialization:
// it may start while its predecessor in the stream is still running. Each
// kernel therefore (1) does only setup that reads nothing a predecessor writes
// and writes nothing a predecessor reads, (2) waits for the predecessor grid to
// complete (griddepcontrol.wait; a no-op without the launch attribute), then
// (3) lets its own successor start launching. A kernel thus overlaps only its
// immediate predecessor, whose own wait has already returned, so everything
// earlier has completed.
// ---------------------------------------------------------------- thread-block clusters
// Address of the same shared-memory location in the CTA of cluster rank `rank`.
DSA_DEVINL uint32_t cluster_map(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
DSA_DEVINL float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
DSA_DEVINL float4 ld_cluster_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
// Every thread of every CTA of the cluster; shared-memory writes before it are
// visible to the whole cluster after it.
DSA_DEVINL void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

DSA_DEVINL void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
DSA_DEVINL void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- host-side checks
inline bool aligned(const void *p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Launch with the programmatic-stream-serialization attribute (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// launch_pdl with a thread-block cluster of cluster_x CTAs along grid x, set at
// launch time (the kernel carries no __cluster_dims__).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t stream, int cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Streaming-multiprocessor count of the current device (persistent grids).
inline int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Raise a kernel's dynamic shared-memory limit once per device (the attribute
// is per device context). Returns false if the runtime refuses.
inline bool ensure_smem_attr(const void *func, int bytes) {
    if (bytes <= 48 * 1024) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, func) != cudaSuccess) return false;
    if (attr.maxDynamicSharedSizeBytes >= bytes) return true;
    return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
           cudaSuccess;
}

}  // namespace dsa
