// common.cuh -- device helpers shared by the scan and residual kernels of libr2l.
//
// Inline PTX for the sm_100a asynchronous machinery used by the kernels: mbarriers,
// bulk (TMA-engine) global->shared copies, the hardware base-2 exponential, and a
// time-bounded mbarrier wait that reports instead of hanging.
#pragma once

#include <cstdint>
#include <cstdio>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace r2l {

// Device status word: bit flags set by kernels that gave up a bounded wait.
// Read and cleared by r2l_device_status().
enum : unsigned {
    kStatusTimeoutScan = 1u,
    kStatusTimeoutGemm = 2u,
    kStatusTimeoutSelftest = 4u,
    kStatusDrainTimeout = 8u  // after a timeout, copies into shared memory were still in flight at exit
};
__device__ unsigned int g_status_word;

// Upper bound for any spin on an mbarrier: 2 s of wall time (%globaltimer is in ns).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies, tcgen05).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __noinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// mbar_wait_bounded with the already-complete case inline (no call).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || mbar_wait_bounded(bar, parity);
}

// One lane of the (fully active) warp: true in exactly one of them.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}

// Bulk asynchronous copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Programmatic dependent launch: wait until the preceding kernel in the stream has completed and
// its writes are visible (returns at once when the launch had no programmatic dependency).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Programmatic dependent launch: allow the next kernel in the stream to be scheduled once every CTA
// of this grid has issued this (or exited).  Its CTAs may then start on SMs this grid leaves idle
// and run their set-up; they still wait in pdl_wait() for this grid to complete before they touch
// global memory, as every kernel of the library does.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Hardware 2^x (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2_hw(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Hardware reciprocal (MUFU), flush-to-zero.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// SiLU(v) = v / (1 + e^-v) with the hardware 2^x and reciprocal (a few ulp, far below bf16).
__device__ __forceinline__ float silu_mufu(float v) { return v * rcp_approx(1.0f + ex2_hw(-1.4426950408889634f * v)); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Host: last failure of a CUDA call made by the library on this thread (see r2l_last_error).
inline char* last_error_buffer() {
    static thread_local char buf[256] = "";
    return buf;
}

inline bool cuda_ok(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return true;
    snprintf(last_error_buffer(), 256, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
    return false;
}

// Host: raise a kernel's dynamic shared-memory limit when a launch needs more than 48 KiB.
// The limit is raised to exactly what is asked (the opt-in maximum minus the kernel's static
// shared memory bounds it) and remembered per kernel, so steady-state launches skip the call.
inline int prepare_kernel_smem(const void* fn, int smem_bytes) {
    static std::mutex mu;
    static const void* fns[256];
    static int limits[256];
    static int n = 0;
    if (smem_bytes <= 48 * 1024) return 0;
    std::lock_guard<std::mutex> lock(mu);
    int slot = -1;
    for (int i = 0; i < n; ++i)
        if (fns[i] == fn) slot = i;
    if (slot >= 0 && limits[slot] >= smem_bytes) return 0;
    if (!cuda_ok(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes),
                 "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)"))
        return -1;
    if (slot < 0 && n < 256) {
        slot = n++;
        fns[slot] = fn;
    }
    if (slot >= 0) limits[slot] = smem_bytes;
    return 0;
}

// Host: launch with programmatic stream serialization, so the kernel's launch and prologue may
// overlap the tail of the previous kernel in the stream (the kernel calls pdl_wait() before it
// touches global memory).
template <typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
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
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Same, with thread-block clusters of cluster_x CTAs along x (grid.x a multiple of cluster_x).
template <typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(Args...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t stream, unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace r2l
