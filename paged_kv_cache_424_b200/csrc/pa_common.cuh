// pa_common.cuh -- shared device helpers for the sm_100a kernels: element
// types, the device error word, mbarrier waits with a time limit, and 1-D
// bulk (TMA engine) copies from global to shared memory.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/pa.h"

namespace pa {

// Device error word: PA_DEVERR_* bits, set with atomicOr, read and cleared by
// pa_device_error().  One per device (a __device__ variable of this library).
extern __device__ unsigned int g_device_error;

__device__ __forceinline__ void flag_error(unsigned int bit) { atomicOr(&g_device_error, bit); }

// ---------------------------------------------------------------------------
// 16-bit element types
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<__half> {
    using T2 = __half2;
    static __device__ __forceinline__ float2 to_float2(uint32_t bits) {
        __half2 h = *reinterpret_cast<const __half2 *>(&bits);
        return __half22float2(h);
    }
    static __device__ __forceinline__ __half from_float(float x) { return __float2half_rn(x); }
    static __device__ __forceinline__ float to_float(__half x) { return __half2float(x); }
};
template <> struct Elem<__nv_bfloat16> {
    using T2 = __nv_bfloat162;
    static __device__ __forceinline__ float2 to_float2(uint32_t bits) {
        // bf16 is the upper half of an fp32: widening is a shift / mask.
        float2 r;
        r.x = __uint_as_float(bits << 16);
        r.y = __uint_as_float(bits & 0xffff0000u);
        return r;
    }
    static __device__ __forceinline__ __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
    static __device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
};

// FP8 E4M3 cache element (stored as its 8-bit code).
struct E4M3 {
    uint8_t code;
};

// Two E4M3 codes (element 0 in the low byte) -> f16x2 bits (element 0 in
// the low half), exactly: one cvt (PTX ISA, cvt with .e4m3x2 source, sm_89+).
__device__ __forceinline__ uint32_t e4m3x2_to_half2_bits(uint16_t pair) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(pair));
    return r;
}

// The two 16-bit halves of a 32-bit word (a register split, no arithmetic).
__device__ __forceinline__ void split_b32(uint32_t w, uint16_t &lo, uint16_t &hi) {
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
}

// Two E4M3 codes (element 0 in the low byte) -> two floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t pair) {
    const uint32_t h = e4m3x2_to_half2_bits(pair);
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Two floats -> two E4M3 codes, nearest with ties to even, clamped to the
// largest finite magnitude (element 0 in the low byte).
__device__ __forceinline__ uint16_t float2_to_e4m3x2(float lo, float hi) {
    return __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

// ---------------------------------------------------------------------------
// shared-memory addresses, mbarriers and bulk copies (PTX ISA: mbarrier,
// cp.async.bulk; available on sm_90 and later, used here for sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy / tensor core) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking: whether the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// about `limit_cycles` SM clock cycles (~2 s at 2 GHz), sets
// PA_DEVERR_TIMEOUT and returns false, so a lost completion can never hang
// the GPU.  The cycle counter is cheap to read, unlike the global timer, so
// a single-thread producer pays almost nothing when it has to wait.
constexpr long long kWaitLimitCycles = 4000000000ll;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit_cycles = kWaitLimitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > limit_cycles) {
            flag_error(PA_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// 1-D bulk copy global -> shared through the TMA engine, completing `bytes`
// transaction bytes on `bar`.  src and dst 16-byte aligned, bytes % 16 == 0.
// No multicast: the copy lands in this CTA's shared memory only.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Programmatic dependent launch (PDL).  Kernels of this library are launched
// so that their launch and prologue may overlap the tail of the kernel before
// them on the stream; each calls pdl_wait() before it touches global memory
// (which waits for the previous grid to finish and flush), and
// pdl_launch_dependents() to let the next kernel start launching early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args) {
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
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pa
