// mbarrier.cuh -- shared-memory mbarriers and bulk global -> shared copies
// (cp.async.bulk, no tensor map, no multicast), for the kernels that stream
// their inputs through shared-memory rings: the decode kernel and the bulk
// quantise-append kernel.
//
// Every wait is bounded: a wait that does not see its phase within
// kSpinLimit polls returns false, and the caller records an error status and
// leaves its loop, so a lost copy never hangs the device.
#pragma once
#include "common.cuh"

namespace tbq4 {

constexpr uint32_t kSpinLimit = 1u << 22;                  // polls per bounded wait

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// One arrival that also raises the phase's expected transaction bytes.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// One plain arrival (release semantics: this thread's shared-memory reads
// before it are ordered before the phase completes).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity; gives up after kSpinLimit
// polls and returns false (warp-uniform).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    bool ok = false;
    for (uint32_t i = 0; i < kSpinLimit && !ok; ++i) ok = mbar_try_wait(bar, parity);
    return __all_sync(kFull, ok);
}

// bytes from global src to shared dst (both 16-byte aligned, bytes a
// multiple of 16), completing as transaction bytes on bar.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

}  // namespace tbq4
