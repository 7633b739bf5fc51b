// mbarrier.cuh -- shared-memory mbarriers, bulk global -> shared copies
// (cp.async.bulk, no tensor map, no multicast) and the proxy fences around
// them: the one home of these helpers for every kernel of the library (the
// decode and quantise-append rings, and the tcgen05 pipelines).
//
// Every wait is bounded: a wait that does not see its phase within its poll
// limit (kSpinLimit unless the caller gives one) returns false, and the
// caller records an error status and leaves its loop, so a lost copy never
// hangs the device.
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

// Makes barrier initialisation visible to the async proxy (bulk copies,
// tensor-core commits) before first use.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy ones (a bulk copy into a reused stage, a tensor-core read of
// an operand tile written by threads).
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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

// One poll that may suspend the thread for a short, hardware-chosen time.
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

// Non-blocking test of a phase (try_wait may suspend the thread for a while,
// which a thread polling several barriers must avoid).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for one thread: false after `limit` polls.
__device__ __forceinline__ bool mbar_wait_thread(uint32_t bar, uint32_t parity,
                                                 uint32_t limit = kSpinLimit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Bounded wait by a whole warp: every lane polls, and the result is the same
// in every lane (a warp never splits on a timeout).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint32_t limit = kSpinLimit) {
    bool ok = false;
    for (uint32_t i = 0; i < limit && !ok; ++i) ok = mbar_try_wait(bar, parity);
    return __all_sync(kFull, ok);
}

// Bounded wait that sleeps `ns` nanoseconds between polls, for a thread that
// runs ahead of its consumers: a polling warp takes issue slots from the
// warps it shares a scheduler with.  False after `limit` polls.
__device__ __forceinline__ bool mbar_wait_lazy(uint32_t bar, uint32_t parity, uint32_t limit,
                                               uint32_t ns) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        __nanosleep(ns);
    }
    return false;
}
__device__ __forceinline__ bool mbar_wait_lazy_warp(uint32_t bar, uint32_t parity,
                                                    uint32_t limit, uint32_t ns) {
    const bool ok = mbar_wait_lazy(bar, parity, limit, ns);
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
