// tma.cuh -- bulk-copy engine (TMA) and mbarrier helpers for sm_100a, inline PTX.
//
// A bulk copy (cp.async.bulk global -> shared) is issued by one thread and signals an
// mbarrier with its byte count; threads that need the data wait on that mbarrier's phase.
// Every wait here is bounded by %globaltimer: on timeout the device status word is set to
// TERN_ETIMEOUT and the caller gets false.
#pragma once
#include <stdint.h>

#include "tern_common.cuh"

namespace tern {

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// arrive (count 1) and add `bytes` to the transaction count of the current phase
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// plain arrive (count 1), release semantics at CTA scope
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// bytes: multiple of 16; both addresses 16-byte aligned
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Shared buffers are rewritten by TMA only after every thread's generic reads of them are
// ordered before the issuing thread by a barrier (CTA, named or mbarrier); write-after-read
// across the generic and async proxies needs no proxy fence.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bounded wait on an mbarrier phase; false on timeout (status set)
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit_ns, int *status) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_test(bar, parity)) {
        if ((long long)(gtimer() - t0) > limit_ns) {
            set_status(status, TERN_ETIMEOUT);
            return false;
        }
    }
    return true;
}

// Same wait, but the thread is suspended inside each try_wait until the phase completes or
// `hint_ns` elapses, so waiting warps take no issue slots from warps that have work.
__device__ __forceinline__ bool mbar_test_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, long long limit_ns, int *status) {
    if (mbar_test_sleep(bar, parity, 20000u)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_test_sleep(bar, parity, 20000u)) {
        if ((long long)(gtimer() - t0) > limit_ns) {
            set_status(status, TERN_ETIMEOUT);
            return false;
        }
    }
    return true;
}

// barrier over `nthreads` threads (multiple of 32) using hardware barrier `id` (1..15)
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace tern
