// cluster.cuh -- thread-block cluster helpers for sm_100a, inline PTX: distributed shared
// memory (a CTA writes straight into another CTA's shared memory and signals that CTA's
// mbarrier), cluster-scope mbarrier waits, the cluster barrier, and L2 prefetch of a byte
// range with the bulk-copy engine.  Every wait is bounded by %globaltimer like the waits of
// tma.cuh: on timeout the device status word gets TERN_ETIMEOUT and the caller gets false.
#pragma once
#include <stdint.h>

#include "tma.cuh"

namespace tern {

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t peer_addr(const void *local, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(smem_u32(local)), "r"(rank));
    return d;
}

// Stores into a peer CTA's shared memory that count their bytes on that CTA's mbarrier (the
// mbarrier must live in the same CTA as the destination).  The receiver arms the mbarrier with
// the total byte count of the phase (mbar_expect_tx); stores may land before it is armed.
__device__ __forceinline__ void st_async_b32(uint32_t raddr, uint32_t v, uint32_t rmbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(raddr), "r"(v),
                 "r"(rmbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_b64(uint32_t raddr, unsigned long long v, uint32_t rmbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(raddr), "l"(v),
                 "r"(rmbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v4(uint32_t raddr, uint4 v, uint32_t rmbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1,%2,%3,%4}, [%5];" ::"r"(raddr),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(rmbar)
                 : "memory");
}

// mbarrier phase test with acquire at cluster scope (for data stored by peer CTAs)
__device__ __forceinline__ bool mbar_test_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, "
        "p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, long long limit_ns, int *status) {
    if (mbar_test_cluster(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    while (!mbar_test_cluster(bar, parity)) {
        if ((long long)(gtimer() - t0) > limit_ns) {
            set_status(status, TERN_ETIMEOUT);
            return false;
        }
    }
    return true;
}

// all threads of all CTAs of the cluster (every thread must call it)
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Fetch [src, src+bytes) into L2 without a destination in shared memory (bytes: multiple of
// 16, src 16-byte aligned).  A hint: it changes no value anywhere.
__device__ __forceinline__ void prefetch_l2_bulk(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 64-bit tagged word stores/loads at GPU scope (single-copy atomic per 8-byte word)
__device__ __forceinline__ void st_relaxed_v2(unsigned long long *p, unsigned long long a, unsigned long long b) {
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1,%2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
__device__ __forceinline__ ulonglong2 ld_relaxed_v2(const unsigned long long *p) {
    ulonglong2 v;
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0,%1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
    return v;
}

}  // namespace tern
