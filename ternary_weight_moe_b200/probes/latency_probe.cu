// latency_probe.cu -- measurements of the on-chip latencies the persistent decode kernel is
// built around, on the current GPU (a standalone program, not part of libternmoe; run with
// `python bench.py --latency-probe`, which compiles it with nvcc and prints its JSON).
//
// Every figure is a median over repetitions of clock64 differences read by one thread, in SM
// cycles:
//   chain_*      one warp, one dependent chain of 256 operations: cycles per operation
//   bar_*        a CTA barrier (512 threads) / a named barrier (256 threads): cycles per barrier
//   topk_*       top-8 of 256 fp64 logits (ties to the lower index): the one-warp filter of the
//                library (tern_common.cuh) and a CTA-wide filter, cycles per selection
//   bulk_*       issuing bulk copies (cp.async.bulk global -> shared): n copies from one lane,
//                or one copy from each of n warps; cycles until the issuing returns / until all
//                copies have landed
//   sts16_*      a 16-byte shared store with and without the async-proxy fence after it
//   mma_*        n tcgen05 kind::i8 MMAs (M = 128, N = 16, K = 32, operands in shared memory)
//                issued by one thread and committed to an mbarrier: cycles from the first issue
//                to the mbarrier's completion seen by the issuing thread
// Every wait is bounded; nothing here waits on another CTA.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <vector>

#include "../csrc/tern_common.cuh"
#include "../csrc/tma.cuh"

using namespace tern;

constexpr int kReps = 64;

__global__ void chains(unsigned long long *out, const double *dsrc, const int *isrc) {
    __shared__ int s_i[1024];
    __shared__ double s_d[256];
    const int lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 1024; i += blockDim.x) s_i[i] = (i * 7 + 3) & 1023;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_d[i] = dsrc[i];
    __syncthreads();
    if (threadIdx.x >= 32) return;
    unsigned long long t0, t1;
    // SHFL chain
    int v = lane;
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) v = __shfl_xor_sync(0xFFFFFFFFu, v, 1) + 1;
    t1 = clock64();
    if (lane == 0) out[0] = (t1 - t0);
    // LDS chain (pointer chasing)
    int ix = lane;
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) ix = s_i[ix];
    t1 = clock64();
    if (lane == 0) out[1] = (t1 - t0);
    // DFMA chain
    double a = dsrc[lane], b = dsrc[lane + 1];
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) a = fma(a, b, 1.0);
    t1 = clock64();
    if (lane == 0) out[2] = (t1 - t0);
    // fp64 division chain
    double q = dsrc[lane] + 2.0;
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) q = 3.0 / q;
    t1 = clock64();
    if (lane == 0) out[3] = (t1 - t0);
    // redux.sync max chain
    unsigned m = (unsigned)lane;
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) m = __reduce_max_sync(0xFFFFFFFFu, m + (unsigned)lane) & 0xFFFFu;
    t1 = clock64();
    if (lane == 0) out[4] = (t1 - t0);
    // fp32 -> fp64 -> fp32 conversion chain
    float fl = (float)dsrc[lane];
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) fl = (float)((double)fl * 1.0000001);
    t1 = clock64();
    if (lane == 0) out[5] = (t1 - t0);
    // integer ALU chain
    unsigned u = (unsigned)lane;
    t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) u = (u ^ (u >> 3)) + 0x9E37u;
    t1 = clock64();
    if (lane == 0) out[6] = (t1 - t0);
    // keep results alive
    // (m stays below 2^16: compare it with a value it can take, or the chain is dropped)
    if (v == -1 || ix == -1 || a == -1.0 || q == -1.0 || m == 12345u || fl == -1.0f || u == 1u) out[7] = 1;
}

__global__ void barriers(unsigned long long *out) {
    unsigned long long t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) __syncthreads();
    unsigned long long t1 = clock64();
    if (threadIdx.x == 0) out[0] = t1 - t0;
    if (threadIdx.x < 256) {
        t0 = clock64();
#pragma unroll 1
        for (int i = 0; i < 256; i++) named_bar_sync(1, 256);
        t1 = clock64();
        if (threadIdx.x == 0) out[1] = t1 - t0;
    }
}

// A 16-byte shared store followed by fence.proxy.async.shared::cta (what a thread does before
// the tensor core may read what it stored), against the store alone: cycles per iteration.
__global__ void proxy_fence(unsigned long long *out) {
    __shared__ uint4 buf[128];
    uint4 v = make_uint4(threadIdx.x, 1u, 2u, 3u);
    __syncthreads();
    unsigned long long t0 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) {
        buf[threadIdx.x] = v;
        v.x += 1u;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    unsigned long long t1 = clock64();
#pragma unroll 1
    for (int i = 0; i < 256; i++) {
        buf[threadIdx.x] = v;
        v.x += 1u;
        asm volatile("" ::: "memory");
    }
    unsigned long long t2 = clock64();
    __syncthreads();
    if (threadIdx.x == 0) {
        out[0] = t1 - t0;
        out[1] = t2 - t1;
        out[2] = buf[7].x;  // keeps the stores
    }
}

// CTA-wide filter: thread t < E holds logit t; result in idx_out (shared); all threads call.
__device__ void block_filter(const double *lg, int E, int k, int32_t *idx_out, uint32_t *s_gm, int *s_nc,
                             ulonglong2 *s_cand) {
    const int tid = threadIdx.x, lane = tid & 31;
    const bool has = tid < E;
    const unsigned long long key = has ? f64_order_key(lg[tid]) : 0ull;
    const uint32_t h = (uint32_t)(key >> 32);
    uint32_t gm = h;
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 1));
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 2));
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 4));
    if (tid < 256 && (tid & 7) == 0) s_gm[tid >> 3] = gm;
    if (tid == 0) *s_nc = 0;
    __syncthreads();
    if (tid < 256) {
        const uint32_t mm = s_gm[lane];
        int above = 0;
#pragma unroll
        for (int q4 = 0; q4 < 8; q4++) {
            const uint4 v = reinterpret_cast<const uint4 *>(s_gm)[q4];
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int z = 0; z < 4; z++) above += (vv[z] > mm || (vv[z] == mm && 4 * q4 + z < lane)) ? 1 : 0;
        }
        const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
        const uint32_t tau = __shfl_sync(0xFFFFFFFFu, mm, __ffs(who) - 1);
        const bool take = has && h >= tau;
        const unsigned msk = __ballot_sync(0xFFFFFFFFu, take);
        int base = 0;
        if (lane == 0 && msk) base = atomicAdd(s_nc, __popc(msk));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (take) s_cand[base + __popc(msk & ((1u << lane) - 1u))] = make_ulonglong2(key, (unsigned long long)tid);
    }
    __syncthreads();
    const int nc = *s_nc;
    if (tid < nc) {
        const ulonglong2 me = s_cand[tid];
        int r = 0;
        for (int q = 0; q < nc; q++) {
            const ulonglong2 o = s_cand[q];
            r += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
        }
        if (r < k) idx_out[r] = (int)me.y;
    }
    __syncthreads();
}

// The one-warp filter with tau taken by 32 shuffles, step by step (a clock64 stamp after each
// step): st[0..5] = keys, tau, ballots, compaction, ranking, total.
__global__ void topk_steps(const double *logits, unsigned long long *out) {
    __shared__ double lg[256];
    __shared__ ulonglong2 cand[256];
    __shared__ int32_t idx_out[8];
    const int lane = threadIdx.x & 31;
    const int E = 256, k = 8;
    for (int rep = 0; rep < kReps; rep++) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) lg[i] = logits[rep * 256 + i];
        __syncthreads();
        if (threadIdx.x < 32) {
            unsigned long long c0 = clock64();
            unsigned long long key[8];
            uint32_t hi[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int e = lane + 32 * j;
                key[j] = f64_order_key(lg[e]);
                hi[j] = (uint32_t)(key[j] >> 32);
            }
            const uint32_t m = max(max(max(hi[0], hi[1]), max(hi[2], hi[3])), max(max(hi[4], hi[5]), max(hi[6], hi[7])));
            __syncwarp();
            unsigned long long c1 = clock64();
            int above4[4] = {0, 0, 0, 0};
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const uint32_t v = __shfl_sync(0xFFFFFFFFu, m, i);
                above4[i & 3] += (v > m || (v == m && i < lane)) ? 1 : 0;
            }
            const int above = (above4[0] + above4[1]) + (above4[2] + above4[3]);
            const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
            const uint32_t tau = __shfl_sync(0xFFFFFFFFu, m, __ffs(who) - 1);
            unsigned long long c2 = clock64();
            unsigned msk[8];
#pragma unroll
            for (int j = 0; j < 8; j++) msk[j] = __ballot_sync(0xFFFFFFFFu, hi[j] >= tau);
            unsigned long long c3 = clock64();
            const unsigned below = (1u << lane) - 1u;
            int base = 0;
#pragma unroll
            for (int j = 0; j < 8; j++) {
                if ((msk[j] >> lane) & 1u) cand[base + __popc(msk[j] & below)] = make_ulonglong2(key[j], (unsigned long long)(lane + 32 * j));
                base += __popc(msk[j]);
            }
            const int nc = base;
            __syncwarp();
            unsigned long long c4 = clock64();
            for (int i = lane; i < nc; i += 32) {
                const ulonglong2 me = cand[i];
                int r4[4] = {0, 0, 0, 0};
                int q = 0;
                for (; q + 4 <= nc; q += 4) {
#pragma unroll
                    for (int z = 0; z < 4; z++) {
                        const ulonglong2 o = cand[q + z];
                        r4[z] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
                    }
                }
                for (; q < nc; q++) {
                    const ulonglong2 o = cand[q];
                    r4[0] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
                }
                const int r = (r4[0] + r4[1]) + (r4[2] + r4[3]);
                if (r < k) idx_out[r] = (int)me.y;
            }
            __syncwarp();
            unsigned long long c5 = clock64();
            if (lane == 0) {
                unsigned long long *o = out + rep * 8;
                o[0] = c1 - c0; o[1] = c2 - c1; o[2] = c3 - c2; o[3] = c4 - c3; o[4] = c5 - c4; o[5] = c5 - c0;
                o[6] = (unsigned long long)nc;
            }
        }
        __syncthreads();
    }
}

__global__ void topk_bench(const double *logits, unsigned long long *out, int32_t *idx_a, int32_t *idx_b) {
    __shared__ double lg[256];
    __shared__ int32_t s_idx[8];
    __shared__ ulonglong2 cand[256];
    __shared__ __align__(16) uint32_t s_tkm[32];
    __shared__ __align__(16) uint32_t s_gm[32];
    __shared__ int s_nc;
    for (int rep = 0; rep < kReps; rep++) {
        if (threadIdx.x < 256) lg[threadIdx.x] = logits[rep * 256 + threadIdx.x];
        __syncthreads();
        unsigned long long t0 = clock64();
        if (threadIdx.x < 32) warp_topk_filter(lg, 256, 8, s_idx, cand, s_tkm);
        __syncthreads();
        unsigned long long t1 = clock64();
        if (threadIdx.x < 8) idx_a[rep * 8 + threadIdx.x] = s_idx[threadIdx.x];
        if (threadIdx.x == 0) out[2 * rep] = t1 - t0;
        __syncthreads();
        t0 = clock64();
        block_filter(lg, 256, 8, s_idx, s_gm, &s_nc, cand);
        t1 = clock64();
        if (threadIdx.x < 8) idx_b[rep * 8 + threadIdx.x] = s_idx[threadIdx.x];
        if (threadIdx.x == 0) out[2 * rep + 1] = t1 - t0;
        __syncthreads();
    }
}

// Two other formulations of the one-warp filter, timed beside the library's (which reads tau
// from shared memory and compacts by ballots): V == 0 takes tau by 32 shuffles; V == 2 reads
// tau like the library but compacts by per-lane counts and a prefix read from shared memory.
template <int V>
static __device__ __noinline__ void topk_variant(const double *lg, int k, int32_t *idx_out, ulonglong2 *cand) {
    __shared__ __align__(16) uint32_t s_m[32];
    __shared__ __align__(16) int s_c[32];
    const int lane = threadIdx.x & 31;
    unsigned long long key[8];
    uint32_t hi[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        key[j] = f64_order_key(lg[lane + 32 * j]);
        hi[j] = (uint32_t)(key[j] >> 32);
    }
    const uint32_t m = max(max(max(hi[0], hi[1]), max(hi[2], hi[3])), max(max(hi[4], hi[5]), max(hi[6], hi[7])));
    int above4[4] = {0, 0, 0, 0};
    uint32_t tau;
    if (V == 0) {
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const uint32_t v = __shfl_sync(0xFFFFFFFFu, m, i);
            above4[i & 3] += (v > m || (v == m && i < lane)) ? 1 : 0;
        }
        const int above = (above4[0] + above4[1]) + (above4[2] + above4[3]);
        const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
        tau = __shfl_sync(0xFFFFFFFFu, m, __ffs(who) - 1);
    } else {
        s_m[lane] = m;
        __syncwarp();
#pragma unroll
        for (int q4 = 0; q4 < 8; q4++) {
            const uint4 v = reinterpret_cast<const uint4 *>(s_m)[q4];
            above4[0] += (v.x > m || (v.x == m && 4 * q4 + 0 < lane)) ? 1 : 0;
            above4[1] += (v.y > m || (v.y == m && 4 * q4 + 1 < lane)) ? 1 : 0;
            above4[2] += (v.z > m || (v.z == m && 4 * q4 + 2 < lane)) ? 1 : 0;
            above4[3] += (v.w > m || (v.w == m && 4 * q4 + 3 < lane)) ? 1 : 0;
        }
        const int above = (above4[0] + above4[1]) + (above4[2] + above4[3]);
        const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
        tau = s_m[__ffs(who) - 1];
    }
    int nc = 0;
    if (V == 2) {
        int c = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) c += hi[j] >= tau ? 1 : 0;
        s_c[lane] = c;
        __syncwarp();
        int pre = 0;
#pragma unroll
        for (int q4 = 0; q4 < 8; q4++) {
            const int4 v = reinterpret_cast<const int4 *>(s_c)[q4];
            pre += (4 * q4 + 0 < lane ? v.x : 0) + (4 * q4 + 1 < lane ? v.y : 0);
            pre += (4 * q4 + 2 < lane ? v.z : 0) + (4 * q4 + 3 < lane ? v.w : 0);
            nc += (v.x + v.y) + (v.z + v.w);
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if (hi[j] >= tau) cand[pre++] = make_ulonglong2(key[j], (unsigned long long)(lane + 32 * j));
        }
    } else {
        unsigned msk[8];
#pragma unroll
        for (int j = 0; j < 8; j++) msk[j] = __ballot_sync(0xFFFFFFFFu, hi[j] >= tau);
        const unsigned below = (1u << lane) - 1u;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            if ((msk[j] >> lane) & 1u) cand[nc + __popc(msk[j] & below)] = make_ulonglong2(key[j], (unsigned long long)(lane + 32 * j));
            nc += __popc(msk[j]);
        }
    }
    __syncwarp();
    for (int i = lane; i < nc; i += 32) {
        const ulonglong2 me = cand[i];
        int r4[4] = {0, 0, 0, 0};
        int q = 0;
        for (; q + 4 <= nc; q += 4) {
#pragma unroll
            for (int z = 0; z < 4; z++) {
                const ulonglong2 o = cand[q + z];
                r4[z] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
            }
        }
        for (; q < nc; q++) {
            const ulonglong2 o = cand[q];
            r4[0] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
        }
        const int r = (r4[0] + r4[1]) + (r4[2] + r4[3]);
        if (r < k) idx_out[r] = (int)me.y;
    }
    __syncwarp();
}

// out[3 * rep + v]: cycles of variant v (0: shuffles, 1: the library's, 2: count prefix);
// idx[(3 * rep + v) * 8 + j]: its selection
__global__ void topk_variants(const double *logits, unsigned long long *out, int32_t *idx) {
    __shared__ double lg[256];
    __shared__ int32_t s_idx[8];
    __shared__ ulonglong2 cand[256];
    __shared__ __align__(16) uint32_t s_tkm[32];
    for (int rep = 0; rep < kReps; rep++) {
        if (threadIdx.x < 256) lg[threadIdx.x] = logits[rep * 256 + threadIdx.x];
        __syncthreads();
        for (int v = 0; v < 3; v++) {
            if (threadIdx.x < 32) {
                const unsigned long long t0 = clock64();
                if (v == 0) topk_variant<0>(lg, 8, s_idx, cand);
                else if (v == 1) warp_topk_filter(lg, 256, 8, s_idx, cand, s_tkm);
                else topk_variant<2>(lg, 8, s_idx, cand);
                const unsigned long long t1 = clock64();
                if (threadIdx.x < 8) idx[(3 * rep + v) * 8 + threadIdx.x] = s_idx[threadIdx.x];
                if (threadIdx.x == 0) out[3 * rep + v] = t1 - t0;
            }
            __syncthreads();
        }
    }
}

// bulk copies of `bytes` each from src into shared memory: mode 0 = n copies from lane 0 of
// warp 0, mode 1 = one copy from lane 0 of each of n warps.
__global__ void bulk_issue(const uint8_t *src, int n, int bytes, int mode, unsigned long long *out, int *status) {
    extern __shared__ __align__(128) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&mb, 1);
        fence_mbar_init();
    }
    __syncthreads();
    for (int rep = 0; rep < 8; rep++) {
        if (threadIdx.x == 0) mbar_expect_tx(&mb, (uint32_t)(n * bytes));
        __syncthreads();
        const unsigned long long t0 = clock64();
        const uint8_t *s = src + (size_t)rep * n * bytes;
        if (mode == 0) {
            if (threadIdx.x == 0)
                for (int i = 0; i < n; i++) bulk_g2s(sm + (size_t)i * bytes, s + (size_t)i * bytes, (uint32_t)bytes, &mb);
        } else if (warp < n && lane == 0) {
            bulk_g2s(sm + (size_t)warp * bytes, s + (size_t)warp * bytes, (uint32_t)bytes, &mb);
        }
        __syncthreads();
        const unsigned long long t1 = clock64();
        mbar_wait(&mb, (uint32_t)(rep & 1), 1000000000ll, status);
        const unsigned long long t2 = clock64();
        if (threadIdx.x == 0) {
            out[2 * rep] = t1 - t0;
            out[2 * rep + 1] = t2 - t0;
        }
        __syncthreads();
    }
}

// tcgen05 pieces (the forms the grouped kernels use): K-major operands without swizzle, 64
// bytes of K per row, core matrices of 8 rows x 16 bytes
__device__ __forceinline__ uint64_t pr_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(512u >> 4) << 32) |
           (1ull << 46);
}
__global__ void mma_commit(unsigned long long *out, int *status) {
    __shared__ __align__(1024) unsigned char A[128 * 64];
    __shared__ __align__(1024) unsigned char B[16 * 64];
    __shared__ __align__(8) uint64_t mb;
    __shared__ uint32_t s_tmem;
    for (int i = threadIdx.x; i < 128 * 64 / 16; i += blockDim.x) reinterpret_cast<uint4 *>(A)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 16 * 64 / 16; i += blockDim.x) reinterpret_cast<uint4 *>(B)[i] = make_uint4(1u, 1u, 1u, 1u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(&mb, 1);
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(64u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;
    const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(16 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    if (threadIdx.x == 0) {
        const uint64_t a0 = pr_desc(smem_u32(A)), b0 = pr_desc(smem_u32(B));
        unsigned ph = 0;
        for (int v = 0; v < 3; v++) {
            const int n = 1 << v;  // 1, 2, 4 MMAs (4: one gate/up tile of the grouped kernel)
            for (int r = 0; r < kReps; r++) {
                const unsigned long long t0 = clock64();
                for (int q = 0; q < n; q++) {
                    const uint64_t off = (uint64_t)((q & 1) * 256) >> 4;  // K step 0 or 1
                    const uint32_t acc = q > 0 ? 1u : 0u;
                    asm volatile(
                        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(tmem),
                        "l"(a0 + off), "l"(b0 + off), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&mb))
                             : "memory");
                mbar_wait(&mb, ph & 1u, 1000000000ll, status);
                ph++;
                const unsigned long long t1 = clock64();
                out[v * kReps + r] = t1 - t0;
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x < 32)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64u) : "memory");
}

static double median(std::vector<double> v) {
    std::sort(v.begin(), v.end());
    return v.empty() ? 0.0 : v[v.size() / 2];
}

#define CK(x)                                                                                         \
    do {                                                                                              \
        cudaError_t e_ = (x);                                                                         \
        if (e_ != cudaSuccess) {                                                                      \
            printf("{\"error\": \"%s: %s\"}\n", #x, cudaGetErrorString(e_));                          \
            return 1;                                                                                 \
        }                                                                                             \
    } while (0)

int main() {
    CK(cudaSetDevice(0));
    unsigned long long *d_out;
    double *d_lg;
    int *d_st, *d_i;
    int32_t *d_ia, *d_ib;
    uint8_t *d_src;
    CK(cudaMalloc(&d_out, 4096 * 8));
    CK(cudaMalloc(&d_lg, kReps * 256 * 8));
    CK(cudaMalloc(&d_st, 4));
    CK(cudaMalloc(&d_i, 4096));
    CK(cudaMalloc(&d_ia, kReps * 8 * 4));
    CK(cudaMalloc(&d_ib, kReps * 8 * 4));
    CK(cudaMalloc(&d_src, 64 << 20));
    CK(cudaMemset(d_src, 1, 64 << 20));
    CK(cudaMemset(d_st, 0, 4));
    // logits: N(0, 1)-like values from a small LCG, a few exact ties
    std::vector<double> h(kReps * 256);
    unsigned long long z = 0x1234567ull;
    for (auto &x : h) {
        z = z * 6364136223846793005ull + 1442695040888963407ull;
        x = ((double)(z >> 11) / 9007199254740992.0 - 0.5) * 4.0;
    }
    for (int r = 0; r < kReps; r += 8) h[r * 256 + 17] = h[r * 256 + 200];
    CK(cudaMemcpy(d_lg, h.data(), h.size() * 8, cudaMemcpyHostToDevice));
    std::vector<unsigned long long> o(4096);

    printf("{");
    chains<<<1, 128>>>(d_out, d_lg, d_i);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(o.data(), d_out, 8 * 8, cudaMemcpyDeviceToHost));
    const char *names[] = {"chain_shfl", "chain_lds", "chain_dfma", "chain_f64_div", "chain_redux_max",
                           "chain_f32_f64_f32", "chain_int_alu"};
    for (int i = 0; i < 7; i++) printf("\"%s\": %.1f, ", names[i], o[i] / 256.0);

    barriers<<<1, 512>>>(d_out);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(o.data(), d_out, 2 * 8, cudaMemcpyDeviceToHost));
    printf("\"bar_cta512\": %.1f, \"bar_named256\": %.1f, ", o[0] / 256.0, o[1] / 256.0);

    proxy_fence<<<1, 128>>>(d_out);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(o.data(), d_out, 2 * 8, cudaMemcpyDeviceToHost));
    printf("\"sts16_proxy_fence\": %.1f, \"sts16_alone\": %.1f, ", o[0] / 256.0, o[1] / 256.0);

    {
        int *d_st;
        CK(cudaMalloc(&d_st, sizeof(int)));
        CK(cudaMemset(d_st, 0, sizeof(int)));
        mma_commit<<<1, 128>>>(d_out, d_st);
        CK(cudaDeviceSynchronize());
        std::vector<unsigned long long> m(3 * kReps);
        CK(cudaMemcpy(m.data(), d_out, 3 * kReps * 8, cudaMemcpyDeviceToHost));
        int mst = 0;
        CK(cudaMemcpy(&mst, d_st, sizeof(int), cudaMemcpyDeviceToHost));
        for (int v = 0; v < 3; v++) {
            std::vector<double> t;
            for (int r = 1; r < kReps; r++) t.push_back((double)m[v * kReps + r]);
            printf("\"mma_%d_commit\": %.0f, ", 1 << v, median(t));
        }
        printf("\"mma_status\": %d, ", mst);
        CK(cudaFree(d_st));
    }

    topk_bench<<<1, 512>>>(d_lg, d_out, d_ia, d_ib);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(o.data(), d_out, 2 * kReps * 8, cudaMemcpyDeviceToHost));
    std::vector<double> ta, tb;
    for (int r = 1; r < kReps; r++) {
        ta.push_back((double)o[2 * r]);
        tb.push_back((double)o[2 * r + 1]);
    }
    std::vector<int32_t> ia(kReps * 8), ib(kReps * 8);
    CK(cudaMemcpy(ia.data(), d_ia, ia.size() * 4, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(ib.data(), d_ib, ib.size() * 4, cudaMemcpyDeviceToHost));
    // check both against a host selection (larger first, ties to the lower index)
    int bad = 0;
    for (int r = 0; r < kReps; r++) {
        std::vector<int> ord(256);
        for (int i = 0; i < 256; i++) ord[i] = i;
        std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return h[r * 256 + a] > h[r * 256 + b]; });
        for (int j = 0; j < 8; j++) bad += (ia[r * 8 + j] != ord[j]) + (ib[r * 8 + j] != ord[j]);
    }
    printf("\"topk_warp_filter\": %.0f, \"topk_block_filter\": %.0f, \"topk_mismatches\": %d, ", median(ta), median(tb),
           bad);

    topk_steps<<<1, 512>>>(d_lg, d_out);
    CK(cudaDeviceSynchronize());
    CK(cudaMemcpy(o.data(), d_out, kReps * 8 * 8, cudaMemcpyDeviceToHost));
    {
        const char *sn[] = {"keys", "tau", "ballots", "compact", "rank", "total", "candidates"};
        for (int st = 0; st < 7; st++) {
            std::vector<double> v;
            for (int r = 1; r < kReps; r++) v.push_back((double)o[r * 8 + st]);
            printf("\"topk_step_%s\": %.0f, ", sn[st], median(v));
        }
    }

    {
        int32_t *d_iv;
        CK(cudaMalloc(&d_iv, kReps * 3 * 8 * 4));
        topk_variants<<<1, 512>>>(d_lg, d_out, d_iv);
        CK(cudaDeviceSynchronize());
        CK(cudaMemcpy(o.data(), d_out, kReps * 3 * 8, cudaMemcpyDeviceToHost));
        std::vector<int32_t> iv(kReps * 3 * 8);
        CK(cudaMemcpy(iv.data(), d_iv, iv.size() * 4, cudaMemcpyDeviceToHost));
        const char *vn[] = {"shuffle_tau", "shared_tau", "count_prefix"};
        for (int v = 0; v < 3; v++) {
            std::vector<double> tv;
            for (int r = 1; r < kReps; r++) tv.push_back((double)o[3 * r + v]);
            int badv = 0;
            for (int r = 0; r < kReps; r++) {
                std::vector<int> ord(256);
                for (int i = 0; i < 256; i++) ord[i] = i;
                std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return h[r * 256 + a] > h[r * 256 + b]; });
                for (int j = 0; j < 8; j++) badv += iv[(3 * r + v) * 8 + j] != ord[j];
            }
            printf("\"topk_variant_%s\": %.0f, \"topk_variant_%s_mismatches\": %d, ", vn[v], median(tv), vn[v], badv);
        }
        CK(cudaFree(d_iv));
    }

    CK(cudaFuncSetAttribute(bulk_issue, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024));
    for (int mode = 0; mode < 2; mode++) {
        for (int n : {1, 4, 8}) {
            bulk_issue<<<1, 512, 128 * 1024>>>(d_src, n, 8192, mode, d_out, d_st);
            CK(cudaDeviceSynchronize());
            CK(cudaMemcpy(o.data(), d_out, 16 * 8, cudaMemcpyDeviceToHost));
            std::vector<double> iss, land;
            for (int r = 1; r < 8; r++) {
                iss.push_back((double)o[2 * r]);
                land.push_back((double)o[2 * r + 1]);
            }
            printf("\"bulk_%s_%d_issue\": %.0f, \"bulk_%s_%d_landed\": %.0f, ", mode ? "warps" : "lane", n, median(iss),
                   mode ? "warps" : "lane", n, median(land));
        }
    }
    int st = 0;
    CK(cudaMemcpy(&st, d_st, 4, cudaMemcpyDeviceToHost));
    int clk = 0;
    cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, 0);
    printf("\"status\": %d, \"clock_khz\": %d}\n", st, clk);
    return 0;
}
