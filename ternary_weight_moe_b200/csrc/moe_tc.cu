// moe_tc.cu -- the grouped gate/up and down stages for >= 32 tokens per step on the fifth
// generation tensor cores (tcgen05.mma kind::i8, accumulators in tensor memory), sm_100a.
//
// At 32 or more tokens the selected experts each serve a few tokens ("iPhone Runs a 20B Model at
// 120 tok/s", "What Makes 120 tok/s So Fast?": batched work turns the matrix-vector products of
// decode into small matrix products), so every expert's rows are decoded once and multiplied
// against all of its tokens at once:
//   * one CTA of 128 threads per (distinct expert, 128 rows); per K-tile of 128 codes each thread
//     decodes one row's 32 packed bytes into int8 weights (a byte permutation of a four-entry
//     table, no memory lookup) and writes them into shared memory in the tensor core's K-major
//     layout; the staged activation limbs of up to 16 tokens (the expert's entries) go beside
//     them;
//   * one thread issues the MMAs, one accumulator per (matrix, limb) in tensor memory: A = the
//     weights (signed int8), B = a limb (hi: signed, mid and lo: unsigned), M = 128, N = 16,
//     K = 32 per instruction; tcgen05.commit signals an mbarrier per buffer, so the next tile is
//     decoded into the other buffer while the tensor core works;
//   * the epilogue reads the accumulators with tcgen05.ld (thread = row) and recombines the
//     limbs exactly in int64, S = hi * 65536 + mid * 256 + lo: the same integers as the dp4a and
//     mma.sync kernels, so the outputs are identical.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

namespace tern {

constexpr int kTcM = 128;        // rows per CTA (the MMA's M)
constexpr int kTcN = 16;         // tokens per pass (the MMA's N)
constexpr int kTcKT = 64;        // codes per K-tile (bytes of int8): 38 KB of shared memory per CTA
constexpr int kTcKW = kTcKT / 64; // 16-byte packed words per row and tile
constexpr int kTcBChunks = kTcN * (kTcKT / 16);  // 16-byte limb chunks per limb and tile
constexpr int kTcThreads = 128;  // warp w reads accumulator lanes 32w .. 32w + 31
constexpr int kTcABytes = kTcM * kTcKT;
constexpr int kTcBBytes = kTcN * kTcKT;
constexpr long long kTcWaitNs = 1000000000ll;

// K-major operand without swizzle: 8 rows x 16 bytes make a contiguous 128-byte core matrix,
// core matrices K-chunk-minor: byte `b` of row `r` of a tile is at
// ((r / 8) * (KT / 16) + b / 16) * 128 + (r % 8) * 16 + b % 16.  The MMA over bytes 32s .. 32s + 31
// starts at 2s * 128; the next 16 bytes of K are 128 bytes on (leading byte offset), the next 8
// rows (KT / 16) * 128 bytes on (stride byte offset).
__device__ __forceinline__ uint32_t tc_off(int r, int b) {
    return (uint32_t)((((r >> 3) * (kTcKT / 16) + (b >> 4)) << 7) + ((r & 7) << 4) + (b & 15));
}

// shared-memory matrix descriptor: start >> 4 in bits 0-13, leading byte offset >> 4 in bits
// 16-29, stride byte offset >> 4 in bits 32-45, version 1 in bits 46-47, base offset 0, layout
// type 0 (no swizzle) in bits 61-63
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    const uint64_t lbo = 128u, sbo = (uint64_t)(kTcKT / 16) * 128u;
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFull) << 16) | (((sbo >> 4) & 0x3FFFull) << 32) |
           (1ull << 46);
}

// instruction descriptor: s32 accumulators (bits 4-5 = 2), A signed 8-bit (bits 7-9 = 1), B
// signed (1) or unsigned (0) 8-bit (bits 10-12), both K-major (bits 15, 16 = 0), N / 8 in bits
// 17-22, M / 16 in bits 24-28
__device__ __forceinline__ uint32_t tc_idesc(bool b_signed) {
    return (2u << 4) | (1u << 7) | ((b_signed ? 1u : 0u) << 10) | ((uint32_t)(kTcN >> 3) << 17) |
           ((uint32_t)(kTcM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(dtmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_alloc(uint32_t *dst, uint32_t ncols) {  // one full warp
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {  // the same warp
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// The 16 int8 weights of a packed word w (codes 0..15, two bits each: 00 = 0, 01 = +1, 10 = -1,
// 11 reads as 0) as four words of four int8, codes in order: each 2-bit code selects a byte of the
// table {0, +1, -1, 0} through __byte_perm (its selector nibbles are the codes).
__device__ __forceinline__ uint4 tc_decode_word(uint32_t w) {
    const uint32_t T = 0x00FF0100u;  // byte c = the weight of code c
    uint32_t lo = w & 0xFFFFu, hi = w >> 16;
    lo = (lo | (lo << 8)) & 0x00FF00FFu;
    hi = (hi | (hi << 8)) & 0x00FF00FFu;
    lo = (lo | (lo << 4)) & 0x0F0F0F0Fu;
    hi = (hi | (hi << 4)) & 0x0F0F0F0Fu;
    lo = (lo | (lo << 2)) & 0x33333333u;  // code j of the low half in nibble j
    hi = (hi | (hi << 2)) & 0x33333333u;
    return make_uint4(__byte_perm(T, 0u, lo), __byte_perm(T, 0u, lo >> 16), __byte_perm(T, 0u, hi),
                      __byte_perm(T, 0u, hi >> 16));
}

// One K-tile's global data for this thread, loaded one tile ahead of its use: the 32 packed bytes
// of row `threadIdx.x` of each matrix, and NL chunks of 16 limb bytes (chunk i = threadIdx.x +
// j * threads: limb l, token row n, 16-byte chunk c of the tile).
constexpr int kTcBPerThread(int NL) { return (NL * kTcBChunks + kTcThreads - 1) / kTcThreads; }

template <int NM, int NL>
struct TcTile {
    uint4 a[NM][kTcKW];
    uint4 b[kTcBPerThread(NL)];
};

template <int NM, int NL>
__device__ __forceinline__ void tc_load(TcTile<NM, NL> &p, const uint8_t *const (&mats)[NM], int64_t rowb, int nrows,
                                        const uint32_t *__restrict__ src, int K4, const int32_t *__restrict__ ent,
                                        int q0, int nb, int div, int t) {
    const int r = threadIdx.x;
#pragma unroll
    for (int m = 0; m < NM; m++) {
        const uint4 *q = reinterpret_cast<const uint4 *>(mats[m] + (int64_t)r * rowb + (int64_t)t * (kTcKT / 4));
#pragma unroll
        for (int w = 0; w < kTcKW; w++) p.a[m][w] = r < nrows ? __ldg(q + w) : make_uint4(0u, 0u, 0u, 0u);
    }
    // chunk i: token row n = i % kTcN (fastest: 8 consecutive threads fill one 128-byte row of
    // core matrices without a bank conflict), 16-byte chunk c, limb l
#pragma unroll
    for (int j = 0; j < kTcBPerThread(NL); j++) {
        const int i = threadIdx.x + j * kTcThreads;
        const int n = i % kTcN, c = (i / kTcN) % (kTcKT / 16), l = i / kTcBChunks;
        p.b[j] = make_uint4(0u, 0u, 0u, 0u);
        if (l < NL && n < nb) {
            const int64_t vec = ent[q0 + n] / div;
            p.b[j] = __ldg(reinterpret_cast<const uint4 *>(src + (vec * NL + l) * K4 + (int64_t)t * (kTcKT / 4)) + c);
        }
    }
}

// the tile into shared memory: weights decoded into A (K-major layout), limbs into B
template <int NM, int NL>
__device__ __forceinline__ void tc_store(const TcTile<NM, NL> &p, unsigned char *A, unsigned char *B) {
    const int r = threadIdx.x;
#pragma unroll
    for (int m = 0; m < NM; m++) {
#pragma unroll
        for (int w = 0; w < kTcKW; w++) {
            const uint32_t pw[4] = {p.a[m][w].x, p.a[m][w].y, p.a[m][w].z, p.a[m][w].w};
#pragma unroll
            for (int c = 0; c < 4; c++)  // 16 codes per packed word = one 16-byte chunk of the tile
                *reinterpret_cast<uint4 *>(A + (size_t)m * kTcABytes + tc_off(r, 16 * (4 * w + c))) =
                    tc_decode_word(pw[c]);
        }
    }
#pragma unroll
    for (int j = 0; j < kTcBPerThread(NL); j++) {
        const int i = threadIdx.x + j * kTcThreads;
        const int n = i % kTcN, c = (i / kTcN) % (kTcKT / 16), l = i / kTcBChunks;
        if (l < NL) *reinterpret_cast<uint4 *>(B + (size_t)l * kTcBBytes + tc_off(n, 16 * c)) = p.b[j];
    }
}

// The K loop of one token pass: NM matrices x NL limbs accumulate into tensor-memory columns
// (m * NL + l) * kTcN .. + kTcN.  `it` counts tiles across passes (buffer it & 1; mbarrier b
// completes once per tile issued on it).  Tile t + 1's global loads are in flight while tile t is
// decoded, stored and multiplied.  Returns false on a timed-out wait.
template <int NM, int NL>
__device__ __forceinline__ bool tc_pass(unsigned char *A, unsigned char *B, uint64_t *mb, uint32_t tmem,
                                        const uint8_t *const (&mats)[NM], int64_t rowb, int nrows, int ntile,
                                        const uint32_t *__restrict__ src, int K4, const int32_t *__restrict__ ent,
                                        int q0, int nb, int div, unsigned &it, int *status) {
    TcTile<NM, NL> cur, nxt;
    tc_load<NM, NL>(nxt, mats, rowb, nrows, src, K4, ent, q0, nb, div, 0);
    for (int t = 0; t < ntile; t++, it++) {
        cur = nxt;
        if (t + 1 < ntile) tc_load<NM, NL>(nxt, mats, rowb, nrows, src, K4, ent, q0, nb, div, t + 1);
        const int b = (int)(it & 1u);
        // the buffer's previous tile (two tiles back) must be consumed by the tensor core
        if (it >= 2 && !mbar_wait(&mb[b], ((it - 2) >> 1) & 1u, kTcWaitNs, status)) return false;
        unsigned char *Ab = A + (size_t)b * NM * kTcABytes;
        unsigned char *Bb = B + (size_t)b * NL * kTcBBytes;
        tc_store<NM, NL>(cur, Ab, Bb);
        fence_async_smem();  // the generic-proxy writes above, visible to the tensor core
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < kTcKT / 32; s++)
#pragma unroll
                for (int m = 0; m < NM; m++)
#pragma unroll
                    for (int l = 0; l < NL; l++)
                        tc_mma(tmem + (uint32_t)((m * NL + l) * kTcN),
                               tc_desc(smem_u32(Ab + (size_t)m * kTcABytes + s * 256)),
                               tc_desc(smem_u32(Bb + (size_t)l * kTcBBytes + s * 256)), tc_idesc(l == 0),
                               (t > 0 || s > 0) ? 1u : 0u);
            tc_commit(&mb[b]);
        }
    }
    // every MMA of the pass done (the last commit covers all earlier ones)
    const unsigned last = it - 1;
    if (!mbar_wait(&mb[last & 1u], (last >> 1) & 1u, kTcWaitNs, status)) return false;
    tc_fence_after();
    return true;
}

// grid: (distinct experts bound, f / 128); 128 rows of gate and up per CTA
template <int NL>
__global__ void __launch_bounds__(kTcThreads) gateup_tc_kernel(
    const uint8_t *__restrict__ gate, const uint8_t *__restrict__ up, const float *__restrict__ sg,
    const float *__restrict__ su, int d, int f, int k, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ xw, const float *__restrict__ xsc, float *__restrict__ h,
    int32_t *__restrict__ acc_g, int32_t *__restrict__ acc_u, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb[2];
    __shared__ uint32_t s_tmem;
    const int u = blockIdx.x;
    if (u >= *n_unique) return;  // before any tensor memory is held
    constexpr int NCOL = 2 * NL * kTcN;
    constexpr uint32_t ALLOC = NCOL <= 32 ? 32u : (NCOL <= 64 ? 64u : 128u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int row0 = blockIdx.y * kTcM, nrows = min(kTcM, f - row0);
    const int64_t rowb = d / 4;
    const uint8_t *const mats[2] = {gate + ((int64_t)e * f + row0) * rowb, up + ((int64_t)e * f + row0) * rowb};
    unsigned char *A = smem;                                // [2 buffers][2 matrices][kTcABytes]
    unsigned char *B = smem + 2 * 2 * kTcABytes;            // [2 buffers][NL][kTcBBytes]
    if (tid == 0) {
        mbar_init(&mb[0], 1);
        mbar_init(&mb[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) tc_alloc(&s_tmem, ALLOC);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    unsigned it = 0;
    bool ok = true;
    for (int q0 = e0; q0 < e1 && ok; q0 += kTcN) {
        const int nb = min(kTcN, e1 - q0);
        ok = tc_pass<2, NL>(A, B, mb, tmem, mats, rowb, nrows, d / kTcKT, xw, d / 4, ent, q0, nb, k, it, status);
        if (!ok) break;
        // thread = row of this tile; the accumulators of token n are column n of each block
        const int j = row0 + tid;
        const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
        long long Sg[kTcN], Su[kTcN];
#pragma unroll
        for (int n = 0; n < kTcN; n++) Sg[n] = Su[n] = 0;
#pragma unroll
        for (int l = 0; l < NL; l++) {
            const long long wgt = (NL == 1) ? 1ll : (l == 0 ? 65536ll : (l == 1 ? 256ll : 1ll));
            uint32_t vg[16], vu[16];
            tc_ld16(ta + (uint32_t)((0 * NL + l) * kTcN), vg);
            tc_ld16(ta + (uint32_t)((1 * NL + l) * kTcN), vu);
            tc_wait_ld();
#pragma unroll
            for (int n = 0; n < kTcN; n++) {
                Sg[n] += (long long)(int32_t)vg[n] * wgt;
                Su[n] += (long long)(int32_t)vu[n] * wgt;
            }
        }
        if (j < f) {
            const int64_t o = (int64_t)e * f + j;
            const float sgv = sg[o], suv = su[o];
#pragma unroll
            for (int n = 0; n < kTcN; n++) {
                if (n >= nb) continue;
                const int entry = ent[q0 + n];
                const float xsv = xsc[entry / k];
                float hv;
                if (NL == 1) {
                    acc_g[(int64_t)entry * f + j] = (int32_t)Sg[n];
                    acc_u[(int64_t)entry * f + j] = (int32_t)Su[n];
                    const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg[n]), sgv), xsv);
                    const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su[n]), suv), xsv);
                    hv = swiglu_f32((double)gv, (double)uv);
                } else {
                    const int sh = __float_as_int(xsv);
                    hv = swiglu_f32(ldexp((double)Sg[n], -sh) * (double)sgv, ldexp((double)Su[n], -sh) * (double)suv);
                }
                h[(int64_t)entry * f + j] = hv;
            }
        }
        // every thread's reads of the accumulators are done before the next pass overwrites them
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tc_dealloc(tmem, ALLOC);
}

// grid: (distinct experts bound, d / 128); 128 output rows per CTA
template <int NL>
__global__ void __launch_bounds__(kTcThreads) down_tc_kernel(
    const uint8_t *__restrict__ down, const float *__restrict__ sd, int d, int f, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ hw, const float *__restrict__ hsc, double *__restrict__ ye,
    int32_t *__restrict__ acc_d, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb[2];
    __shared__ uint32_t s_tmem;
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    constexpr int NCOL = NL * kTcN;
    constexpr uint32_t ALLOC = NCOL <= 32 ? 32u : (NCOL <= 64 ? 64u : 128u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int row0 = blockIdx.y * kTcM, nrows = min(kTcM, d - row0);
    const int64_t rowb = f / 4;
    const uint8_t *const mats[1] = {down + ((int64_t)e * d + row0) * rowb};
    unsigned char *A = smem;                            // [2 buffers][kTcABytes]
    unsigned char *B = smem + 2 * kTcABytes;            // [2 buffers][NL][kTcBBytes]
    if (tid == 0) {
        mbar_init(&mb[0], 1);
        mbar_init(&mb[1], 1);
        fence_mbar_init();
    }
    if (warp == 0) tc_alloc(&s_tmem, ALLOC);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    unsigned it = 0;
    bool ok = true;
    for (int q0 = e0; q0 < e1 && ok; q0 += kTcN) {
        const int nb = min(kTcN, e1 - q0);
        ok = tc_pass<1, NL>(A, B, mb, tmem, mats, rowb, nrows, f / kTcKT, hw, f / 4, ent, q0, nb, 1, it, status);
        if (!ok) break;
        const int i = row0 + tid;
        const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
        long long S[kTcN];
#pragma unroll
        for (int n = 0; n < kTcN; n++) S[n] = 0;
#pragma unroll
        for (int l = 0; l < NL; l++) {
            const long long wgt = (NL == 1) ? 1ll : (l == 0 ? 65536ll : (l == 1 ? 256ll : 1ll));
            uint32_t v[16];
            tc_ld16(ta + (uint32_t)(l * kTcN), v);
            tc_wait_ld();
#pragma unroll
            for (int n = 0; n < kTcN; n++) S[n] += (long long)(int32_t)v[n] * wgt;
        }
        if (i < d) {
            const float sdv = sd[(int64_t)e * d + i];
#pragma unroll
            for (int n = 0; n < kTcN; n++) {
                if (n >= nb) continue;
                const int entry = ent[q0 + n];
                const float hs = hsc[entry];
                double v;
                if (NL == 1) {
                    acc_d[(int64_t)entry * d + i] = (int32_t)S[n];
                    v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S[n]), sdv), hs);
                } else {
                    v = ldexp((double)S[n], -__float_as_int(hs)) * (double)sdv;
                }
                ye[(int64_t)entry * d + i] = v;
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tc_dealloc(tmem, ALLOC);
}

bool tc_grouped_supported(int d, int f) { return d % kTcKT == 0 && f % kTcKT == 0; }

template <int NL>
cudaError_t launch_grouped_tc(const tern_moe_layer *L, int T, const FfnWs &w, cudaStream_t s, int phase) {
    const int d = (int)L->d, f = (int)L->f, E = L->E, k = L->k;
    const int umax = (E < T * k) ? E : T * k;
    int *st = status_word();
    if (phase == 0) {
        const size_t sm = (size_t)2 * 2 * kTcABytes + (size_t)2 * NL * kTcBBytes;
        cudaFuncSetAttribute(gateup_tc_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        gateup_tc_kernel<NL><<<dim3(umax, (f + kTcM - 1) / kTcM), kTcThreads, sm, s>>>(
            L->gate, L->up, L->gate_scale, L->up_scale, d, f, k, w.n_unique, w.uexp, w.uoff, w.ent,
            (const uint32_t *)w.xw, (const float *)w.xsc, w.h, w.acc_g, w.acc_u, st);
    } else {
        const size_t sm = (size_t)2 * kTcABytes + (size_t)2 * NL * kTcBBytes;
        cudaFuncSetAttribute(down_tc_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        down_tc_kernel<NL><<<dim3(umax, (d + kTcM - 1) / kTcM), kTcThreads, sm, s>>>(
            L->down, L->down_scale, d, f, w.n_unique, w.uexp, w.uoff, w.ent, (const uint32_t *)w.hw,
            (const float *)w.hsc, w.ye, w.acc_d, st);
    }
    return cudaGetLastError();
}

template cudaError_t launch_grouped_tc<1>(const tern_moe_layer *, int, const FfnWs &, cudaStream_t, int);
template cudaError_t launch_grouped_tc<3>(const tern_moe_layer *, int, const FfnWs &, cudaStream_t, int);

}  // namespace tern
