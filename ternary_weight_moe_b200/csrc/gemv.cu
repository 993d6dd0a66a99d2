// gemv.cu -- packing, absmax quantisation and the ternary GEMV (sm_100a).
//
// Ternary GEMV ("A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac
// Mini", "What Ternary Actually Means": batch-1 decode is a sequence of matrix-vector
// products; multiplying by -1, 0, +1 needs no multiply).  Memory layout and mapping:
//   - a row of K codes is K/4 bytes = K/64 segments of 16 bytes; G = min(32, K/64) lanes
//     cover one row slice of <= 2048 codes with one coalesced 128-bit load each;
//   - each lane keeps the activation limbs of ITS segment in registers for the whole kernel,
//     so activations are read once per CTA, never per row;
//   - K > 2048 is split across the warps of a CTA (split-K) and combined in shared memory
//     in a fixed order;
//   - large calls: every byte of weights is decoded with one table read and consumed by one
//     dp4a per limb (ring kernel); small one-token calls: decoded without a table (lean kernel).
#include <cuda_runtime.h>

#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

namespace tern {

// ------------------------------------------------------------------------ pack / unpack
__global__ void pack_kernel(const int8_t *__restrict__ w, int64_t M, int64_t K, uint8_t *__restrict__ out,
                            unsigned long long *bad) {
    const int64_t nb = M * (K / 4);
    unsigned long long nbad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nb; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / (K / 4), b = i % (K / 4);
        const int8_t *src = w + m * K + 4 * b;
        uint32_t byte = 0;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int v = src[j];
            uint32_t c = 0;
            if (v == 1) c = 1;
            else if (v == -1) c = 2;
            else if (v != 0) nbad++;
            byte |= c << (2 * j);
        }
        out[i] = (uint8_t)byte;
    }
    if (nbad) atomicAdd(bad, nbad);
}

__global__ void unpack_kernel(const uint8_t *__restrict__ p, int64_t M, int64_t K, int8_t *__restrict__ w,
                              unsigned long long *bad) {
    const int64_t nb = M * (K / 4);
    unsigned long long nbad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nb; i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t byte = p[i];
        const int64_t m = i / (K / 4), b = i % (K / 4);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t c = (byte >> (2 * j)) & 3u;
            if (c == 3u) nbad++;
            w[m * K + 4 * b + j] = (int8_t)(c == 1u ? 1 : (c == 2u ? -1 : 0));
        }
    }
    if (nbad) atomicAdd(bad, nbad);
}

static int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    if (g > 148 * 16) g = 148 * 16;
    return (int)(g < 1 ? 1 : g);
}

cudaError_t launch_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, unsigned long long *bad,
                        cudaStream_t s) {
    pack_kernel<<<grid_for(M * K / 4, 256), 256, 0, s>>>(w, M, K, packed, bad);
    return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t *p, int64_t M, int64_t K, int8_t *w, unsigned long long *bad,
                          cudaStream_t s) {
    unpack_kernel<<<grid_for(M * K / 4, 256), 256, 0, s>>>(p, M, K, w, bad);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- absmax quantisation
__global__ void quant_kernel(const uint16_t *__restrict__ x, int64_t n, int8_t *__restrict__ q,
                             float *__restrict__ sc) {
    __shared__ float red[32];
    const uint16_t *xr = x + blockIdx.x * n;
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, fabsf(bf16_to_f32(xr[i])));
    const float amax = block_max_f32(m, red);
    int8_t *qr = q + blockIdx.x * n;
    if (amax == 0.0f) {
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) qr[i] = 0;
        if (threadIdx.x == 0) sc[blockIdx.x] = 0.0f;
        return;
    }
    const float inv = quant_inv(amax);
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) qr[i] = (int8_t)quant_one(bf16_to_f32(xr[i]), inv);
    if (threadIdx.x == 0) sc[blockIdx.x] = __fdiv_rn(amax, 127.0f);
}

cudaError_t launch_quant_absmax(const uint16_t *x, int64_t T, int64_t n, int8_t *q, float *sc, cudaStream_t s) {
    quant_kernel<<<(unsigned)T, 256, 0, s>>>(x, n, q, sc);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------ ternary GEMV
// The 64 int8 activations of segment `seg` (64 codes) of token vector xt as 16 words.
__device__ __forceinline__ void gemv_load_x(SegX<1> &X, const int8_t *xt, int seg) {
    const uint4 *p = reinterpret_cast<const uint4 *>(xt + (int64_t)seg * 64);
#pragma unroll
    for (int v = 0; v < 4; v++) {
        const uint4 t = __ldg(p + v);
        X.w[0][4 * v + 0] = t.x;
        X.w[0][4 * v + 1] = t.y;
        X.w[0][4 * v + 2] = t.z;
        X.w[0][4 * v + 3] = t.w;
    }
}

// ------------------------------------------------------------ the TMA-fed GEMV kernel
// One CTA per SM.  A producer warp streams chunks of R consecutive rows (R*K/4 contiguous
// bytes, up to 32 KB) plus their row scales into a ring of kGvStages shared-memory stages
// with bulk copies; 16 consumer warps decode each stage as it lands and release it through
// an mbarrier, so about 96 KB of weights per SM stay in flight while the consumers compute.
// Waiting warps sleep inside mbarrier.try_wait instead of spinning.
//   K <= 2048: G = K/64 lanes per row, 32/G rows per warp pass; every warp takes two passes
//              at a time (two independent dot chains) and reduces both with one shuffle tree;
//   K  > 2048: NS = K/2048 slices of 512 bytes; warp w takes slice w % NS of rows
//              w / NS, w / NS + 16/NS, ...; each slice's exact integer partial goes to shared
//              memory and the producer warp sums the NS partials of a row (fixed order) and
//              writes it before it refills the stage.
// bf16 activations: the 24-bit fixed-point limbs of the token are built once per CTA in
// shared memory; each lane then keeps its segment's limbs in registers.
constexpr int kGvCons = 16;  // consumer warps
constexpr int kGvConsThreads = kGvCons * 32;
constexpr int kGvThreads = kGvConsThreads + 32;
constexpr int kGvStages = 3;
constexpr int kGvStageBytes = 32768;
constexpr int kGvMaxRows = 256;      // rows per chunk (scale ring entries per stage)
constexpr int kGvMaxSplitRows = 32;  // rows per chunk when K > 2048 (32 KB / 1 KB)
constexpr int kGvMaxSlices = 8;
constexpr int kGvMaxK = 16384;
constexpr int kGvMaxT = 64;
constexpr long long kGvWaitNs = 1000000000ll;

struct GvSmem {
    uint32_t lut, ring, rs, part, xl, total;
};
__host__ __device__ constexpr GvSmem gv_smem() {
    return GvSmem{0u,
                  (uint32_t)kLutBytes,
                  (uint32_t)(kLutBytes + kGvStages * kGvStageBytes),
                  (uint32_t)(kLutBytes + kGvStages * kGvStageBytes + kGvStages * kGvMaxRows * 4),
                  (uint32_t)(kLutBytes + kGvStages * kGvStageBytes + kGvStages * kGvMaxRows * 4 +
                             kGvStages * kGvMaxSplitRows * kGvMaxSlices * 8),
                  (uint32_t)(kLutBytes + kGvStages * kGvStageBytes + kGvStages * kGvMaxRows * 4 +
                             kGvStages * kGvMaxSplitRows * kGvMaxSlices * 8 + 3 * (kGvMaxK / 4) * 4)};
}

template <int NL, int G>
__global__ void __launch_bounds__(kGvThreads, 1)
    gemv_kernel(const uint8_t *__restrict__ Wp, const float *__restrict__ rs, int M, int K, int NS, int R,
                int nchunks, const void *__restrict__ x, const float *__restrict__ xs, int T,
                int32_t *__restrict__ acc_out, float *__restrict__ y, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kGvStages], empty[kGvStages];
    __shared__ float red[32];
    __shared__ int s_shift[kGvMaxT];
    constexpr GvSmem L = gv_smem();
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem + L.lut);
    unsigned char *ring = smem + L.ring;
    float *s_rs = reinterpret_cast<float *>(smem + L.rs);           // [S][kGvMaxRows]
    long long *s_part = reinterpret_cast<long long *>(smem + L.part);  // [S][16][8]
    uint32_t *xl = reinterpret_cast<uint32_t *>(smem + L.xl);       // [NL][K/4] limb words

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int RB = K / 4;
    const int my_n = (nchunks - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;  // chunks per token
    const int total = my_n * T;
    const bool rs_bulk = ((uintptr_t)rs % 16u) == 0;
    // chunk n of this CTA (n counts over tokens too): rows [r0, r0 + nr)
    auto chunk_rows = [&](int n, int &r0, int &nr) {
        r0 = ((int)blockIdx.x + (n % my_n) * (int)gridDim.x) * R;
        nr = min(R, M - r0);
    };
    auto issue = [&](int n) {
        const int st = n % kGvStages;
        int r0, nr;
        chunk_rows(n, r0, nr);
        const uint32_t wbytes = (uint32_t)nr * (uint32_t)RB;
        const uint32_t sbytes = rs_bulk ? (uint32_t)(nr / 4) * 16u : 0u;
        mbar_expect_tx(&full[st], wbytes + sbytes);
        bulk_g2s(ring + (size_t)st * kGvStageBytes, Wp + (size_t)r0 * RB, wbytes, &full[st]);
        if (sbytes) bulk_g2s(s_rs + st * kGvMaxRows, rs + r0, sbytes, &full[st]);
    };
    // y for row r0 + row of token t from its exact integer sum S
    auto finish = [&](int t, int r0, int nr, int st, int row, long long S) {
        const float sc = (rs_bulk && row < (nr & ~3)) ? s_rs[st * kGvMaxRows + row] : __ldg(rs + r0 + row);
        const int64_t o = (int64_t)t * M + r0 + row;
        if (NL == 1) {
            if (acc_out) acc_out[o] = (int32_t)S;
            float v = __fmul_rn(__int2float_rn((int)S), sc);
            if (xs != nullptr) v = __fmul_rn(v, xs[t]);
            y[o] = v;
        } else {
            y[o] = (float)(ldexp((double)S, -s_shift[t]) * (double)sc);
        }
    };

    int issued = 0;
    if (tid == kGvConsThreads) {
        for (int q = 0; q < kGvStages; q++) {
            mbar_init(&full[q], 1);
            mbar_init(&empty[q], kGvCons);
        }
        fence_mbar_init();
        // the first stages need no release: start them before the table is built
        for (; issued < kGvStages && issued < total; issued++) issue(issued);
    }
    lut_fill(lut);
    __syncthreads();

    if (warp == kGvCons) {  // ------------------------------------------------ producer
        bool ok = true;
        // iteration n: stage n % S is free again once chunk n - S is consumed; for K > 2048
        // that chunk's rows are summed and written here, then chunk n is issued
        for (int n = kGvStages; ok && n < total + kGvStages; n++) {
            const int st = n % kGvStages;
            ok = mbar_wait_sleep(&empty[st], (uint32_t)((n / kGvStages) - 1) & 1u, kGvWaitNs, status);
            if (!ok) break;
            if (NS > 1) {
                const int m = n - kGvStages;
                int r0, nr;
                chunk_rows(m, r0, nr);
                if (lane < nr) {
                    long long S = 0;
                    for (int sl = 0; sl < NS; sl++) S += s_part[(st * kGvMaxSplitRows + lane) * kGvMaxSlices + sl];
                    finish(m / my_n, r0, nr, st, lane, S);
                }
                __syncwarp();
            }
            if (n < total && lane == 0) {
                issue(n);
                issued = n + 1;
            }
        }
        // on a timeout: leave only after every copy into this CTA's shared memory has landed
        if (!ok && lane == 0)
            for (int q = 0; q < kGvStages && q < issued; q++) {
                const int cnt = (issued - q + kGvStages - 1) / kGvStages;
                mbar_wait(&full[q], (uint32_t)(cnt - 1) & 1u, kGvWaitNs, status);
            }
        return;
    }

    // ---------------------------------------------------------------------- consumers
    constexpr int RPW = 32 / G;  // rows per warp pass (K <= 2048)
    const int sub = lane / G, gl = lane % G;
    const int slice = warp % NS, rg = warp / NS, ngroups = kGvCons / NS;
    const int seg = (NS > 1) ? slice * 32 + lane : gl;
    const uint32_t lane4 = (uint32_t)lane << 2;
    bool alive = true;
    int st = 0;        // stage of the next chunk
    uint32_t ph = 0u;  // its fill phase parity
    for (int t = 0; t < T; t++) {
        SegX<NL> X;
        if constexpr (NL == 1) {
            gemv_load_x(X, static_cast<const int8_t *>(x) + (int64_t)t * K, seg);
        } else {
            const uint16_t *xb = static_cast<const uint16_t *>(x) + (int64_t)t * K;
            float m = 0.0f;
            for (int i = tid; i < K; i += kGvConsThreads) m = fmaxf(m, fabsf(bf16_to_f32(xb[i])));
            m = warp_max_f32(m);
            if (lane == 0) red[warp] = m;
            named_bar_sync(1, kGvConsThreads);
            float amax = 0.0f;
#pragma unroll
            for (int w = 0; w < kGvCons; w++) amax = fmaxf(amax, red[w]);
            const int sh = fixed_shift(amax);
            if (tid == 0) s_shift[t] = sh;
            // limb words of four consecutive values, one word per limb, built once per CTA
            for (int wd = tid; wd < K / 4; wd += kGvConsThreads) {
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(xb) + wd);
                const uint32_t hw[2] = {v.x, v.y};
                uint32_t wl[3] = {0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const uint16_t bb = (uint16_t)((e & 1) ? (hw[e >> 1] >> 16) : (hw[e >> 1] & 0xFFFFu));
                    uint32_t h, mi, lo;
                    fixed_limbs(bf16_to_f32(bb), sh, h, mi, lo);
                    wl[0] |= h << (8 * e);
                    wl[1] |= mi << (8 * e);
                    wl[2] |= lo << (8 * e);
                }
                xl[wd] = wl[0];
                xl[K / 4 + wd] = wl[1];
                xl[2 * (K / 4) + wd] = wl[2];
            }
            named_bar_sync(1, kGvConsThreads);
            seg_load_x_smem<NL>(X, xl, K / 4, seg);
        }

        for (int j = 0; j < my_n; j++) {
            if (alive) alive = mbar_wait_sleep(&full[st], ph, kGvWaitNs, status);
            const int r0 = ((int)blockIdx.x + j * (int)gridDim.x) * R;
            const int nr = min(R, M - r0);
            const unsigned char *stage = ring + (size_t)st * kGvStageBytes;
            if (alive && NS == 1) {
                // passes p and p + 16 of this warp at once
                for (int p = warp; p * RPW < nr; p += 2 * kGvCons) {
                    const int rowA = p * RPW + sub, rowB = (p + kGvCons) * RPW + sub;
                    const bool vA = rowA < nr, vB = rowB < nr;
                    const uint4 wA = vA ? *reinterpret_cast<const uint4 *>(stage + (size_t)rowA * RB + gl * 16)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    const uint4 wB = vB ? *reinterpret_cast<const uint4 *>(stage + (size_t)rowB * RB + gl * 16)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    int accA[NL], accB[NL];
#pragma unroll
                    for (int l = 0; l < NL; l++) accA[l] = accB[l] = 0;
                    seg_dot<NL>(wA, X, lut, lane4, accA);
                    seg_dot<NL>(wB, X, lut, lane4, accB);
                    int aA, bA, aB, bB;
                    acc_to_pair<NL>(accA, aA, bA);
                    acc_to_pair<NL>(accB, aB, bB);
                    if (G == 1) {
                        if (vA) finish(t, r0, nr, st, rowA, pair_value(NL, aA, bA));
                        if (vB) finish(t, r0, nr, st, rowB, pair_value(NL, aB, bB));
                    } else {
                        const int a = group_sum2<(G > 1 ? G : 2)>(aA, aB);
                        const int b = (NL > 1) ? group_sum2<(G > 1 ? G : 2)>(bA, bB) : 0;
                        if (gl == 0 && vA) finish(t, r0, nr, st, rowA, pair_value(NL, a, b));
                        if (gl == G / 2 && vB) finish(t, r0, nr, st, rowB, pair_value(NL, a, b));
                    }
                }
            } else if (alive && rg < ngroups) {
                for (int rowA = rg; rowA < nr; rowA += 2 * ngroups) {
                    const int rowB = rowA + ngroups;
                    const bool vB = rowB < nr;
                    const uint4 wA = *reinterpret_cast<const uint4 *>(stage + (size_t)rowA * RB + slice * 512 + lane * 16);
                    const uint4 wB = vB ? *reinterpret_cast<const uint4 *>(stage + (size_t)rowB * RB + slice * 512 +
                                                                             lane * 16)
                                        : make_uint4(0u, 0u, 0u, 0u);
                    int accA[NL], accB[NL];
#pragma unroll
                    for (int l = 0; l < NL; l++) accA[l] = accB[l] = 0;
                    seg_dot<NL>(wA, X, lut, lane4, accA);
                    seg_dot<NL>(wB, X, lut, lane4, accB);
                    int aA, bA, aB, bB;
                    acc_to_pair<NL>(accA, aA, bA);
                    acc_to_pair<NL>(accB, aB, bB);
                    const int a = group_sum2<32>(aA, aB);
                    const int b = (NL > 1) ? group_sum2<32>(bA, bB) : 0;
                    if (lane == 0) s_part[(st * kGvMaxSplitRows + rowA) * kGvMaxSlices + slice] = pair_value(NL, a, b);
                    if (lane == 16 && vB)
                        s_part[(st * kGvMaxSplitRows + rowB) * kGvMaxSlices + slice] = pair_value(NL, a, b);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            if (++st == kGvStages) {
                st = 0;
                ph ^= 1u;
            }
        }
        if (NL > 1) named_bar_sync(1, kGvConsThreads);  // red[] and xl[] are rewritten by the next token
    }
}

// ------------------------------------------------------------ the lean GEMV (small calls)
// For one token and a few MB of weights the ring kernel's fixed costs dominate: a 64 KB
// decode-table fill per CTA, a producer warp, and for bf16 two passes over x before the
// first dot.  This kernel has none of them:
//   - the weights are decoded without a table (decode.cuh);
//   - every warp first puts the loads of all its rows' segments in flight (<= kLnMaxIter per
//     lane, ld.global.nc), so their HBM latency overlaps the work on x;
//   - the activations go to each lane in position-major order (word 4q + j of a limb holds
//     the activations of position j of packed word q: 16q + j, 16q + 4 + j, 16q + 8 + j,
//     16q + 12 + j): int8 by a byte transpose of the lane's own 64 values; bf16 limbs are
//     built once per CTA in shared memory (four values per thread, after a CTA-wide absmax)
//     and each lane loads its segment's;
//   - K <= 2048: G = K/64 lanes per row, 32/G rows per warp pass; K > 2048: NS = K/2048
//     slices, warp w takes slice w % NS of rows w / NS, w / NS + 16/NS, ...; the exact slice
//     partials meet in shared memory and are added in slice order.
// The integers are the ring kernel's, so y is identical.
constexpr int kLnWarps = 16;
constexpr int kLnThreads = kLnWarps * 32;
constexpr int kLnMaxIter = 8;    // row segments per lane kept in flight
constexpr int kLnMaxRows = 256;  // rows per CTA when K > 2048 (slice partials in shared memory)
constexpr int kLnMaxSlices = 8;
constexpr int64_t kLnMaxBytes = 16ll << 20;
constexpr int kLnMaxXPass = 8;   // groups of four activations per thread (K <= 16384)

template <int NL, int G>
__global__ void __launch_bounds__(kLnThreads, 1)
    gemv_lean_kernel(const uint8_t *__restrict__ Wp, const float *__restrict__ rs, int M, int K, int NS, int Rc,
                     const void *__restrict__ x, const float *__restrict__ xs, int32_t *__restrict__ acc_out,
                     float *__restrict__ y) {
    __shared__ float s_red[kLnWarps];
    __shared__ long long s_part[kLnMaxRows * kLnMaxSlices];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int RB = K / 4;
    const int r0c = (int)blockIdx.x * Rc, nrc = min(Rc, M - r0c);  // this CTA's rows
    constexpr int RPW = 32 / G;                                     // rows per warp pass
    const int sub = lane / G, gl = lane % G;
    const int slice = (G == 32) ? warp % NS : 0;
    const int rg = (G == 32) ? warp / NS : 0, ngroups = (G == 32) ? kLnWarps / NS : 1;
    const int seg = (G == 32) ? slice * 32 + lane : gl;  // this lane's 64 codes
    auto row_of = [&](int i) { return (G == 32) ? rg + i * ngroups : (warp + i * kLnWarps) * RPW + sub; };

    // 1. this lane's segment of every row it will take, all loads in flight
    uint4 wv[kLnMaxIter];
#pragma unroll
    for (int i = 0; i < kLnMaxIter; i++) {
        const int r = row_of(i);
        wv[i] = r < nrc ? __ldg(reinterpret_cast<const uint4 *>(Wp + (size_t)(r0c + r) * RB) + seg)
                        : make_uint4(0u, 0u, 0u, 0u);
    }
    // scales of the rows this thread writes, early as well
    const bool split = (G == 32) && NS > 1;
    float scp[kLnMaxIter];
#pragma unroll
    for (int i = 0; i < kLnMaxIter; i++) {
        const int r = split ? tid + i * kLnThreads : row_of(i);
        scp[i] = (r < nrc && (split || gl == 0)) ? __ldg(rs + r0c + r) : 0.0f;
    }

    // 2. the activations of this lane's segment, as limbs in position-major order
    SegX<NL> X;
    int sh = 0;
    if constexpr (NL == 1) {
        const uint4 *xp = reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(x) + (size_t)seg * 64);
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const uint4 t = __ldg(xp + q);
            bytes_transpose4(t.x, t.y, t.z, t.w, X.w[0][4 * q], X.w[0][4 * q + 1], X.w[0][4 * q + 2], X.w[0][4 * q + 3]);
        }
    } else {
        // bf16: the CTA builds the limbs of x once, four values per thread and pass
        // (position-major, padded: store_limbs4), then each lane loads its segment's
        const uint16_t *xb = static_cast<const uint16_t *>(x);
        const int ng = K / 4, xlp = (K / 64) * kSegPad;
        uint2 xg[kLnMaxXPass];
        float am = 0.0f;
#pragma unroll
        for (int u = 0; u < kLnMaxXPass; u++) {
            const int g = tid + u * kLnThreads;
            xg[u] = g < ng ? __ldg(reinterpret_cast<const uint2 *>(xb) + g) : make_uint2(0u, 0u);
            am = fmaxf(am, fmaxf(fmaxf(fabsf(bf16_to_f32((uint16_t)(xg[u].x & 0xFFFFu))),
                                       fabsf(bf16_to_f32((uint16_t)(xg[u].x >> 16)))),
                                 fmaxf(fabsf(bf16_to_f32((uint16_t)(xg[u].y & 0xFFFFu))),
                                       fabsf(bf16_to_f32((uint16_t)(xg[u].y >> 16))))));
        }
        am = warp_max_f32(am);
        if (lane == 0) s_red[warp] = am;
        __syncthreads();
        float amax = 0.0f;
#pragma unroll
        for (int w = 0; w < kLnWarps; w++) amax = fmaxf(amax, s_red[w]);
        sh = fixed_shift(amax);
        extern __shared__ __align__(16) uint32_t ln_xl[];  // [3][K/64 segments][kSegPad words]
#pragma unroll
        for (int u = 0; u < kLnMaxXPass; u++) {
            const int g = tid + u * kLnThreads;
            if (g < ng) {
                const float v4[4] = {bf16_to_f32((uint16_t)(xg[u].x & 0xFFFFu)), bf16_to_f32((uint16_t)(xg[u].x >> 16)),
                                     bf16_to_f32((uint16_t)(xg[u].y & 0xFFFFu)), bf16_to_f32((uint16_t)(xg[u].y >> 16))};
                store_limbs4<NL>(ln_xl, xlp, g, v4, sh, 0.0f, true);
            }
        }
        __syncthreads();
        seg_load_x_padded<NL>(X, ln_xl, xlp, seg);
    }
    auto finish = [&](int r, float sc, long long S) {
        const int row = r0c + r;
        if (NL == 1) {
            if (acc_out) acc_out[row] = (int32_t)S;
            float v = __fmul_rn(__int2float_rn((int)S), sc);
            if (xs != nullptr) v = __fmul_rn(v, xs[0]);
            y[row] = v;
        } else {
            y[row] = (float)(ldexp((double)S, -sh) * (double)sc);
        }
    };

    // 3. the dots
#pragma unroll
    for (int i = 0; i < kLnMaxIter; i++) {
        const int r = row_of(i);
        if (!__any_sync(0xFFFFFFFFu, r < nrc)) break;
        int acc[NL];
#pragma unroll
        for (int z = 0; z < NL; z++) acc[z] = 0;
        seg_dot_alu<NL>(wv[i], X, acc);
        int a, b;
        acc_to_pair_x64<NL>(acc, a, b);
        a = group_sum<G>(a);
        if (NL > 1) b = group_sum<G>(b);
        if (r < nrc && gl == 0) {
            if (split) {
                if (lane == 0) s_part[r * kLnMaxSlices + slice] = pair_value(NL, a, b);
            } else {
                finish(r, scp[i], pair_value(NL, a, b));
            }
        }
    }
    if (split) {
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kLnMaxIter; i++) {
            const int r = tid + i * kLnThreads;
            if (r < nrc) {
                long long S = 0;
                for (int sl = 0; sl < NS; sl++) S += s_part[r * kLnMaxSlices + sl];
                finish(r, scp[i], S);
            }
        }
    }
}

static int device_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// The lean kernel's plan for one token: rows per CTA Rc over the SMs; false when the call is
// too large for it (more row segments per lane than kLnMaxIter, or more bytes than kLnMaxBytes)
static bool lean_plan(int64_t M, int64_t K, int64_t T, int sms, int &Rc, int &grid) {
    if (T != 1 || M * K / 4 > kLnMaxBytes) return false;
    const int NS = K > 2048 ? (int)(K / 2048) : 1;
    const int G = NS > 1 ? 32 : (int)(K / 64);
    if (NS > kLnMaxSlices || NS > kLnWarps) return false;
    Rc = (int)((M + sms - 1) / sms);
    grid = (int)((M + Rc - 1) / Rc);
    const int per_iter = G == 32 ? kLnWarps / NS : kLnWarps * (32 / G);  // rows per CTA per iteration
    if ((Rc + per_iter - 1) / per_iter > kLnMaxIter) return false;
    if (NS > 1 && (Rc > kLnMaxRows || Rc > kLnMaxIter * kLnThreads)) return false;
    return true;
}

template <int NL>
static cudaError_t gemv_dispatch(const uint8_t *Wp, const float *rs, int M, int K, const void *x,
                                 const float *xs, int T, int32_t *acc, float *y, cudaStream_t s) {
    const int RB = K / 4;
    const int NS = K > 2048 ? K / 2048 : 1;
    const int G = NS > 1 ? 32 : RB / 16;
    const int sms = device_sms();
    int Rl = 0, gl = 0;
    if (lean_plan(M, K, T, sms, Rl, gl)) {
        const int lsm = NL == 1 ? 0 : 3 * (K / 64) * kSegPad * 4;  // bf16 limbs of x
#define TERN_LEAN_CASE(GG)                                                                           \
    case GG:                                                                                         \
        if (lsm > 48 * 1024)                                                                         \
            cudaFuncSetAttribute(gemv_lean_kernel<NL, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, lsm); \
        gemv_lean_kernel<NL, GG><<<gl, kLnThreads, lsm, s>>>(Wp, rs, M, K, NS, Rl, x, xs, acc, y);   \
        break;
        switch (G) {
            TERN_LEAN_CASE(1)
            TERN_LEAN_CASE(2)
            TERN_LEAN_CASE(4)
            TERN_LEAN_CASE(8)
            TERN_LEAN_CASE(16)
            TERN_LEAN_CASE(32)
            default: return cudaErrorInvalidValue;
        }
#undef TERN_LEAN_CASE
        return cudaGetLastError();
    }
    // rows per chunk: a full stage, fewer when that would leave SMs without a chunk; always a
    // multiple of 4 so that every chunk's scales start on a 16-byte boundary
    int R = (kGvStageBytes / RB) & ~3;  // >= 4: RB <= 4096
    if (R > kGvMaxRows) R = kGvMaxRows;
    if ((M + R - 1) / R < sms) {
        int r = (M + sms - 1) / sms;
        r = (r + 3) & ~3;
        if (r < R) R = r;
    }
    const int nchunks = (M + R - 1) / R;
    const int grid = nchunks < sms ? nchunks : sms;
    const size_t smem = gv_smem().total;
#define TERN_GEMV_CASE(GG)                                                                               \
    case GG: {                                                                                           \
        auto kern = gemv_kernel<NL, GG>;                                                                 \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);             \
        kern<<<grid, kGvThreads, smem, s>>>(Wp, rs, M, K, NS, R, nchunks, x, xs, T, acc, y, status_word()); \
        break;                                                                                           \
    }
    switch (G) {
        TERN_GEMV_CASE(1)
        TERN_GEMV_CASE(2)
        TERN_GEMV_CASE(4)
        TERN_GEMV_CASE(8)
        TERN_GEMV_CASE(16)
        TERN_GEMV_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef TERN_GEMV_CASE
    return cudaGetLastError();
}

cudaError_t launch_gemv(const uint8_t *Wp, const float *rs, int64_t M, int64_t K, tern_act act, const void *x,
                        const float *xs, int64_t T, int32_t *acc, float *y, cudaStream_t s) {
    if (act == TERN_ACT_INT8) return gemv_dispatch<1>(Wp, rs, (int)M, (int)K, x, xs, (int)T, acc, y, s);
    return gemv_dispatch<3>(Wp, rs, (int)M, (int)K, x, nullptr, (int)T, nullptr, y, s);
}

// ------------------------------------------------------------- bounded-wait test hook
__global__ void test_wait_kernel(int32_t *flag, long long limit, int *status) {
    if (threadIdx.x == 0) {
        long long n = 0;
        while (*(volatile int32_t *)flag == 0) {
            if (++n > limit) {
                set_status(status, TERN_ETIMEOUT);
                break;
            }
        }
    }
}

cudaError_t launch_test_wait(int32_t *flag, long long limit, int *status, cudaStream_t s) {
    test_wait_kernel<<<1, 32, 0, s>>>(flag, limit, status);
    return cudaGetLastError();
}

}  // namespace tern
