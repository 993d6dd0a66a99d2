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
//   - every byte of weights is decoded with one table read and consumed by one dp4a per limb.
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
// Fill the limb registers of one lane for the segment `seg` (64 codes) of token vector xt.
//  int8 (NL == 1): the 64 int8 values as 16 words;
//  bf16 (NL == 3): 24-bit fixed point with per-token shift sh.
template <int NL>
__device__ __forceinline__ void gemv_load_x(SegX<NL> &X, const void *xt, int64_t seg, int sh) {
    if (NL == 1) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const int8_t *>(xt) + seg * 64);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const uint4 t = __ldg(p + v);
            X.w[0][4 * v + 0] = t.x;
            X.w[0][4 * v + 1] = t.y;
            X.w[0][4 * v + 2] = t.z;
            X.w[0][4 * v + 3] = t.w;
        }
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(xt) + seg * 64);
#pragma unroll
        for (int v = 0; v < 8; v++) {  // 8 bf16 per uint4 -> two limb words per limb
            const uint4 t = __ldg(p + v);
            const uint32_t hw[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int half = 0; half < 2; half++) {
                uint32_t wl[3] = {0, 0, 0};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const uint32_t pairw = hw[2 * half + (e >> 1)];
                    const uint16_t b = (uint16_t)((e & 1) ? (pairw >> 16) : (pairw & 0xFFFFu));
                    uint32_t h, m, l;
                    fixed_limbs(bf16_to_f32(b), sh, h, m, l);
                    wl[0] |= h << (8 * e);
                    wl[1] |= m << (8 * e);
                    wl[2] |= l << (8 * e);
                }
                const int word = 2 * v + half;
                X.w[0][word] = wl[0];
                X.w[NL > 1 ? 1 : 0][word] = wl[1];
                X.w[NL > 2 ? 2 : 0][word] = wl[2];
            }
        }
    }
}

// ------------------------------------------------------------ the TMA-fed GEMV kernel
// One CTA per SM.  A producer warp streams chunks of R consecutive rows (R*K/4 contiguous
// bytes, up to 16 KB) plus their row scales into a ring of kGvStages shared-memory stages
// with bulk copies; 16 consumer warps decode each stage as it lands and release it through
// an mbarrier, so about 96 KB of weights per SM stay in flight while the consumers compute.
//   K <= 2048: G = K/64 lanes per row, 32/G rows per warp pass, no cross-warp combine;
//   K  > 2048: NS = K/2048 slices of 512 bytes; warp w takes slice w % NS of rows
//              w / NS, w / NS + 16/NS, ...; the exact integer partial sums of a row meet in
//              shared memory (order-free 64-bit atomic adds), and the warp that adds the last
//              one writes the row.
constexpr int kGvCons = 16;  // consumer warps
constexpr int kGvThreads = (kGvCons + 1) * 32;
constexpr int kGvStages = 6;
constexpr int kGvStageBytes = 16384;
constexpr int kGvMaxRows = 128;    // rows per chunk (scale ring entries per stage)
constexpr int kGvMaxSplitRows = 16;  // rows per chunk when K > 2048 (16 KB / 1 KB)
constexpr long long kGvWaitNs = 1000000000ll;

constexpr size_t gv_smem_bytes() {
    return (size_t)kLutBytes + (size_t)kGvStages * kGvStageBytes + (size_t)kGvStages * kGvMaxRows * 4 +
           (size_t)kGvStages * kGvMaxSplitRows * (8 + 4);
}

template <int NL, int G>
__global__ void __launch_bounds__(kGvThreads, 1)
    gemv_kernel(const uint8_t *__restrict__ Wp, const float *__restrict__ rs, int M, int K, int NS, int R,
                int nchunks, const void *__restrict__ x, const float *__restrict__ xs, int T,
                int32_t *__restrict__ acc_out, float *__restrict__ y, int *status) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kGvStages], empty[kGvStages];
    __shared__ float red[32];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    unsigned char *ring = smem + kLutBytes;
    float *s_rs = reinterpret_cast<float *>(ring + (size_t)kGvStages * kGvStageBytes);             // [S][kGvMaxRows]
    unsigned long long *s_acc = reinterpret_cast<unsigned long long *>(s_rs + kGvStages * kGvMaxRows);  // [S][16]
    int *s_cnt = reinterpret_cast<int *>(s_acc + kGvStages * kGvMaxSplitRows);                    // [S][16]

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

    int issued = 0;
    if (tid == kGvCons * 32) {
        for (int q = 0; q < kGvStages; q++) {
            mbar_init(&full[q], 1);
            mbar_init(&empty[q], kGvCons);
        }
        fence_mbar_init();
        // the first stages need no release: start them before the table is built
        for (; issued < kGvStages && issued < total; issued++) issue(issued);
    }
    lut_fill(lut);
    for (int q = tid; q < kGvStages * kGvMaxSplitRows; q += blockDim.x) {
        s_acc[q] = 0ull;
        s_cnt[q] = 0;
    }
    __syncthreads();

    if (warp == kGvCons) {  // ------------------------------------------------ producer
        if (lane == 0) {
            for (; issued < total; issued++) {
                const int st = issued % kGvStages;
                if (!mbar_wait(&empty[st], (uint32_t)((issued / kGvStages) - 1) & 1u, kGvWaitNs, status)) break;
                issue(issued);
            }
            // leave only after every copy into this CTA's shared memory has landed
            for (int q = 0; q < kGvStages && q < issued; q++) {
                const int cnt = (issued - q + kGvStages - 1) / kGvStages;
                mbar_wait(&full[q], (uint32_t)(cnt - 1) & 1u, kGvWaitNs, status);
            }
        }
        return;
    }

    // ---------------------------------------------------------------------- consumers
    constexpr int RPW = 32 / G;  // rows per warp pass (K <= 2048)
    const int sub = lane / G, gl = lane % G;
    const int slice = warp % NS, rg = warp / NS, ngroups = kGvCons / NS;
    const int64_t seg = (NS > 1) ? (int64_t)slice * 32 + lane : (int64_t)gl;
    const uint32_t lane4 = (uint32_t)lane << 2;
    bool alive = true;
    int n = 0;
    for (int t = 0; t < T; t++) {
        int sh = 0;
        const void *xt;
        if (NL == 1) {
            xt = static_cast<const int8_t *>(x) + (int64_t)t * K;
        } else {
            const uint16_t *xb = static_cast<const uint16_t *>(x) + (int64_t)t * K;
            xt = xb;
            float m = 0.0f;
            for (int i = tid; i < K; i += kGvCons * 32) m = fmaxf(m, fabsf(bf16_to_f32(xb[i])));
            m = warp_max_f32(m);
            if (lane == 0) red[warp] = m;
            named_bar_sync(1, kGvCons * 32);
            float amax = 0.0f;
#pragma unroll
            for (int w = 0; w < kGvCons; w++) amax = fmaxf(amax, red[w]);
            sh = fixed_shift(amax);
        }
        SegX<NL> X;
        gemv_load_x<NL>(X, xt, seg, sh);
        const float xscale = (NL == 1 && xs != nullptr) ? xs[t] : 1.0f;
        auto epilogue = [&](int r0, int nr, int st, int row, long long S) {
            const float sc = (rs_bulk && row < (nr & ~3)) ? s_rs[st * kGvMaxRows + row] : __ldg(rs + r0 + row);
            const int64_t o = (int64_t)t * M + r0 + row;
            if (NL == 1) {
                if (acc_out) acc_out[o] = (int32_t)S;
                float v = __fmul_rn(__int2float_rn((int)S), sc);
                if (xs != nullptr) v = __fmul_rn(v, xscale);
                y[o] = v;
            } else {
                y[o] = (float)(ldexp((double)S, -sh) * (double)sc);
            }
        };

        for (int j = 0; j < my_n; j++, n++) {
            const int st = n % kGvStages;
            if (alive) alive = mbar_wait(&full[st], (uint32_t)(n / kGvStages) & 1u, kGvWaitNs, status);
            int r0, nr;
            chunk_rows(n, r0, nr);
            const unsigned char *stage = ring + (size_t)st * kGvStageBytes;
            if (alive && NS == 1) {
                for (int p = warp; p * RPW < nr; p += kGvCons) {
                    const int row = p * RPW + sub;
                    const bool valid = row < nr;
                    const uint4 wv = valid ? *reinterpret_cast<const uint4 *>(stage + (size_t)row * RB + gl * 16)
                                           : make_uint4(0u, 0u, 0u, 0u);
                    int acc[NL];
#pragma unroll
                    for (int l = 0; l < NL; l++) acc[l] = 0;
                    seg_dot<NL>(wv, X, lut, lane4, acc);
                    int a, b;
                    acc_to_pair<NL>(acc, a, b);
                    a = group_sum<G>(a);
                    if (NL > 1) b = group_sum<G>(b);
                    if (valid && gl == 0) epilogue(r0, nr, st, row, pair_value(NL, a, b));
                }
            } else if (alive && rg < ngroups) {
                for (int row = rg; row < nr; row += ngroups) {
                    const uint4 wv = *reinterpret_cast<const uint4 *>(stage + (size_t)row * RB + slice * 512 + lane * 16);
                    int acc[NL];
#pragma unroll
                    for (int l = 0; l < NL; l++) acc[l] = 0;
                    seg_dot<NL>(wv, X, lut, lane4, acc);
                    int a, b;
                    acc_to_pair<NL>(acc, a, b);
                    a = group_sum<32>(a);
                    if (NL > 1) b = group_sum<32>(b);
                    if (lane == 0) {
                        const int q = st * kGvMaxSplitRows + row;
                        atomicAdd(&s_acc[q], (unsigned long long)pair_value(NL, a, b));
                        __threadfence_block();
                        if (atomicAdd(&s_cnt[q], 1) == NS - 1) {  // the last slice of this row
                            const long long S = (long long)atomicExch(&s_acc[q], 0ull);
                            s_cnt[q] = 0;
                            epilogue(r0, nr, st, row, S);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (NL > 1) named_bar_sync(1, kGvCons * 32);  // red[] is rewritten by the next token
    }
}

static int device_sms() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int NL>
static cudaError_t gemv_dispatch(const uint8_t *Wp, const float *rs, int M, int K, const void *x,
                                 const float *xs, int T, int32_t *acc, float *y, cudaStream_t s) {
    const int RB = K / 4;
    const int NS = K > 2048 ? K / 2048 : 1;
    const int G = NS > 1 ? 32 : RB / 16;
    const int sms = device_sms();
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
    const size_t smem = gv_smem_bytes();
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
