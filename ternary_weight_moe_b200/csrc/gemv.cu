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
constexpr int kGemvWarps = 8;

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

// G lanes per row slice; NS row slices of KS = 64*G codes (split-K across warps when NS > 1).
template <int NL, int G>
__global__ void __launch_bounds__(kGemvWarps * 32) gemv_kernel(const uint8_t *__restrict__ Wp,
                                                                const float *__restrict__ rs, int M, int K,
                                                                int NS, const void *__restrict__ x,
                                                                const float *__restrict__ xs, int T,
                                                                int32_t *__restrict__ acc_out,
                                                                float *__restrict__ y) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *lut = smem;                                            // kLutWords
    long long *part = reinterpret_cast<long long *>(smem + kLutWords);  // [kGemvWarps][32/G]
    __shared__ float red[32];
    __shared__ int sh_shift;

    lut_fill(lut);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lane4 = (uint32_t)lane << 2;
    const int slice = warp % NS;              // K slice of this warp
    const int rgroup = warp / NS;             // row group inside the CTA
    const int ngroups = kGemvWarps / NS;
    constexpr int RPW = 32 / G;               // rows per warp pass
    const int sub = lane / G, gl = lane % G;  // row inside the pass, lane inside the row
    const int64_t seg = (int64_t)slice * G + gl;  // segment index along K
    const int64_t row_bytes = K / 4;
    const int rows_per_cta = ngroups * RPW;

    for (int t = 0; t < T; t++) {
        int sh = 0;
        const void *xt;
        if (NL == 1) {
            xt = static_cast<const int8_t *>(x) + (int64_t)t * K;
        } else {
            const uint16_t *xb = static_cast<const uint16_t *>(x) + (int64_t)t * K;
            xt = xb;
            float m = 0.0f;
            for (int i = threadIdx.x; i < K; i += blockDim.x) m = fmaxf(m, fabsf(bf16_to_f32(xb[i])));
            const float amax = block_max_f32(m, red);
            if (threadIdx.x == 0) sh_shift = fixed_shift(amax);
            __syncthreads();
            sh = sh_shift;
        }
        SegX<NL> X;
        gemv_load_x<NL>(X, xt, seg, sh);
        __syncthreads();  // lut ready (first iteration) / red reuse
        const float xscale = (NL == 1 && xs != nullptr) ? xs[t] : 1.0f;

        for (int base = blockIdx.x * rows_per_cta; base < M; base += gridDim.x * rows_per_cta) {
            const int row = base + rgroup * RPW + sub;
            int a = 0, b = 0;
            if (row < M) {
                const uint4 wb = __ldg(reinterpret_cast<const uint4 *>(Wp + (int64_t)row * row_bytes) + seg);
                int acc[NL];
#pragma unroll
                for (int l = 0; l < NL; l++) acc[l] = 0;
                seg_dot<NL>(wb, X, lut, lane4, acc);
                acc_to_pair<NL>(acc, a, b);
            }
            a = group_sum<G>(a);
            if (NL > 1) b = group_sum<G>(b);
            long long S = pair_value(NL, a, b);
            if (NS > 1) {
                __syncthreads();
                if (gl == 0) part[warp * RPW + sub] = S;
                __syncthreads();
                if (slice != 0) continue;
                S = 0;
                for (int sl = 0; sl < NS; sl++) S += part[(rgroup * NS + sl) * RPW + sub];  // fixed order
            }
            if (gl == 0 && row < M) {
                if (NL == 1) {
                    if (acc_out) acc_out[(int64_t)t * M + row] = (int32_t)S;
                    float v = __fmul_rn(__int2float_rn((int)S), rs[row]);
                    if (xs != nullptr) v = __fmul_rn(v, xscale);
                    y[(int64_t)t * M + row] = v;
                } else {
                    y[(int64_t)t * M + row] = (float)(ldexp((double)S, -sh) * (double)rs[row]);
                }
            }
        }
        __syncthreads();
    }
}

template <int NL>
static cudaError_t gemv_dispatch(const uint8_t *Wp, const float *rs, int M, int K, const void *x,
                                 const float *xs, int T, int32_t *acc, float *y, cudaStream_t s) {
    const int KS = K > 2048 ? 2048 : K;
    const int NS = K / KS;
    const int G = KS / 64;
    const int RPW = 32 / G;
    const int rows_per_cta = (kGemvWarps / NS) * RPW;
    int grid = (M + rows_per_cta - 1) / rows_per_cta;
    if (grid > 148 * 8) grid = 148 * 8;
    const size_t smem = kLutBytes + sizeof(long long) * kGemvWarps * 32;
#define TERN_GEMV_CASE(GG)                                                                              \
    case GG: {                                                                                          \
        auto kern = gemv_kernel<NL, GG>;                                                                \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);            \
        kern<<<grid, kGemvWarps * 32, smem, s>>>(Wp, rs, M, K, NS, x, xs, T, acc, y);                 \
        break;                                                                                          \
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
