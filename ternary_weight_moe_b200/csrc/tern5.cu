// tern5.cu -- the base-3 packed format: five ternary weights per byte (sm_100a).
//
// A ternary weight carries log2(3) ~ 1.585 bits of information ("How a 20B Model Hits 120
// tok/s on an iPhone", "Why the number is plausible"; "A 20B AI Model Trained in Ternary Just
// Hit 218 Tokens/Second on a $599 Mac Mini", "What Ternary Actually Means").  3^5 = 243 <= 256,
// so five weights fit one byte (1.6 bits): 19% fewer bytes than four 2-bit codes per byte.
// Byte b of a row holds t_0 + 3 t_1 + 9 t_2 + 27 t_3 + 81 t_4, t_i the 2-bit code of weight
// 5b+i (0 -> 0, 1 -> +1, 2 -> -1); positions past K are 0; rows are padded with zero bytes to a
// multiple of 16 bytes.
//
// GEMV: one warp per row, lane l takes 16-byte segments l, l+32, ... (80 weights each).  A
// byte is decoded by ONE 8-byte table read: its first four weights as int8 lanes (one dp4a per
// limb against the limbs of activations 5b..5b+3) and its fifth weight, which joins the fifth
// weights of the three neighbouring bytes in one word (two byte-permutes) for one more dp4a per
// limb against a word of fifth activations.  The activations are re-laid out once per CTA in
// shared memory to match: per limb, word b = activations 5b..5b+3, and word c = the fifth
// activations of bytes 4c..4c+3.  Same exact integer sums as the 2-bit GEMV.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ternmoe.h"
#include "kernels.h"
#include "tern_common.cuh"

namespace {

using namespace tern;

__device__ unsigned long long g_code5_errors = 0;

constexpr int kT5Warps = 8;
constexpr int64_t kT5MaxK = 16384;
constexpr int kT5Pre = 7;  // row segments per lane loaded ahead: ceil(row_bytes5(kT5MaxK) / 16 / 32)
constexpr int64_t kT5MaxT = 64;

__host__ __device__ inline int64_t row_bytes5(int64_t K) { return ((K + 4) / 5 + 15) / 16 * 16; }

// digits of b (b < 243) as int8 weights: x = weights 0..3, y = weight 4 in byte 0
__device__ __forceinline__ uint2 decode5(uint32_t b) {
    if (b >= 243u) return make_uint2(0u, 0u);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 5; i++) {
        const uint32_t t = b % 3u;
        b /= 3u;
        const uint32_t v = (t == 1u) ? 0x01u : (t == 2u) ? 0xFFu : 0x00u;
        if (i < 4) lo |= v << (8 * i);
        else hi = v;
    }
    return make_uint2(lo, hi);
}

__global__ void pack5_kernel(const int8_t *__restrict__ w, int64_t M, int64_t K, int64_t rb,
                             uint8_t *__restrict__ out, unsigned long long *bad) {
    unsigned long long nbad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < M * rb; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / rb, b = i % rb;
        uint32_t value = 0, place = 1;
#pragma unroll
        for (int j = 0; j < 5; j++) {
            const int64_t k = 5 * b + j;
            uint32_t t = 0;
            if (k < K) {
                const int v = w[m * K + k];
                if (v == 1) t = 1;
                else if (v == -1) t = 2;
                else if (v != 0) nbad++;
            }
            value += t * place;
            place *= 3;
        }
        out[i] = (uint8_t)value;
    }
    if (nbad) atomicAdd(bad, nbad);
}

__global__ void unpack5_kernel(const uint8_t *__restrict__ p, int64_t M, int64_t K, int64_t rb,
                               int8_t *__restrict__ w, unsigned long long *bad) {
    const int64_t nb = (K + 4) / 5;  // bytes of a row that hold weights
    unsigned long long nbad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < M * nb; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = i / nb, b = i % nb;
        uint32_t value = p[m * rb + b];
        if (value >= 243u) {
            nbad++;
            value = 0;
        }
#pragma unroll
        for (int j = 0; j < 5; j++) {
            const int64_t k = 5 * b + j;
            const uint32_t t = value % 3u;
            value /= 3u;
            if (k < K) w[m * K + k] = (int8_t)(t == 1u ? 1 : (t == 2u ? -1 : 0));
        }
    }
    if (nbad) atomicAdd(bad, nbad);
}

// activation limb of x[k] (zero past K): int8 path the value itself, bf16 path byte l of the
// 24-bit fixed-point value
template <int NL>
__device__ __forceinline__ void limbs_at(const void *xt, int64_t k, int64_t K, int sh, uint32_t (&lb)[3]) {
    lb[0] = lb[1] = lb[2] = 0;
    if (k >= K) return;
    if (NL == 1) {
        lb[0] = (uint32_t)(uint8_t) static_cast<const int8_t *>(xt)[k];
    } else {
        fixed_limbs(bf16_to_f32(static_cast<const uint16_t *>(xt)[k]), sh, lb[0], lb[1], lb[2]);
    }
}

template <int NL>
__global__ void __launch_bounds__(kT5Warps * 32) gemv5_kernel(const uint8_t *__restrict__ W5, const float *__restrict__ rs,
                                                              int M, int K, int rb, const void *__restrict__ x,
                                                              const float *__restrict__ xs, int T,
                                                              int32_t *__restrict__ acc_out, float *__restrict__ y) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint2 *lut = reinterpret_cast<uint2 *>(smem);                 // [256][32] lane-private 8-byte entries
    // activations 5b..5b+3 of byte b: [NL][segments][kSegPad words] (16 used per segment; the
    // padding puts the 16-byte loads of 8 lanes reading 8 segments in 8 different bank groups)
    const int nseg = rb / 16, xap = nseg * kSegPad;
    uint32_t *xa = smem + 256 * 32 * 2;
    uint32_t *xb = xa + NL * xap;                                 // [NL][rb/4] fifth activations
    uint8_t *xbb = reinterpret_cast<uint8_t *>(xb);
    __shared__ float red[32];
    __shared__ int s_sh;
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) lut[i] = decode5((uint32_t)(i >> 5));
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lane8 = (uint32_t)lane << 3;
    const char *lbase = reinterpret_cast<const char *>(lut);
    for (int t = 0; t < T; t++) {
        const void *xt;
        int sh = 0;
        if (NL == 1) {
            xt = static_cast<const int8_t *>(x) + (int64_t)t * K;
        } else {
            const uint16_t *xh = static_cast<const uint16_t *>(x) + (int64_t)t * K;
            xt = xh;
            float m = 0.0f;
            for (int i = threadIdx.x; i < K; i += blockDim.x) m = fmaxf(m, fabsf(bf16_to_f32(xh[i])));
            const float amax = block_max_f32(m, red);
            if (threadIdx.x == 0) s_sh = fixed_shift(amax);
            __syncthreads();
            sh = s_sh;
        }
        for (int b = threadIdx.x; b < rb; b += blockDim.x) {
            uint32_t w4[3] = {0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 4; j++) {
                uint32_t lb[3];
                limbs_at<NL>(xt, 5 * (int64_t)b + j, K, sh, lb);
#pragma unroll
                for (int l = 0; l < NL; l++) w4[l] |= lb[l] << (8 * j);
            }
            uint32_t l5[3];
            limbs_at<NL>(xt, 5 * (int64_t)b + 4, K, sh, l5);
#pragma unroll
            for (int l = 0; l < NL; l++) {
                xa[l * xap + (b >> 4) * kSegPad + (b & 15)] = w4[l];
                xbb[l * rb + b] = (uint8_t)l5[l];
            }
        }
        __syncthreads();  // table (first token) and this token's limbs ready
        const float xscale = (NL == 1 && xs != nullptr) ? xs[t] : 1.0f;
        for (int row = blockIdx.x * kT5Warps + warp; row < M; row += gridDim.x * kT5Warps) {
            int acc[NL];
#pragma unroll
            for (int l = 0; l < NL; l++) acc[l] = 0;
            // every segment of the row this lane takes, all loads in flight before any decode
            // (K <= 16384: at most 205 segments, kT5Pre per lane)
            uint4 wpre[kT5Pre];
#pragma unroll
            for (int u = 0; u < kT5Pre; u++) {
                const int sg = lane + 32 * u;
                wpre[u] = sg < nseg ? __ldg(reinterpret_cast<const uint4 *>(W5 + (int64_t)row * rb) + sg)
                                    : make_uint4(0u, 0u, 0u, 0u);
            }
            const float rsv = lane == 0 ? rs[row] : 0.0f;
#pragma unroll
            for (int u = 0; u < kT5Pre; u++) {
                const int seg = lane + 32 * u;
                if (seg >= nseg) break;
                const uint4 wv = wpre[u];
                const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
                uint4 x5v[NL];  // fifth activations of the segment's 16 bytes, one 16-byte load per limb
#pragma unroll
                for (int l = 0; l < NL; l++) x5v[l] = *reinterpret_cast<const uint4 *>(xb + l * (rb / 4) + seg * 4);
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    uint2 e[4];
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        e[i] = *reinterpret_cast<const uint2 *>(lbase + __byte_perm(words[q], lane8, 0x5504u | ((uint32_t)i << 4)));
                    // fifth weights of the four bytes in one word (bytes 1..3 of e[i].y are zero)
                    const uint32_t c01 = __byte_perm(e[0].y, e[1].y, 0x1140u);
                    const uint32_t c23 = __byte_perm(e[2].y, e[3].y, 0x1140u);
                    const uint32_t c5 = __byte_perm(c01, c23, 0x5410u);
#pragma unroll
                    for (int l = 0; l < NL; l++) {
                        const uint4 xv = *reinterpret_cast<const uint4 *>(xa + l * xap + seg * kSegPad + 4 * q);
                        const uint32_t xl[4] = {xv.x, xv.y, xv.z, xv.w};
                        const uint32_t x5 = q == 0 ? x5v[l].x : q == 1 ? x5v[l].y : q == 2 ? x5v[l].z : x5v[l].w;
                        if (l == 0) {
#pragma unroll
                            for (int i = 0; i < 4; i++) acc[l] = dp4a_ss(e[i].x, xl[i], acc[l]);
                            acc[l] = dp4a_ss(c5, x5, acc[l]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; i++) acc[l] = dp4a_su(e[i].x, xl[i], acc[l]);
                            acc[l] = dp4a_su(c5, x5, acc[l]);
                        }
                    }
                }
            }
            int a, b;
            acc_to_pair<NL>(acc, a, b);
            a = group_sum<32>(a);
            if (NL > 1) b = group_sum<32>(b);
            if (lane == 0) {
                const long long S = pair_value(NL, a, b);
                const int64_t o = (int64_t)t * M + row;
                if (NL == 1) {
                    if (acc_out) acc_out[o] = (int32_t)S;
                    float v = __fmul_rn(__int2float_rn((int)S), rsv);
                    if (xs != nullptr) v = __fmul_rn(v, xscale);
                    y[o] = v;
                } else {
                    y[o] = (float)(ldexp((double)S, -sh) * (double)rsv);
                }
            }
        }
        __syncthreads();  // limbs and red[] are rewritten by the next token
    }
}

inline bool aligned5(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

int grid5(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    if (g > 148 * 16) g = 148 * 16;
    return (int)(g < 1 ? 1 : g);
}

tern_status code_pass(bool pack, const void *src, int64_t M, int64_t K, void *dst, void *stream) {
    if (!src || !dst || M <= 0 || K <= 0 || M > (1ll << 30) || K > (1ll << 30)) return TERN_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned long long *bad = nullptr;
    if (cudaGetSymbolAddress((void **)&bad, g_code5_errors) != cudaSuccess) return TERN_ECUDA;
    if (cudaMemsetAsync(bad, 0, sizeof(unsigned long long), s) != cudaSuccess) return TERN_ECUDA;
    const int64_t rb = row_bytes5(K);
    if (pack)
        pack5_kernel<<<grid5(M * rb, 256), 256, 0, s>>>(static_cast<const int8_t *>(src), M, K, rb,
                                                         static_cast<uint8_t *>(dst), bad);
    else
        unpack5_kernel<<<grid5(M * ((K + 4) / 5), 256), 256, 0, s>>>(static_cast<const uint8_t *>(src), M, K, rb,
                                                                      static_cast<int8_t *>(dst), bad);
    if (cudaGetLastError() != cudaSuccess) return TERN_ECUDA;
    unsigned long long h = 0;
    if (cudaMemcpyAsync(&h, bad, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return TERN_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return TERN_ECUDA;
    return h ? TERN_ECODE : TERN_OK;
}

template <int NL>
cudaError_t gemv5_launch(const uint8_t *W5, const float *rs, int M, int K, const void *x, const float *xs, int T,
                         int32_t *acc, float *y, cudaStream_t s) {
    const int rb = (int)row_bytes5(K);
    // table, padded activation words (kSegPad per 16 bytes of row), fifth activations
    const size_t smem = (size_t)256 * 32 * 8 + (size_t)NL * (rb / 16) * kSegPad * 4 + (size_t)NL * rb;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int grid = (M + kT5Warps - 1) / kT5Warps;
    if (grid > 2 * sms) grid = 2 * sms;
    cudaFuncSetAttribute(gemv5_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    gemv5_kernel<NL><<<grid, kT5Warps * 32, smem, s>>>(W5, rs, M, K, rb, x, xs, T, acc, y);
    return cudaGetLastError();
}

}  // namespace

extern "C" int64_t tern5_row_bytes(int64_t K) { return K > 0 ? row_bytes5(K) : 0; }

extern "C" tern_status tern5_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, void *stream) {
    return code_pass(true, w, M, K, packed, stream);
}

extern "C" tern_status tern5_unpack(const uint8_t *packed, int64_t M, int64_t K, int8_t *w, void *stream) {
    return code_pass(false, packed, M, K, w, stream);
}

extern "C" tern_status tern5_gemv(const uint8_t *W5, const float *row_scale, int64_t M, int64_t K, tern_act act,
                                  const void *x, const float *x_scale, int64_t T, int32_t *acc, float *y,
                                  void *stream) {
    if (!W5 || !row_scale || !x || !y || M <= 0 || M > (1ll << 30) || T < 1 || T > kT5MaxT) return TERN_EINVAL;
    if (K < 1 || K > kT5MaxK) return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    if (act == TERN_ACT_BF16 && (acc || x_scale)) return TERN_EINVAL;
    if (!aligned5(W5, 16) || !aligned5(x, 2) || !aligned5(row_scale, 4) || !aligned5(y, 4) ||
        (acc && !aligned5(acc, 4)) || (x_scale && !aligned5(x_scale, 4)))
        return TERN_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = (act == TERN_ACT_INT8)
                              ? gemv5_launch<1>(W5, row_scale, (int)M, (int)K, x, x_scale, (int)T, acc, y, s)
                              : gemv5_launch<3>(W5, row_scale, (int)M, (int)K, x, nullptr, (int)T, nullptr, y, s);
    return e == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
