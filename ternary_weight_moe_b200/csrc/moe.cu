// moe.cu -- one MoE FFN layer for T decode tokens, stage by stage (sm_100a).
//
//   route   router GEMV in fp64 + top-k + renormalised gates; the last CTA to finish
//           also groups the (token, slot) pairs by expert ("iPhone Runs a 20B Model at 120
//           tok/s", "MoE Is the Other Half of the Story Behind the 20B Figure": tokens routed
//           to different experts make the runtime fetch scattered weights -- grouping makes
//           every selected expert stream from HBM once per step);
//   xprep   activation limbs per token (int8 absmax codes, or 24-bit fixed point);
//   gateup  per (expert, block of rows): G and U rows are read once and applied to every
//           token routed to that expert; SwiGLU epilogue in fp64, h stored as fp32;
//   hprep   limbs of h per (token, slot);
//   down    per (expert, block of output rows): D rows read once per step;
//   combine fixed-order (top-k order) gate-weighted sum in fp64 -> bf16 (+ residual).
#include <cuda_runtime.h>
#include <math.h>

#include "kernels.h"
#include "tern_common.cuh"

namespace tern {

constexpr int kRouteWarps = 8;
constexpr int kMaxE = 1024;

// ------------------------------------------------------------------------- route kernel
// Warp per expert row, all T tokens; fp64 accumulation of exact bf16 x bf16 products, so
// the logits do not depend on summation order.  The last CTA (arrival counter) runs
// top-k for every token and, if asked, groups (token, slot) pairs by expert.
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(
    const uint16_t *__restrict__ Wg, const uint16_t *__restrict__ x, int T, int d, int E, int k,
    double *__restrict__ logits, int32_t *__restrict__ idx, float *__restrict__ g32, double *__restrict__ g64,
    unsigned int *counter, int dispatch, int32_t *n_unique, int32_t *uexp, int32_t *uoff, int32_t *ent) {
    __shared__ int s_last;
    __shared__ int s_cnt[kMaxE + 1];
    __shared__ int s_flag[kMaxE + 1];
    __shared__ int s_wsum[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e = blockIdx.x * kRouteWarps + warp;
    if (e < E) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(Wg + (int64_t)e * d);
        const int nchunk = d / 8;
        for (int t = 0; t < T; t++) {
            const uint4 *xr = reinterpret_cast<const uint4 *>(x + (int64_t)t * d);
            double acc = 0.0;
            for (int c = lane; c < nchunk; c += 32) {
                const uint4 wv = __ldg(wr + c), xv = __ldg(xr + c);
                const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    // bf16 x bf16 has at most 16 significant bits: the fp32 product is exact
                    acc += (double)__fmul_rn(bf16_to_f32((uint16_t)(ww[q] & 0xFFFFu)),
                                             bf16_to_f32((uint16_t)(xx[q] & 0xFFFFu)));
                    acc += (double)__fmul_rn(bf16_to_f32((uint16_t)(ww[q] >> 16)),
                                             bf16_to_f32((uint16_t)(xx[q] >> 16)));
                }
            }
            acc = warp_sum_f64(acc);
            if (lane == 0) logits[(int64_t)t * E + e] = acc;
        }
    }
    // last block out does the selection
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (E <= 256) {
        __shared__ double s_lg[kRouteWarps][256];
        for (int t = warp; t < T; t += kRouteWarps) {
            const double *lg = logits + (int64_t)t * E;  // written by other blocks: read through L2
#pragma unroll
            for (int j = 0; j < 8; j++) {
                const int ee = lane + 32 * j;
                s_lg[warp][ee] = (ee < E) ? __ldcg(lg + ee) : 0.0;
            }
            __syncwarp();
            warp_topk<8>(s_lg[warp], E, k, idx + (int64_t)t * k, g64 + (int64_t)t * k, g32 + (int64_t)t * k);
            __syncwarp();
        }
    } else if (warp == 0) {
        __shared__ double s_big[kMaxE];
        for (int t = 0; t < T; t++) {
            const double *lg = logits + (int64_t)t * E;
            for (int ee = lane; ee < E; ee += 32) s_big[ee] = __ldcg(lg + ee);
            __syncwarp();
            warp_topk<32>(s_big, E, k, idx + (int64_t)t * k, g64 + (int64_t)t * k, g32 + (int64_t)t * k);
            __syncwarp();
        }
    }
    if (threadIdx.x == 0) *counter = 0u;  // workspace control word back to zero
    if (!dispatch) return;
    __syncthreads();
    __threadfence_block();
    // ---- group (token, slot) pairs by expert: counts, offsets, stable placement
    const int n = T * k;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&s_cnt[idx[i]], 1);
    __syncthreads();
    // exclusive scans over experts of counts and of "selected" flags (serial per 32-chunk)
    if (threadIdx.x < 32) {
        const int per = (E + 31) / 32;
        int c0 = 0, f0 = 0;
        for (int j = 0; j < per; j++) {
            const int ee = threadIdx.x * per + j;
            if (ee < E) {
                c0 += s_cnt[ee];
                f0 += s_cnt[ee] > 0;
            }
        }
        // inclusive warp scan of the chunk totals
        int cs = c0, fs = f0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xFFFFFFFFu, cs, o), b = __shfl_up_sync(0xFFFFFFFFu, fs, o);
            if ((int)threadIdx.x >= o) {
                cs += a;
                fs += b;
            }
        }
        int crun = cs - c0, frun = fs - f0;
        for (int j = 0; j < per; j++) {
            const int ee = threadIdx.x * per + j;
            if (ee < E) {
                const int c = s_cnt[ee];
                s_flag[ee] = (c > 0) ? frun : -1;  // position among unique experts
                s_cnt[ee] = crun;                  // offset of the expert's entries
                crun += c;
                frun += c > 0;
            }
        }
        if (threadIdx.x == 31) {
            *n_unique = fs;
            s_wsum[0] = fs;
            s_wsum[1] = cs;
        }
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += blockDim.x) {
        const int u = s_flag[ee];
        if (u >= 0) {
            uexp[u] = ee;
            uoff[u] = s_cnt[ee];
        }
    }
    if (threadIdx.x == 0) uoff[s_wsum[0]] = s_wsum[1];
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int ex = idx[i];
        int rank = 0;
        for (int j = 0; j < i; j++) rank += (idx[j] == ex);
        ent[s_cnt[ex] + rank] = i;  // entry = t*k + slot, ascending within an expert
    }
}

cudaError_t launch_route(const uint16_t *Wg, const uint16_t *x, int T, int d, int E, int k, double *logits,
                         int32_t *idx, float *g32, double *g64, unsigned int *counter, bool dispatch,
                         int32_t *n_unique, int32_t *uexp, int32_t *uoff, int32_t *ent, cudaStream_t s) {
    const int grid = (E + kRouteWarps - 1) / kRouteWarps;
    route_kernel<<<grid, kRouteWarps * 32, 0, s>>>(Wg, x, T, d, E, k, logits, idx, g32, g64, counter,
                                                   dispatch ? 1 : 0, n_unique, uexp, uoff, ent);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------ prep kernels
// Activation limbs of one vector v[0..n) into words laid out [NL][n/4]:
//   NL == 1: absmax int8 codes (q), scale s = absmax/127 stored in sc;
//   NL == 3: 24-bit fixed point, shift stored (as int bits) in sc.
// The source is bf16 (src16) or fp32 (src32).
template <int NL>
__global__ void prep_kernel(const uint16_t *__restrict__ src16, const float *__restrict__ src32, int n,
                            uint32_t *__restrict__ words, float *__restrict__ sc, const int32_t *n_valid_entries) {
    __shared__ float red[32];
    const int v = blockIdx.x;
    if (n_valid_entries != nullptr && v >= *n_valid_entries) return;
    auto val = [&](int i) -> float { return src16 ? bf16_to_f32(src16[(int64_t)v * n + i]) : src32[(int64_t)v * n + i]; };
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, fabsf(val(i)));
    const float amax = block_max_f32(m, red);
    uint32_t *wv = words + (int64_t)v * NL * (n / 4);
    if (NL == 1) {
        const float inv = amax > 0.0f ? quant_inv(amax) : 0.0f;
        for (int b = threadIdx.x; b < n / 4; b += blockDim.x) {
            uint32_t w = 0;
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int q = amax > 0.0f ? quant_one(val(4 * b + e), inv) : 0;
                w |= ((uint32_t)q & 0xFFu) << (8 * e);
            }
            wv[b] = w;
        }
        if (threadIdx.x == 0) sc[v] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    } else {
        const int sh = fixed_shift(amax);
        for (int b = threadIdx.x; b < n / 4; b += blockDim.x) {
            uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
            for (int e = 0; e < 4; e++) {
                uint32_t h, mi, lo;
                fixed_limbs(val(4 * b + e), sh, h, mi, lo);
                w0 |= h << (8 * e);
                w1 |= mi << (8 * e);
                w2 |= lo << (8 * e);
            }
            wv[b] = w0;
            wv[(n / 4) + b] = w1;
            wv[2 * (n / 4) + b] = w2;
        }
        if (threadIdx.x == 0) sc[v] = __int_as_float(sh);
    }
}

// ----------------------------------------------------------------------- gate / up
constexpr int kFfnWarps = 8;

// grid: (n_unique_max, f / rows_per_block). G = d/64 lanes per row.
template <int NL, int G>
__global__ void __launch_bounds__(kFfnWarps * 32) gateup_kernel(
    const uint8_t *__restrict__ gate, const uint8_t *__restrict__ up, const float *__restrict__ sg,
    const float *__restrict__ su, int d, int f, int k, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ xw, const float *__restrict__ xsc, float *__restrict__ h,
    int32_t *__restrict__ acc_g, int32_t *__restrict__ acc_u, int rows_per_block) {
    extern __shared__ __align__(16) uint32_t lut[];
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    lut_fill(lut);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int RPW = 32 / G;
    const int sub = lane / G, gl = lane % G;
    const int e = uexp[u];
    const int e0 = uoff[u], e1 = uoff[u + 1];
    const int64_t rowb = d / 4;
    const uint8_t *G0 = gate + (int64_t)e * f * rowb;
    const uint8_t *U0 = up + (int64_t)e * f * rowb;
    const int r0 = blockIdx.y * rows_per_block;
    const uint32_t lane4 = (uint32_t)lane << 2;
    for (int q = e0; q < e1; q++) {
        const int entry = ent[q];
        const int t = entry / k;
        SegX<NL> X;
        seg_load_x<NL>(X, xw + (int64_t)t * NL * (d / 4), d / 4, gl);
        const float xs = xsc[t];
        for (int rr = warp * RPW; rr < rows_per_block; rr += kFfnWarps * RPW) {
            const int j = r0 + rr + sub;
            int ga = 0, gb = 0, ua = 0, ub = 0;
            if (j < f) {
                const uint4 wg = __ldg(reinterpret_cast<const uint4 *>(G0 + (int64_t)j * rowb) + gl);
                const uint4 wu = __ldg(reinterpret_cast<const uint4 *>(U0 + (int64_t)j * rowb) + gl);
                int ag[NL], au[NL];
#pragma unroll
                for (int l = 0; l < NL; l++) ag[l] = au[l] = 0;
                seg_dot<NL>(wg, X, lut, lane4, ag);
                seg_dot<NL>(wu, X, lut, lane4, au);
                acc_to_pair<NL>(ag, ga, gb);
                acc_to_pair<NL>(au, ua, ub);
            }
            ga = group_sum<G>(ga);
            ua = group_sum<G>(ua);
            if (NL > 1) {
                gb = group_sum<G>(gb);
                ub = group_sum<G>(ub);
            }
            if (gl == 0 && j < f) {
                const long long Sg = pair_value(NL, ga, gb), Su = pair_value(NL, ua, ub);
                float hv;
                if (NL == 1) {
                    acc_g[(int64_t)entry * f + j] = (int32_t)Sg;
                    acc_u[(int64_t)entry * f + j] = (int32_t)Su;
                    const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg), sg[(int64_t)e * f + j]), xs);
                    const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su), su[(int64_t)e * f + j]), xs);
                    hv = swiglu_f32((double)gv, (double)uv);
                } else {
                    const int sh = __float_as_int(xs);
                    const double gv = ldexp((double)Sg, -sh) * (double)sg[(int64_t)e * f + j];
                    const double uv = ldexp((double)Su, -sh) * (double)su[(int64_t)e * f + j];
                    hv = swiglu_f32(gv, uv);
                }
                h[(int64_t)entry * f + j] = hv;
            }
        }
    }
}

// ---------------------------------------------------------------------------- down
// grid: (n_unique_max, d / rows_per_block). G = f/64 lanes per row.
template <int NL, int G>
__global__ void __launch_bounds__(kFfnWarps * 32) down_kernel(
    const uint8_t *__restrict__ down, const float *__restrict__ sd, int d, int f,
    const int32_t *__restrict__ n_unique, const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff,
    const int32_t *__restrict__ ent, const uint32_t *__restrict__ hw, const float *__restrict__ hsc,
    double *__restrict__ ye, int32_t *__restrict__ acc_d, int rows_per_block) {
    extern __shared__ __align__(16) uint32_t lut[];
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    lut_fill(lut);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int RPW = 32 / G;
    const int sub = lane / G, gl = lane % G;
    const int e = uexp[u];
    const int e0 = uoff[u], e1 = uoff[u + 1];
    const int64_t rowb = f / 4;
    const uint8_t *D0 = down + (int64_t)e * d * rowb;
    const int r0 = blockIdx.y * rows_per_block;
    const uint32_t lane4 = (uint32_t)lane << 2;
    for (int q = e0; q < e1; q++) {
        const int entry = ent[q];
        SegX<NL> X;
        seg_load_x<NL>(X, hw + (int64_t)entry * NL * (f / 4), f / 4, gl);
        const float hs = hsc[entry];
        for (int rr = warp * RPW; rr < rows_per_block; rr += kFfnWarps * RPW) {
            const int i = r0 + rr + sub;
            int a = 0, b = 0;
            if (i < d) {
                const uint4 wd = __ldg(reinterpret_cast<const uint4 *>(D0 + (int64_t)i * rowb) + gl);
                int acc[NL];
#pragma unroll
                for (int l = 0; l < NL; l++) acc[l] = 0;
                seg_dot<NL>(wd, X, lut, lane4, acc);
                acc_to_pair<NL>(acc, a, b);
            }
            a = group_sum<G>(a);
            if (NL > 1) b = group_sum<G>(b);
            if (gl == 0 && i < d) {
                const long long S = pair_value(NL, a, b);
                double v;
                if (NL == 1) {
                    acc_d[(int64_t)entry * d + i] = (int32_t)S;
                    v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S), sd[(int64_t)e * d + i]), hs);
                } else {
                    v = ldexp((double)S, -__float_as_int(hs)) * (double)sd[(int64_t)e * d + i];
                }
                ye[(int64_t)entry * d + i] = v;
            }
        }
    }
}

// ------------------------------------------------------------------------- combine
// y[t,i] = sum over slots (top-k order) of g64[t,slot] * ye[t*k+slot, i], fp64.
__global__ void combine_kernel(const double *__restrict__ g64, const double *__restrict__ ye, int T, int d, int k,
                               uint16_t *__restrict__ y, float *__restrict__ y32, const uint16_t *__restrict__ resid,
                               uint16_t *__restrict__ x_out) {
    const int64_t n = (int64_t)T * d;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(p / d), i = (int)(p % d);
        double acc = 0.0;
        for (int s = 0; s < k; s++) acc += g64[t * k + s] * ye[((int64_t)t * k + s) * d + i];
        const uint16_t yb = f64_to_bf16_rne(acc);
        if (y) y[p] = yb;
        if (y32) y32[p] = (float)acc;
        if (x_out) x_out[p] = f64_to_bf16_rne((double)bf16_to_f32(resid[p]) + (double)bf16_to_f32(yb));
    }
}

// ------------------------------------------------------------------------- RMSNorm
// n = bf16(x / sqrt(mean(x^2) + eps)) in fp64; squares of bf16 are exact and their fp64
// sum is exact for these magnitudes, so the result is independent of reduction order.
__global__ void rmsnorm_kernel(const uint16_t *__restrict__ x, int d, double eps, uint16_t *__restrict__ n) {
    __shared__ double red[32];
    __shared__ double s_r;
    const uint16_t *xr = x + (int64_t)blockIdx.x * d;
    double ss = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        const double v = (double)bf16_to_f32(xr[i]);
        ss = fma(v, v, ss);
    }
    ss = warp_sum_f64(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = (threadIdx.x < (blockDim.x + 31) / 32) ? red[threadIdx.x] : 0.0;
        v = warp_sum_f64(v);
        if (threadIdx.x == 0) s_r = sqrt(v / (double)d + eps);
    }
    __syncthreads();
    const double r = s_r;
    for (int i = threadIdx.x; i < d; i += blockDim.x)
        n[(int64_t)blockIdx.x * d + i] = f64_to_bf16_rne((double)bf16_to_f32(xr[i]) / r);
}

cudaError_t launch_rmsnorm(const uint16_t *x, int T, int d, double eps, uint16_t *n, cudaStream_t s) {
    rmsnorm_kernel<<<T, 256, 0, s>>>(x, d, eps, n);
    return cudaGetLastError();
}

// ----------------------------------------------------------------- stage launcher
template <int NL>
static cudaError_t ffn_stages_nl(const tern_moe_layer *L, const uint16_t *x, int T, const FfnWs &w, uint16_t *y,
                                 float *y32, const uint16_t *resid, uint16_t *x_out, cudaStream_t s) {
    const int d = (int)L->d, f = (int)L->f, E = L->E, k = L->k;
    cudaError_t err;
    err = launch_route(L->router, x, T, d, E, k, w.logits, w.idx, w.g32, w.g64, w.ctrl, true, w.n_unique, w.uexp,
                       w.uoff, w.ent, s);
    if (err != cudaSuccess) return err;
    prep_kernel<NL><<<T, 256, 0, s>>>(x, nullptr, d, w.xw, w.xsc, nullptr);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int umax = (E < T * k) ? E : T * k;
    const int Gd = d / 64, Gf = f / 64;
    const int rpb_gu = 32, rpb_dn = 128;
    dim3 g1(umax, (f + rpb_gu - 1) / rpb_gu), g2(umax, (d + rpb_dn - 1) / rpb_dn);
#define TERN_GU_CASE(GG)                                                                                   \
    case GG: {                                                                                             \
        auto kern = gateup_kernel<NL, GG>;                                                                 \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);                \
        kern<<<g1, kFfnWarps * 32, kLutBytes, s>>>(L->gate, L->up, L->gate_scale, L->up_scale, d, f, k,    \
                                                   w.n_unique, w.uexp, w.uoff, w.ent, w.xw, w.xsc, w.h,   \
                                                   w.acc_g, w.acc_u, rpb_gu);                              \
        break;                                                                                             \
    }
    switch (Gd) {
        TERN_GU_CASE(1) TERN_GU_CASE(2) TERN_GU_CASE(4) TERN_GU_CASE(8) TERN_GU_CASE(16) TERN_GU_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef TERN_GU_CASE
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    prep_kernel<NL><<<T * k, 128, 0, s>>>(nullptr, w.h, f, w.hw, w.hsc, nullptr);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
#define TERN_DN_CASE(GG)                                                                                   \
    case GG: {                                                                                             \
        auto kern = down_kernel<NL, GG>;                                                                   \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);                \
        kern<<<g2, kFfnWarps * 32, kLutBytes, s>>>(L->down, L->down_scale, d, f, w.n_unique, w.uexp,       \
                                                   w.uoff, w.ent, w.hw, w.hsc, w.ye, w.acc_d, rpb_dn);     \
        break;                                                                                             \
    }
    switch (Gf) {
        TERN_DN_CASE(1) TERN_DN_CASE(2) TERN_DN_CASE(4) TERN_DN_CASE(8) TERN_DN_CASE(16) TERN_DN_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef TERN_DN_CASE
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    int cg = (T * d + 255) / 256;
    combine_kernel<<<cg, 256, 0, s>>>(w.g64, w.ye, T, d, k, y, y32, resid, x_out);
    return cudaGetLastError();
}

cudaError_t launch_ffn_stages(const tern_moe_layer *L, const uint16_t *x, int T, tern_act act, const FfnWs &w,
                              uint16_t *y, float *y_f32, const uint16_t *residual, uint16_t *x_out, cudaStream_t s) {
    if (act == TERN_ACT_INT8) return ffn_stages_nl<1>(L, x, T, w, y, y_f32, residual, x_out, s);
    return ffn_stages_nl<3>(L, x, T, w, y, y_f32, residual, x_out, s);
}

}  // namespace tern
