// moe.cu -- one MoE FFN layer for T decode tokens, stage by stage (sm_100a).
//
//   logits  router GEMV in fp64 (exact products, fused multiply-add), eight tokens per CTA;
//   select  per token: top-k + renormalised gates; the last CTA to finish also groups the
//           (token, slot) pairs by expert ("iPhone Runs a 20B Model at 120 tok/s", "MoE Is
//           the Other Half of the Story Behind the 20B Figure": tokens routed to different
//           experts make the runtime fetch scattered weights -- grouping makes every selected
//           expert stream from HBM once per step);
//   xprep   activation limbs per token (int8 absmax codes, or 24-bit fixed point);
//   gateup  per (expert, block of rows): G and U rows are read once and applied to every
//           token routed to that expert; SwiGLU epilogue in fp64, h stored as fp32;
//   hprep   limbs of h per (token, slot);
//   down    per (expert, block of output rows): D rows read once per step;
//   combine fixed-order (top-k order) gate-weighted sum in fp64 -> bf16 (+ residual).
#include <cuda_runtime.h>
#include <math.h>

#include <utility>

#include "kernels.h"
#include "tern_common.cuh"

namespace tern {

// Launch with arguments converted to the kernel's parameter types; returns the launch error.
template <typename... K, typename... A>
static cudaError_t launch_k(void (*kern)(K...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}


// ------------------------------------------------------------------------- route kernels
// logits_kernel: each warp takes 4 expert rows and each CTA 4 tokens (8 warps: 32 experts x 4
// tokens).  The tokens' x is converted to fp64 once per CTA, 512 elements at a time, into shared
// memory; a lane reads two adjacent columns of x per load and applies them to the 4 rows of its
// warp, so every shared-memory read feeds 8 products per token.  Each product of two bf16 values
// is exact in fp64 (at most 16 significant bits), so one fp64 fma per product adds the exact
// product with one rounding; the sums are exact for the router's magnitudes (checked by the
// oracle), so the summation order does not change the logits.
constexpr int kRouteTok = 4;
constexpr int kLogitWarps = 8;
constexpr int kLogitEPW = 4;  // expert rows per warp
constexpr int kLogitChunk = 512;

__global__ void __launch_bounds__(kLogitWarps * 32) logits_kernel(const uint16_t *__restrict__ Wg,
                                                                   const uint16_t *__restrict__ x, int T, int d,
                                                                   int E, double *__restrict__ logits) {
    __shared__ __align__(16) double s_x[kRouteTok][kLogitChunk];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int eb = (blockIdx.x * kLogitWarps + warp) * kLogitEPW;  // first expert row of this warp
    const int t0 = blockIdx.y * kRouteTok;
    const int nt = min(kRouteTok, T - t0);
    double acc[kLogitEPW][kRouteTok];
#pragma unroll
    for (int q = 0; q < kLogitEPW; q++)
#pragma unroll
        for (int tt = 0; tt < kRouteTok; tt++) acc[q][tt] = 0.0;
    constexpr int PPL = kLogitChunk / 64;                               // column pairs per lane per chunk
    constexpr int XPT = kRouteTok * kLogitChunk / (kLogitWarps * 32);  // x values per thread per chunk
    uint32_t wv[kLogitEPW][PPL];
    uint16_t xv[XPT];
    // loads of chunk c0 into registers (all issued before any is used); pair i of a lane is
    // columns 2 * lane + 64 * i and the next one
    auto fetch = [&](int c0) {
        const int n = min(kLogitChunk, d - c0);
#pragma unroll
        for (int q = 0; q < kLogitEPW; q++) {
            const int e = eb + q;
#pragma unroll
            for (int i = 0; i < PPL; i++) {
                const int j = 2 * lane + 64 * i;
                wv[q][i] = (e < E && j < n)
                               ? __ldg(reinterpret_cast<const uint32_t *>(Wg + (int64_t)e * d + c0 + j))
                               : 0u;
            }
        }
#pragma unroll
        for (int i = 0; i < XPT; i++) {
            const int qq = threadIdx.x + i * kLogitWarps * 32, tt = qq / kLogitChunk, j = qq % kLogitChunk;
            xv[i] = (tt < nt && j < n) ? __ldg(x + (int64_t)(t0 + tt) * d + c0 + j) : (uint16_t)0;
        }
    };
    fetch(0);
    for (int c0 = 0; c0 < d; c0 += kLogitChunk) {
        __syncthreads();  // previous chunk consumed
#pragma unroll
        for (int i = 0; i < XPT; i++) {
            const int qq = threadIdx.x + i * kLogitWarps * 32;
            s_x[qq / kLogitChunk][qq % kLogitChunk] = bf16_to_f64(xv[i]);
        }
        uint32_t w[kLogitEPW][PPL];
#pragma unroll
        for (int q = 0; q < kLogitEPW; q++)
#pragma unroll
            for (int i = 0; i < PPL; i++) w[q][i] = wv[q][i];
        if (c0 + kLogitChunk < d) fetch(c0 + kLogitChunk);  // next chunk's loads fly during this one
        __syncthreads();
#pragma unroll
        for (int i = 0; i < PPL; i++) {
            const int j = 2 * lane + 64 * i;
            double2 xs[kRouteTok];
#pragma unroll
            for (int tt = 0; tt < kRouteTok; tt++) xs[tt] = *reinterpret_cast<const double2 *>(&s_x[tt][j]);
#pragma unroll
            for (int q = 0; q < kLogitEPW; q++) {
                const double w0 = bf16_to_f64((uint16_t)(w[q][i] & 0xFFFFu)), w1 = bf16_to_f64((uint16_t)(w[q][i] >> 16));
#pragma unroll
                for (int tt = 0; tt < kRouteTok; tt++) {
                    acc[q][tt] = fma(w0, xs[tt].x, acc[q][tt]);
                    acc[q][tt] = fma(w1, xs[tt].y, acc[q][tt]);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kLogitEPW; q++) {
        const int e = eb + q;
#pragma unroll
        for (int tt = 0; tt < kRouteTok; tt++) {
            const double v = warp_sum_f64(acc[q][tt]);
            if (lane == 0 && tt < nt && e < E) logits[(int64_t)(t0 + tt) * E + e] = v;
        }
    }
}

// select_kernel: one CTA per token -- top-k of its logits, renormalised gates.  The last CTA
// to finish (arrival counter) groups the (token, slot) pairs by expert when asked.
constexpr int kSelectThreads = 256;

__global__ void __launch_bounds__(kSelectThreads) select_kernel(
    const double *__restrict__ logits, int T, int E, int k, int32_t *__restrict__ idx, float *__restrict__ g32,
    double *__restrict__ g64, unsigned int *counter, int dispatch, int32_t *n_unique, int32_t *uexp, int32_t *uoff,
    int32_t *ent) {
    __shared__ int s_last;
    __shared__ int s_cnt[kMaxE + 1];
    __shared__ int s_flag[kMaxE + 1];
    __shared__ int s_wsum[32];
    __shared__ double s_lg[kMaxE];
    __shared__ int32_t s_idx[8];
    __shared__ __align__(16) uint32_t s_gm[32];
    __shared__ int s_nc;
    __shared__ ulonglong2 s_cand[256];
    __shared__ int32_t s_all[kMaxT * kMaxKsel];  // every (token, slot) expert index
    const int t = blockIdx.x;
    const double *lg = logits + (int64_t)t * E;
    double mine = 0.0;
    for (int e = threadIdx.x; e < E; e += kSelectThreads) {
        const double v = lg[e];
        s_lg[e] = v;
        if (e == (int)threadIdx.x) mine = v;
    }
    __syncthreads();
    if (E <= 256) {
        block_topk_select(mine, E, k, s_idx, s_gm, &s_nc, s_cand);
    } else {
        if (threadIdx.x < 32) warp_topk_select<32>(s_lg, E, k, s_idx);
        __syncthreads();
    }
    if (threadIdx.x < 32) {
        warp_topk_gates(s_lg, k, s_idx, g64 + (int64_t)t * k, g32 + (int64_t)t * k);
        if (threadIdx.x < k) idx[(int64_t)t * k + threadIdx.x] = s_idx[threadIdx.x];
    }
    // last CTA out groups the pairs
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) *counter = 0u;  // workspace control word back to zero
    if (!dispatch) return;
    // ---- group (token, slot) pairs by expert: counts, offsets, stable placement
    const int n = T * k;
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s_cnt[i] = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_all[i] = __ldcg(idx + i);  // other CTAs' results
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&s_cnt[s_all[i]], 1);
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
    __syncthreads();  // uoff written from s_cnt; s_cnt now becomes the running placement offset
    if (threadIdx.x < 32) {
        // stable placement, 32 entries at a time: entries of one expert keep ascending order
        const int lane = threadIdx.x;
        for (int c0 = 0; c0 < n; c0 += 32) {
            const int i = c0 + lane;
            const bool v = i < n;
            const int ex = v ? s_all[i] : -1 - lane;  // distinct values for lanes past the end
            const unsigned m = __match_any_sync(0xFFFFFFFFu, ex);
            const int before = __popc(m & ((1u << lane) - 1u));
            const int base = v ? s_cnt[ex] : 0;
            __syncwarp();
            if (v) {
                ent[base + before] = i;  // entry = t*k + slot
                if (lane == __ffs(m) - 1) s_cnt[ex] = base + __popc(m);
            }
            __syncwarp();
        }
    }
}

cudaError_t launch_route(const uint16_t *Wg, const uint16_t *x, int T, int d, int E, int k, double *logits,
                         int32_t *idx, float *g32, double *g64, unsigned int *counter, bool dispatch,
                         int32_t *n_unique, int32_t *uexp, int32_t *uoff, int32_t *ent, cudaStream_t s) {
    const dim3 g1((E + kLogitWarps * kLogitEPW - 1) / (kLogitWarps * kLogitEPW), (T + kRouteTok - 1) / kRouteTok);
    cudaError_t err = launch_k(logits_kernel, g1, dim3(kLogitWarps * 32), 0, s, Wg, x, T, d, E, logits);
    if (err != cudaSuccess) return err;
    return launch_k(select_kernel, dim3(T), dim3(kSelectThreads), 0, s, (const double *)logits, T, E, k, idx,
                    g32, g64, counter, dispatch ? 1 : 0, n_unique, uexp, uoff, ent);
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

// ------------------------------------------------- grouped path on int8 tensor cores (T >= 32)
// At 32 or more tokens a step routes ~2+ tokens to each selected expert and the dp4a kernels
// above become bound by their decode instructions (one table read and NL dp4a per packed byte
// PER TOKEN).  Here the decoded weights feed int8 MMAs (mma.sync m16n8k32): a warp owns 16
// rows; the A fragment register of row r and codes 4c..4c+3 is exactly the table entry of
// packed byte c of that row, so one table read per packed byte serves up to 8 tokens and
// every activation limb.  B columns are tokens (expert entries); each limb is its own MMA
// (hi limb signed x signed, mid and lo signed x unsigned) and the limbs recombine exactly in
// int64: S = hi * 65536 + mid * 256 + lo.  Same integers as the dp4a kernels, bit for bit.
constexpr int kMmaGroupedMinT = 32;
constexpr int kMmaWarps = 8;
constexpr int kMmaRows = 16 * kMmaWarps;  // rows per CTA
constexpr int kMmaTok = 8;                // tokens (B columns) per pass
constexpr int kMmaPad = 4;                // words of padding per staged limb row (bank spread)

template <bool USIGNED>
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    if (USIGNED)
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stage the limb words of entries q0..q0+nb-1 (vector v = ent[q] / div, NL*n4 words each) as
// [kMmaTok][NL][n4 + kMmaPad]; columns nb..kMmaTok-1 are zero.
template <int NL>
__device__ __forceinline__ void mma_stage(uint32_t *dst, const uint32_t *__restrict__ src, int n4,
                                          const int32_t *__restrict__ ent, int q0, int nb, int div) {
    const int rs = n4 + kMmaPad;
    for (int i = threadIdx.x; i < kMmaTok * NL * n4; i += blockDim.x) {
        const int b = i / (NL * n4), r = i % (NL * n4), l = r / n4, w = r % n4;
        dst[(b * NL + l) * rs + w] = (b < nb) ? __ldg(src + (int64_t)(ent[q0 + b] / div) * NL * n4 + r) : 0u;
    }
}

// One 16-row tile x K codes of one matrix against the staged columns: acc[l] += A * B_l.
// row0 = the tile's first row; rows >= nrows contribute zeros.  K % 64 == 0.  lut: the compact
// 256-word decode table (entry = the four int8 weights of a packed byte); it keeps shared
// memory small enough for four CTAs per SM, which hide the row loads' latency.
template <int NL, int NM>
__device__ __forceinline__ void mma_tile(const uint8_t *const (&mats)[NM], int64_t rowb, int row0, int nrows, int K,
                                         const uint32_t *xs, int rs, const uint32_t *lut, int (&acc)[NM][NL][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    const int sh = 8 * tig;  // byte tig of a word
    const bool v0 = row0 + g < nrows, v1 = row0 + g + 8 < nrows;
    for (int m = 0; m < K / 64; m++) {  // 16 packed bytes = two k-blocks of 32 codes
        uint4 w0[NM], w1[NM];
#pragma unroll
        for (int q = 0; q < NM; q++) {
            w0[q] = v0 ? __ldg(reinterpret_cast<const uint4 *>(mats[q] + (int64_t)(row0 + g) * rowb) + m)
                       : make_uint4(0u, 0u, 0u, 0u);
            w1[q] = v1 ? __ldg(reinterpret_cast<const uint4 *>(mats[q] + (int64_t)(row0 + g + 8) * rowb) + m)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int jj = 0; jj < 2; jj++) {
            const int j = 2 * m + jj;  // k-block: codes 32j .. 32j+31, limb words 8j .. 8j+7
            uint32_t b0[NL], b1[NL];
#pragma unroll
            for (int l = 0; l < NL; l++) {
                b0[l] = xs[(g * NL + l) * rs + 8 * j + tig];
                b1[l] = xs[(g * NL + l) * rs + 8 * j + 4 + tig];
            }
#pragma unroll
            for (int q = 0; q < NM; q++) {
                const uint32_t lo0 = jj ? w0[q].z : w0[q].x, hi0 = jj ? w0[q].w : w0[q].y;
                const uint32_t lo1 = jj ? w1[q].z : w1[q].x, hi1 = jj ? w1[q].w : w1[q].y;
                const uint32_t a0 = lut[(lo0 >> sh) & 0xFFu], a1 = lut[(lo1 >> sh) & 0xFFu];
                const uint32_t a2 = lut[(hi0 >> sh) & 0xFFu], a3 = lut[(hi1 >> sh) & 0xFFu];
                mma_s8<false>(acc[q][0], a0, a1, a2, a3, b0[0], b1[0]);
                if (NL > 1) {
                    mma_s8<true>(acc[q][NL > 1 ? 1 : 0], a0, a1, a2, a3, b0[NL > 1 ? 1 : 0], b1[NL > 1 ? 1 : 0]);
                    mma_s8<true>(acc[q][NL > 2 ? 2 : 0], a0, a1, a2, a3, b0[NL > 2 ? 2 : 0], b1[NL > 2 ? 2 : 0]);
                }
            }
        }
    }
}

// grid: (n_unique_max, ceil(f / 128)); 8 warps x 16 rows of gate and up.
template <int NL>
__global__ void __launch_bounds__(kMmaWarps * 32) gateup_mma_kernel(
    const uint8_t *__restrict__ gate, const uint8_t *__restrict__ up, const float *__restrict__ sg,
    const float *__restrict__ su, int d, int f, int k, const int32_t *__restrict__ n_unique,
    const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff, const int32_t *__restrict__ ent,
    const uint32_t *__restrict__ xw, const float *__restrict__ xsc, float *__restrict__ h,
    int32_t *__restrict__ acc_g, int32_t *__restrict__ acc_u) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *lut = smem;        // [256] compact decode table
    uint32_t *xs = smem + 256;  // [kMmaTok][NL][d/4 + pad]
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) lut[b] = decode_byte((uint32_t)b);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, tig = lane & 3;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int64_t rowb = d / 4;
    const int row0 = blockIdx.y * kMmaRows + warp * 16;  // within the expert
    const uint8_t *const mats[2] = {gate + (int64_t)e * f * rowb, up + (int64_t)e * f * rowb};
    const int rs = d / 4 + kMmaPad;
    for (int q0 = e0; q0 < e1; q0 += kMmaTok) {
        const int nb = min(kMmaTok, e1 - q0);
        __syncthreads();  // table ready (first pass) / previous columns consumed
        mma_stage<NL>(xs, xw, d / 4, ent, q0, nb, k);
        __syncthreads();
        int acc[2][NL][4];
#pragma unroll
        for (int q = 0; q < 2; q++)
#pragma unroll
            for (int l = 0; l < NL; l++) acc[q][l][0] = acc[q][l][1] = acc[q][l][2] = acc[q][l][3] = 0;
        mma_tile<NL, 2>(mats, rowb, row0, f, d, xs, rs, lut, acc);
        // thread holds rows g, g+8 and columns 2*tig, 2*tig+1
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const int j = row0 + g + ((c & 2) ? 8 : 0), col = 2 * tig + (c & 1);
            if (j >= f || col >= nb) continue;
            const int entry = ent[q0 + col];
            const float xsv = xsc[entry / k];
            long long Sg, Su;
            if (NL == 1) {
                Sg = acc[0][0][c];
                Su = acc[1][0][c];
            } else {
                Sg = (long long)acc[0][0][c] * 65536ll + (long long)acc[0][NL > 1 ? 1 : 0][c] * 256ll +
                     (long long)acc[0][NL > 2 ? 2 : 0][c];
                Su = (long long)acc[1][0][c] * 65536ll + (long long)acc[1][NL > 1 ? 1 : 0][c] * 256ll +
                     (long long)acc[1][NL > 2 ? 2 : 0][c];
            }
            const int64_t o = (int64_t)e * f + j;
            float hv;
            if (NL == 1) {
                acc_g[(int64_t)entry * f + j] = (int32_t)Sg;
                acc_u[(int64_t)entry * f + j] = (int32_t)Su;
                const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg), sg[o]), xsv);
                const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su), su[o]), xsv);
                hv = swiglu_f32((double)gv, (double)uv);
            } else {
                const int sh = __float_as_int(xsv);
                hv = swiglu_f32(ldexp((double)Sg, -sh) * (double)sg[o], ldexp((double)Su, -sh) * (double)su[o]);
            }
            h[(int64_t)entry * f + j] = hv;
        }
    }
}

// grid: (n_unique_max, ceil(d / 128)); 8 warps x 16 output rows.
template <int NL>
__global__ void __launch_bounds__(kMmaWarps * 32) down_mma_kernel(
    const uint8_t *__restrict__ down, const float *__restrict__ sd, int d, int f,
    const int32_t *__restrict__ n_unique, const int32_t *__restrict__ uexp, const int32_t *__restrict__ uoff,
    const int32_t *__restrict__ ent, const uint32_t *__restrict__ hw, const float *__restrict__ hsc,
    double *__restrict__ ye, int32_t *__restrict__ acc_d) {
    extern __shared__ __align__(16) uint32_t smem[];
    uint32_t *lut = smem;        // [256] compact decode table
    uint32_t *xs = smem + 256;  // [kMmaTok][NL][f/4 + pad]
    const int u = blockIdx.x;
    if (u >= *n_unique) return;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) lut[b] = decode_byte((uint32_t)b);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, tig = lane & 3;
    const int e = uexp[u], e0 = uoff[u], e1 = uoff[u + 1];
    const int64_t rowb = f / 4;
    const int row0 = blockIdx.y * kMmaRows + warp * 16;
    const uint8_t *const mats[1] = {down + (int64_t)e * d * rowb};
    const int rs = f / 4 + kMmaPad;
    for (int q0 = e0; q0 < e1; q0 += kMmaTok) {
        const int nb = min(kMmaTok, e1 - q0);
        __syncthreads();
        mma_stage<NL>(xs, hw, f / 4, ent, q0, nb, 1);
        __syncthreads();
        int acc[1][NL][4];
#pragma unroll
        for (int l = 0; l < NL; l++) acc[0][l][0] = acc[0][l][1] = acc[0][l][2] = acc[0][l][3] = 0;
        mma_tile<NL, 1>(mats, rowb, row0, d, f, xs, rs, lut, acc);
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const int i = row0 + g + ((c & 2) ? 8 : 0), col = 2 * tig + (c & 1);
            if (i >= d || col >= nb) continue;
            const int entry = ent[q0 + col];
            const float hs = hsc[entry];
            long long S;
            if (NL == 1) S = acc[0][0][c];
            else
                S = (long long)acc[0][0][c] * 65536ll + (long long)acc[0][NL > 1 ? 1 : 0][c] * 256ll +
                    (long long)acc[0][NL > 2 ? 2 : 0][c];
            const float sdv = sd[(int64_t)e * d + i];
            double v;
            if (NL == 1) {
                acc_d[(int64_t)entry * d + i] = (int32_t)S;
                v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S), sdv), hs);
            } else {
                v = ldexp((double)S, -__float_as_int(hs)) * (double)sdv;
            }
            ye[(int64_t)entry * d + i] = v;
        }
    }
}

// ------------------------------------------------------------------------- combine
// y[t,i] = sum over slots (top-k order) of g64[t,slot] * fp32(ye[t*k+slot, i]), in fp64.  The
// expert outputs enter the sum rounded to fp32 (one rounding, 2^-24 relative): that is the
// precision in which the persistent stack kernel passes them between SMs, and both paths give
// the same bits.  On the int8 path ye is an fp32 value already.
__global__ void combine_kernel(const double *__restrict__ g64, const double *__restrict__ ye, int T, int d, int k,
                               uint16_t *__restrict__ y, float *__restrict__ y32, const uint16_t *__restrict__ resid,
                               uint16_t *__restrict__ x_out) {
    const int64_t n = (int64_t)T * d;
    for (int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; p < n; p += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(p / d), i = (int)(p % d);
        double acc = 0.0;
        for (int s = 0; s < k; s++) acc += g64[t * k + s] * (double)(float)ye[((int64_t)t * k + s) * d + i];
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
    return launch_k(rmsnorm_kernel, dim3(T), dim3(256), 0, s, x, d, eps, n);
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
    err = launch_k(prep_kernel<NL>, dim3(T), dim3(256), 0, s, x, (const float *)nullptr, d, w.xw, w.xsc,
                   (const int32_t *)nullptr);
    if (err != cudaSuccess) return err;
    const int umax = (E < T * k) ? E : T * k;
    const int Gd = d / 64, Gf = f / 64;
    if (T >= kMmaGroupedMinT && tc_grouped_supported(d, f)) {  // grouped path on tcgen05 tensor cores
        err = launch_grouped_tc<NL>(L, T, w, s, 0);
        if (err != cudaSuccess) return err;
        err = launch_k(prep_kernel<NL>, dim3(T * k), dim3(128), 0, s, (const uint16_t *)nullptr,
                       (const float *)w.h, f, w.hw, w.hsc, (const int32_t *)nullptr);
        if (err != cudaSuccess) return err;
        err = launch_grouped_tc<NL>(L, T, w, s, 1);
        if (err != cudaSuccess) return err;
        int cg = (T * d + 255) / 256;
        return launch_k(combine_kernel, dim3(cg), dim3(256), 0, s, (const double *)w.g64, (const double *)w.ye, T,
                        d, k, y, y32, resid, x_out);
    }
    if (T >= kMmaGroupedMinT) {  // grouped path on mma.sync (other shapes)
        const dim3 m1(umax, (f + kMmaRows - 1) / kMmaRows), m2(umax, (d + kMmaRows - 1) / kMmaRows);
        const size_t sm1 = 1024 + (size_t)kMmaTok * NL * (d / 4 + kMmaPad) * 4;
        const size_t sm2 = 1024 + (size_t)kMmaTok * NL * (f / 4 + kMmaPad) * 4;
        cudaFuncSetAttribute(gateup_mma_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
        cudaFuncSetAttribute(down_mma_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
        err = launch_k(gateup_mma_kernel<NL>, m1, dim3(kMmaWarps * 32), sm1, s, L->gate, L->up, L->gate_scale,
                       L->up_scale, d, f, k, (const int32_t *)w.n_unique, (const int32_t *)w.uexp,
                       (const int32_t *)w.uoff, (const int32_t *)w.ent, (const uint32_t *)w.xw,
                       (const float *)w.xsc, w.h, w.acc_g, w.acc_u);
        if (err != cudaSuccess) return err;
        err = launch_k(prep_kernel<NL>, dim3(T * k), dim3(128), 0, s, (const uint16_t *)nullptr,
                       (const float *)w.h, f, w.hw, w.hsc, (const int32_t *)nullptr);
        if (err != cudaSuccess) return err;
        err = launch_k(down_mma_kernel<NL>, m2, dim3(kMmaWarps * 32), sm2, s, L->down, L->down_scale, d, f,
                       (const int32_t *)w.n_unique, (const int32_t *)w.uexp, (const int32_t *)w.uoff,
                       (const int32_t *)w.ent, (const uint32_t *)w.hw, (const float *)w.hsc, w.ye, w.acc_d);
        if (err != cudaSuccess) return err;
        int cg = (T * d + 255) / 256;
        return launch_k(combine_kernel, dim3(cg), dim3(256), 0, s, (const double *)w.g64, (const double *)w.ye, T,
                        d, k, y, y32, resid, x_out);
    }
    const int rpb_gu = 32, rpb_dn = 128;
    dim3 g1(umax, (f + rpb_gu - 1) / rpb_gu), g2(umax, (d + rpb_dn - 1) / rpb_dn);
#define TERN_GU_CASE(GG)                                                                                   \
    case GG: {                                                                                             \
        auto kern = gateup_kernel<NL, GG>;                                                                 \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);                \
        err = launch_k(kern, g1, dim3(kFfnWarps * 32), kLutBytes, s, L->gate, L->up, L->gate_scale,  \
                       L->up_scale, d, f, k, (const int32_t *)w.n_unique, (const int32_t *)w.uexp,          \
                       (const int32_t *)w.uoff, (const int32_t *)w.ent, (const uint32_t *)w.xw,            \
                       (const float *)w.xsc, w.h, w.acc_g, w.acc_u, rpb_gu);                               \
        break;                                                                                             \
    }
    switch (Gd) {
        TERN_GU_CASE(1) TERN_GU_CASE(2) TERN_GU_CASE(4) TERN_GU_CASE(8) TERN_GU_CASE(16) TERN_GU_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef TERN_GU_CASE
    if (err != cudaSuccess) return err;
    err = launch_k(prep_kernel<NL>, dim3(T * k), dim3(128), 0, s, (const uint16_t *)nullptr,
                   (const float *)w.h, f, w.hw, w.hsc, (const int32_t *)nullptr);
    if (err != cudaSuccess) return err;
#define TERN_DN_CASE(GG)                                                                                   \
    case GG: {                                                                                             \
        auto kern = down_kernel<NL, GG>;                                                                   \
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);                \
        err = launch_k(kern, g2, dim3(kFfnWarps * 32), kLutBytes, s, L->down, L->down_scale, d, f,   \
                       (const int32_t *)w.n_unique, (const int32_t *)w.uexp, (const int32_t *)w.uoff,       \
                       (const int32_t *)w.ent, (const uint32_t *)w.hw, (const float *)w.hsc, w.ye,         \
                       w.acc_d, rpb_dn);                                                                   \
        break;                                                                                             \
    }
    switch (Gf) {
        TERN_DN_CASE(1) TERN_DN_CASE(2) TERN_DN_CASE(4) TERN_DN_CASE(8) TERN_DN_CASE(16) TERN_DN_CASE(32)
        default: return cudaErrorInvalidValue;
    }
#undef TERN_DN_CASE
    if (err != cudaSuccess) return err;
    int cg = (T * d + 255) / 256;
    return launch_k(combine_kernel, dim3(cg), dim3(256), 0, s, (const double *)w.g64, (const double *)w.ye,
                    T, d, k, y, y32, resid, x_out);
}

cudaError_t launch_ffn_stages(const tern_moe_layer *L, const uint16_t *x, int T, tern_act act, const FfnWs &w,
                              uint16_t *y, float *y_f32, const uint16_t *residual, uint16_t *x_out, cudaStream_t s) {
    if (act == TERN_ACT_INT8) return ffn_stages_nl<1>(L, x, T, w, y, y_f32, residual, x_out, s);
    return ffn_stages_nl<3>(L, x, T, w, y, y_f32, residual, x_out, s);
}

}  // namespace tern
