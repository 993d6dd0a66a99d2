// stack.cu -- persistent whole-stack decode for ONE token (batch 1), sm_100a.
//
// Batch-1 decode streams the active weights layer after layer and is bound by memory
// bandwidth ("How a 20B Model Hits 120 tok/s on an iPhone", "Why the number is plausible";
// "A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What
// Ternary Actually Means").  At d = 2048 one layer moves only 7.4 MB, about a microsecond of
// HBM time on a B200, so the chain router -> top-k -> expert rows -> h -> down -> residual
// is bound by latency, not by bytes.  This kernel therefore:
//   * runs the whole stack in ONE launch: one CTA per SM, co-resident (cooperative launch),
//     three bounded grid barriers per layer (after the router logits, after h, after x');
//   * gives every CTA a fixed share of each layer's bytes and moves it with TMA bulk copies
//     (cp.async.bulk, global -> shared, mbarrier completion), issued as early as the data
//     dependencies allow: the next layer's router rows during the current layer, and a
//     CTA's gate/up AND down rows together as soon as top-k is known -- the down rows do not
//     depend on h, so they land while gate/up is computed;
//   * decodes the packed bytes in registers (one table read + one dp4a per limb per byte).
//
// Per layer l (x_l in global memory, bf16):
//   A  every CTA: n = bf16(x / sqrt(mean x^2 + eps)) (fp64), its router rows -> logits (fp64)
//   -- grid barrier --
//   B  every CTA: top-k + gates (identical in every CTA), issue its TMA copies
//   C  its (slot, row) pairs of gate/up -> h = silu(g) * u (fp64 epilogue) -> global
//   -- grid barrier --
//   D  every CTA: limbs of all h; its output rows: down for every slot, gate-weighted sum in
//      top-k order (fp64), bf16, residual add -> x_{l+1}
//   -- grid barrier --
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include "kernels.h"
#include "tern_common.cuh"

namespace tern {

constexpr int kStackWarps = 16;
constexpr int kStackThreads = kStackWarps * 32;
constexpr int kMaxStackLayers = 64;
constexpr int kSK = 8;  // max experts per token on this path
constexpr int kMaxTraceCtas = 256;

struct StackParams {
    StackLayerDev layer[kMaxStackLayers];
    int n_layers, d, f, E, k;
    double eps;
    uint16_t *x;          // [d] in/out
    unsigned int *bar;    // [0] arrivals, [1] leavers
    double *logits;       // [E]
    float *H;             // [k][f]
    uint16_t *hist;       // [n_layers+1][d]  x before each layer and after the last
    int32_t *idx_hist;    // [n_layers][k]
    double *gate_hist;    // [n_layers][k]
    int *status;
    long long limit_ns;   // bound on every in-kernel wait
    unsigned long long *ttrace;  // [n_layers][P][16] %globaltimer stamps of every CTA at phase boundaries
    // static work split (host computed)
    int P;                // CTAs
    int rb_rows;          // max router rows per CTA
    int gu_pairs;         // max gate/up pairs per CTA
    int dn_rows;          // max output rows per CTA
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
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

// bounded grid barrier on a monotonic arrival counter (zero at launch, reset by the last
// CTA to leave).  Returns false on timeout.
__device__ __forceinline__ bool stack_grid_sync(unsigned int *arrive, unsigned int target, long long limit_ns,
                                                int *status, int *s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        red_release_gpu_add(arrive, 1u);
        int ok = 1;
        if ((int)(ld_acquire_gpu(arrive) - target) < 0) {
            const unsigned long long t0 = gtimer();
            while ((int)(ld_acquire_gpu(arrive) - target) < 0) {
                if ((long long)(gtimer() - t0) > limit_ns) {
                    ok = 0;
                    set_status(status, TERN_ETIMEOUT);
                    break;
                }
            }
        }
        *s_ok = ok;
    }
    __syncthreads();
    return *s_ok != 0;
}

__device__ __forceinline__ double block_sum_f64(double v, double *red) {
    v = warp_sum_f64(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = (l < kStackWarps) ? red[l] : 0.0;
    r = warp_sum_f64(r);
    __syncthreads();
    return r;
}

__device__ __forceinline__ float block_max_nonneg(float v, float *red) {
    v = warp_max_f32(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    float r = (l < kStackWarps) ? red[l] : 0.0f;
    r = warp_max_f32(r);
    __syncthreads();
    return r;
}

// ------------------------------------------------------------------ the kernel
// Shared memory map (bytes): lut | router rows | gate rows | up rows | down rows | x | n |
// h limbs | small arrays.  D = d elements, F = f elements.
struct SmemMap {
    uint32_t lut, rbuf, gbuf, ubuf, dbuf, xs, ns, xl, hl, total;
};

__host__ __device__ inline uint32_t align128(uint32_t v) { return (v + 127u) & ~127u; }

__host__ __device__ inline SmemMap smem_map(int d, int f, int k, int rb_rows, int gu_pairs, int dn_rows, int NL) {
    SmemMap m;
    uint32_t p = 0;
    m.lut = p;
    p = align128(p + kLutBytes);
    m.rbuf = p;
    p = align128(p + (uint32_t)rb_rows * d * 2);
    m.gbuf = p;
    p = align128(p + (uint32_t)gu_pairs * (d / 4));
    m.ubuf = p;
    p = align128(p + (uint32_t)gu_pairs * (d / 4));
    m.dbuf = p;
    p = align128(p + (uint32_t)k * dn_rows * (f / 4));
    m.xs = p;
    p = align128(p + (uint32_t)d * 2);
    m.ns = p;
    p = align128(p + (uint32_t)d * 2);
    m.xl = p;
    p = align128(p + (uint32_t)NL * (d / 64) * kSegPad * 4);
    m.hl = p;
    p = align128(p + (uint32_t)k * NL * (f / 64) * kSegPad * 4);
    m.total = p;
    return m;
}

template <int NL>
__global__ void __launch_bounds__(kStackThreads, 1) stack_kernel(const __grid_constant__ StackParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_router, mb_gu, mb_dn;
    __shared__ double s_red[32];
    __shared__ float s_redf[32];
    __shared__ double s_part[kStackWarps][kStackWarps];
    __shared__ double s_logit[1024];
    __shared__ int s_idx[kSK];
    __shared__ double s_gate[kSK];
    __shared__ int s_hshift[kSK];
    __shared__ float s_hscale[kSK];
    __shared__ double s_ye[64][kSK];
    __shared__ float s_sg[64], s_su[64], s_sd[kSK * 64];
    __shared__ unsigned int s_hmax[kSK];
    __shared__ int s_ok;
    __shared__ double s_r;
    __shared__ float s_nscale;  // int8: s_x ; bf16: shift as int bits

    const int d = p.d, f = p.f, E = p.E, k = p.k, P = p.P;
    const int c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const SmemMap sm = smem_map(d, f, k, p.rb_rows, p.gu_pairs, p.dn_rows, NL);
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem + sm.lut);
    uint16_t *rbuf = reinterpret_cast<uint16_t *>(smem + sm.rbuf);
    uint8_t *gbuf = smem + sm.gbuf;
    uint8_t *ubuf = smem + sm.ubuf;
    uint8_t *dbuf = smem + sm.dbuf;
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem + sm.xs);
    uint16_t *ns = reinterpret_cast<uint16_t *>(smem + sm.ns);
    uint32_t *xl = reinterpret_cast<uint32_t *>(smem + sm.xl);
    uint32_t *hl = reinterpret_cast<uint32_t *>(smem + sm.hl);
    const int xlp = (d / 64) * kSegPad;  // padded words per limb of n
    const int hlp = (f / 64) * kSegPad;  // padded words per limb of one slot's h

    // static shares of this CTA
    const int nr = (E - c + P - 1) / P;                        // router rows: c, c+P, ...
    const int NPt = k * f;
    const int p0 = (int)((long long)c * NPt / P), p1 = (int)((long long)(c + 1) * NPt / P);
    const int i0 = (int)((long long)c * d / P), i1 = (int)((long long)(c + 1) * d / P);
    const int nrows = i1 - i0;
    const long long lim = p.limit_ns;
    unsigned int bar_target = 0;
    bool alive = true;
    unsigned int n_rt = 0, n_gu = 0, n_dn = 0;  // phases issued per mbarrier (thread 0)

    unsigned long long *tt = (tid == 0) ? p.ttrace : nullptr;
#define TSTAMP(l, ph) \
    if (tt) tt[((size_t)(l) * P + c) * 16 + (ph)] = gtimer();

    lut_fill(lut);
    if (tid == 0) {
        mbar_init(&mb_router, 1);
        mbar_init(&mb_gu, 1);
        mbar_init(&mb_dn, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // router rows of layer 0
    if (tid == 0 && nr > 0) {
        mbar_expect_tx(&mb_router, (uint32_t)(nr * d * 2));
        n_rt++;
        for (int r = 0; r < nr; r++)
            bulk_g2s(rbuf + (size_t)r * d, p.layer[0].router + (size_t)(c + r * P) * d, (uint32_t)(d * 2), &mb_router);
    }

    for (int l = 0; l < p.n_layers && alive; l++) {
        const StackLayerDev &Ly = p.layer[l];
        const uint32_t par = (uint32_t)(l & 1);
        const uint16_t *xin = (l == 0) ? p.x : p.hist + (size_t)l * d;
        // ---------------------------------------------------------------- A: norm + router
        TSTAMP(l, 0)
        double ss = 0.0;
        for (int i4 = tid; i4 < d / 4; i4 += kStackThreads) {
            const uint2 v4 = __ldcg(reinterpret_cast<const uint2 *>(xin) + i4);
            reinterpret_cast<uint2 *>(xs)[i4] = v4;
            const uint16_t bb[4] = {(uint16_t)(v4.x & 0xFFFFu), (uint16_t)(v4.x >> 16), (uint16_t)(v4.y & 0xFFFFu),
                                    (uint16_t)(v4.y >> 16)};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const double v = (double)bf16_to_f32(bb[e]);
                ss = fma(v, v, ss);
            }
        }
        ss = block_sum_f64(ss, s_red);
        if (tid == 0) s_r = sqrt(ss / (double)d + p.eps);
        if (l == 0 && c == 0)
            for (int i = tid; i < d; i += kStackThreads) p.hist[i] = xs[i];
        __syncthreads();
        const double r = s_r;
        float amax = 0.0f;
        for (int i = tid; i < d; i += kStackThreads) {
            const uint16_t nb = f64_to_bf16_rne((double)bf16_to_f32(xs[i]) / r);
            ns[i] = nb;
            amax = fmaxf(amax, fabsf(bf16_to_f32(nb)));
        }
        amax = block_max_nonneg(amax, s_redf);
        TSTAMP(l, 1)
        if (tid == 0) {
            if (NL == 1) s_nscale = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
            else s_nscale = __int_as_float(fixed_shift(amax));
        }
        // router rows (prefetched): each row split over kStackWarps / rb_rows warps
        if (nr > 0) {
            const bool okw = mbar_wait(&mb_router, par, lim, p.status);
            alive = __syncthreads_and(okw ? 1 : 0) && alive;
            const int wpr = kStackWarps / p.rb_rows;  // warps per row (rb_rows <= 16)
            const int rr = warp / wpr, part = warp % wpr;
            double acc = 0.0;
            if (rr < nr) {
                const int per = d / wpr;
                const uint16_t *wrow = rbuf + (size_t)rr * d + part * per;
                const uint16_t *nrow = ns + part * per;
                for (int i = lane; i < per; i += 32)
                    acc = fma((double)bf16_to_f32(wrow[i]), (double)bf16_to_f32(nrow[i]), acc);
            }
            acc = warp_sum_f64(acc);
            if (lane == 0 && rr < nr) s_part[rr][part] = acc;
            __syncthreads();
            if (tid < nr) {
                double s = 0.0;
                for (int q = 0; q < wpr; q++) s += s_part[tid][q];
                p.logits[c + tid * P] = s;
            }
        }
        __syncthreads();
        // prefetch the next layer's router rows into the now free buffer
        if (tid == 0 && nr > 0 && l + 1 < p.n_layers) {
            mbar_expect_tx(&mb_router, (uint32_t)(nr * d * 2));
            n_rt++;
            for (int q = 0; q < nr; q++)
                bulk_g2s(rbuf + (size_t)q * d, p.layer[l + 1].router + (size_t)(c + q * P) * d, (uint32_t)(d * 2),
                         &mb_router);
        }
        TSTAMP(l, 2)
        bar_target += (unsigned)P;
        if (!stack_grid_sync(p.bar, bar_target, lim, p.status, &s_ok) || !alive) {
            alive = false;
            break;
        }
        // ---------------------------------------------------------------- B: top-k, issue copies
        TSTAMP(l, 3)
        for (int e = tid; e < E; e += kStackThreads) s_logit[e] = __ldcg(p.logits + e);
        __syncthreads();
        if (warp == 0) {
            if (E <= 256) warp_topk<8>(s_logit, E, k, s_idx, s_gate, nullptr);
            else warp_topk<32>(s_logit, E, k, s_idx, s_gate, nullptr);
            __syncwarp();
            if (lane == 0 && c == 0)
                for (int q = 0; q < k; q++) {
                    p.idx_hist[l * k + q] = s_idx[q];
                    p.gate_hist[l * k + q] = s_gate[q];
                }
        }
        __syncthreads();
        TSTAMP(l, 4)
        if (tid == 0) {
            // gate/up rows of this CTA's (slot,row) pairs, then its down rows for every slot
            const uint32_t rowb = (uint32_t)(d / 4);
            mbar_expect_tx(&mb_gu, (uint32_t)(2 * (p1 - p0)) * rowb);
            n_gu++;
            int q = 0;
            for (int pp = p0; pp < p1;) {
                const int s = pp / f, j = pp % f;
                const int cnt = min(p1 - pp, f - j);
                const size_t src = ((size_t)s_idx[s] * f + j) * rowb;
                bulk_g2s(gbuf + (size_t)q * rowb, Ly.gate + src, (uint32_t)cnt * rowb, &mb_gu);
                bulk_g2s(ubuf + (size_t)q * rowb, Ly.up + src, (uint32_t)cnt * rowb, &mb_gu);
                q += cnt;
                pp += cnt;
            }
            const uint32_t rowd = (uint32_t)(f / 4);
            mbar_expect_tx(&mb_dn, (uint32_t)(k * nrows) * rowd);
            n_dn++;
            for (int s = 0; s < k; s++)
                bulk_g2s(dbuf + (size_t)s * p.dn_rows * rowd, Ly.down + ((size_t)s_idx[s] * d + i0) * rowd,
                         (uint32_t)nrows * rowd, &mb_dn);
        }
        TSTAMP(l, 5)
        // per-row scales of this CTA's rows, fetched while the weight copies are in flight
        for (int q = tid; q < p1 - p0; q += kStackThreads) {
            const int pp = p0 + q, s2 = pp / f, j = pp % f;
            const size_t o = (size_t)s_idx[s2] * f + j;
            s_sg[q] = __ldg(Ly.sg + o);
            s_su[q] = __ldg(Ly.su + o);
        }
        for (int q = tid; q < k * nrows; q += kStackThreads)
            s_sd[q] = __ldg(Ly.sd + (size_t)s_idx[q / nrows] * d + i0 + q % nrows);
        TSTAMP(l, 6)
        // activation limbs of n: one word (4 elements) per thread into the padded layout,
        // then every lane loads the limbs of its segment (G = d/64 lanes per row)
        {
            const int sh = __float_as_int(s_nscale);
            const float inv = (NL == 1 && amax > 0.0f) ? quant_inv(amax) : 0.0f;
            for (int w = tid; w < d / 4; w += kStackThreads) {
                const uint2 v4 = reinterpret_cast<const uint2 *>(ns)[w];
                const uint16_t bb[4] = {(uint16_t)(v4.x & 0xFFFFu), (uint16_t)(v4.x >> 16), (uint16_t)(v4.y & 0xFFFFu),
                                        (uint16_t)(v4.y >> 16)};
                uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const float v = bf16_to_f32(bb[e]);
                    if (NL == 1) {
                        w0 |= ((uint32_t)(amax > 0.0f ? quant_one(v, inv) : 0) & 0xFFu) << (8 * e);
                    } else {
                        uint32_t h, m, lo;
                        fixed_limbs(v, sh, h, m, lo);
                        w0 |= h << (8 * e);
                        w1 |= m << (8 * e);
                        w2 |= lo << (8 * e);
                    }
                }
                const int pw = padded_word(w);
                xl[pw] = w0;
                if (NL > 1) {
                    xl[xlp + pw] = w1;
                    xl[2 * xlp + pw] = w2;
                }
            }
        }
        __syncthreads();
        SegX<NL> X;
        seg_load_x_padded<NL>(X, xl, xlp, lane % (d / 64));
        // ---------------------------------------------------------------- C: gate/up -> h
        if (p1 > p0) {
            const bool okw = mbar_wait(&mb_gu, par, lim, p.status);
            alive = __syncthreads_and(okw ? 1 : 0) && alive;
            TSTAMP(l, 7)
            const uint32_t *lut_lane = lut + lane;
            const int rowb = d / 4;
            for (int q = warp; q < p1 - p0; q += kStackWarps) {
                const int pp = p0 + q, s = pp / f, j = pp % f;
                const uint4 wg = *reinterpret_cast<const uint4 *>(gbuf + (size_t)q * rowb + lane * 16);
                const uint4 wu = *reinterpret_cast<const uint4 *>(ubuf + (size_t)q * rowb + lane * 16);
                int ag[NL], au[NL];
#pragma unroll
                for (int z = 0; z < NL; z++) ag[z] = au[z] = 0;
                seg_dot<NL>(wg, X, lut_lane, ag);
                seg_dot<NL>(wu, X, lut_lane, au);
                int ga, gb2, ua, ub;
                acc_to_pair<NL>(ag, ga, gb2);
                acc_to_pair<NL>(au, ua, ub);
                ga = group_sum<32>(ga);
                ua = group_sum<32>(ua);
                if (NL > 1) {
                    gb2 = group_sum<32>(gb2);
                    ub = group_sum<32>(ub);
                }
                if (lane == 0) {
                    const long long Sg = pair_value(NL, ga, gb2), Su = pair_value(NL, ua, ub);
                    const float sg = s_sg[q], su = s_su[q];
                    float hv;
                    if (NL == 1) {
                        const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg), sg), s_nscale);
                        const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su), su), s_nscale);
                        hv = swiglu_f32((double)gv, (double)uv);
                    } else {
                        const int sh = __float_as_int(s_nscale);
                        hv = swiglu_f32(ldexp((double)Sg, -sh) * (double)sg, ldexp((double)Su, -sh) * (double)su);
                    }
                    p.H[(size_t)s * f + j] = hv;
                }
            }
        }
        TSTAMP(l, 8)
        bar_target += (unsigned)P;
        if (!stack_grid_sync(p.bar, bar_target, lim, p.status, &s_ok) || !alive) {
            alive = false;
            break;
        }
        // ---------------------------------------------------------------- D: down + combine + residual
        {
            // every slot's h, read once from L2; per-slot absmax via shared atomics
            TSTAMP(l, 9)
            const int wpl = f / 4;  // float4 (= limb words) per slot
            constexpr int kMaxV = 8;
            float4 hv[kMaxV];
            if (tid < kSK) s_hmax[tid] = 0u;
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kMaxV; j++) {
                const int w = tid + j * kStackThreads;
                if (w < k * wpl) {
                    hv[j] = __ldcg(reinterpret_cast<const float4 *>(p.H) + w);
                    const float m4 = fmaxf(fmaxf(fabsf(hv[j].x), fabsf(hv[j].y)), fmaxf(fabsf(hv[j].z), fabsf(hv[j].w)));
                    atomicMax(&s_hmax[w / wpl], __float_as_uint(m4));
                }
            }
            __syncthreads();
            if (tid < k) {
                const float a = __uint_as_float(s_hmax[tid]);
                if (NL == 1) {
                    s_hscale[tid] = a > 0.0f ? __fdiv_rn(a, 127.0f) : 0.0f;
                    s_hshift[tid] = __float_as_int(a);  // keep absmax for the quantiser
                } else {
                    s_hshift[tid] = fixed_shift(a);
                }
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < kMaxV; j++) {
                const int w = tid + j * kStackThreads;
                if (w >= k * wpl) continue;
                const int ss2 = w / wpl, b = w % wpl;
                const float vv[4] = {hv[j].x, hv[j].y, hv[j].z, hv[j].w};
                uint32_t w0 = 0, w1 = 0, w2 = 0;
                if (NL == 1) {
                    const float a = __int_as_float(s_hshift[ss2]);
                    const float inv = a > 0.0f ? quant_inv(a) : 0.0f;
#pragma unroll
                    for (int e = 0; e < 4; e++) w0 |= ((uint32_t)(a > 0.0f ? quant_one(vv[e], inv) : 0) & 0xFFu) << (8 * e);
                    hl[(size_t)ss2 * hlp + padded_word(b)] = w0;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        uint32_t h, mi, lo;
                        fixed_limbs(vv[e], s_hshift[ss2], h, mi, lo);
                        w0 |= h << (8 * e);
                        w1 |= mi << (8 * e);
                        w2 |= lo << (8 * e);
                    }
                    hl[((size_t)ss2 * NL + 0) * hlp + padded_word(b)] = w0;
                    hl[((size_t)ss2 * NL + (NL > 1 ? 1 : 0)) * hlp + padded_word(b)] = w1;
                    hl[((size_t)ss2 * NL + (NL > 2 ? 2 : 0)) * hlp + padded_word(b)] = w2;
                }
            }
            __syncthreads();
            TSTAMP(l, 10)
            if (nrows > 0) {
                const bool okw = mbar_wait(&mb_dn, par, lim, p.status);
                alive = __syncthreads_and(okw ? 1 : 0) && alive;
            }
            TSTAMP(l, 11)
            // (row, slot) pairs, G = f/64 lanes each; 512-wide rows -> 8 lanes, 4 pairs per warp pass
            const int G = f / 64;
            const int ppw = 32 / G;
            const int sub = lane / G, gl = lane % G;
            const uint32_t *lut_lane = lut + lane;
            const int npairs = nrows * k;
            for (int base = warp * ppw; base < npairs; base += kStackWarps * ppw) {
                const int pi = base + sub;
                const bool valid = pi < npairs;
                const int rrow = valid ? pi / k : 0, sl = valid ? pi % k : 0;
                SegX<NL> Hx;
                seg_load_x_padded<NL>(Hx, hl + (size_t)sl * NL * hlp, hlp, gl);
                int acc[NL];
#pragma unroll
                for (int z = 0; z < NL; z++) acc[z] = 0;
                const uint4 wd = *reinterpret_cast<const uint4 *>(dbuf + ((size_t)sl * p.dn_rows + rrow) * (f / 4) + gl * 16);
                seg_dot<NL>(wd, Hx, lut_lane, acc);
                int a, b;
                acc_to_pair<NL>(acc, a, b);
                // reduce within the G lanes of this pair (G = 8 for f = 512)
                for (int o = G / 2; o > 0; o >>= 1) {
                    a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
                    if (NL > 1) b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
                }
                if (valid && gl == 0) {
                    const long long S = pair_value(NL, a, b);
                    const float sd = s_sd[sl * nrows + rrow];
                    double v;
                    if (NL == 1) v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S), sd), s_hscale[sl]);
                    else v = ldexp((double)S, -s_hshift[sl]) * (double)sd;
                    s_ye[rrow][sl] = v;
                }
            }
            __syncthreads();
            TSTAMP(l, 12)
            const bool last = (l + 1 == p.n_layers);
            if (tid < nrows) {
                double y = 0.0;
                for (int q = 0; q < k; q++) y += s_gate[q] * s_ye[tid][q];
                const uint16_t yb = f64_to_bf16_rne(y);
                const int i = i0 + tid;
                const uint16_t xo = f64_to_bf16_rne((double)bf16_to_f32(xs[i]) + (double)bf16_to_f32(yb));
                p.hist[(size_t)(l + 1) * d + i] = xo;
                if (last) p.x[i] = xo;
            }
            TSTAMP(l, 13)
            if (!last) {
                bar_target += (unsigned)P;
                if (!stack_grid_sync(p.bar, bar_target, lim, p.status, &s_ok) || !alive) {
                    alive = false;
                    break;
                }
            }
        }
    }
#undef TSTAMP
    // after a timeout, let this CTA's own copies in flight land (bounded) before leaving
    if (!alive && tid == 0) {
        if (n_rt) mbar_wait(&mb_router, (n_rt - 1) & 1u, lim, p.status);
        if (n_gu) mbar_wait(&mb_gu, (n_gu - 1) & 1u, lim, p.status);
        if (n_dn) mbar_wait(&mb_dn, (n_dn - 1) & 1u, lim, p.status);
    }
    // leave: the last CTA out resets the barrier counters for the next launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned int n = atomicAdd(p.bar + 1, 1u);
        if (n == (unsigned)P - 1) {
            atomicExch(p.bar + 0, 0u);
            atomicExch(p.bar + 1, 0u);
        }
    }
}

// ------------------------------------------------------------------ host side
// Persistent-path workspace: barrier words, logits [E], H [k][f], x history
// [(kMaxStackLayers+1)][d], routing history [kMaxStackLayers][k] (int32 + fp64).
struct StackWs {
    int64_t bar, logits, H, hist, idx_hist, gate_hist, ttrace, total;
};

static inline int64_t up256_(int64_t v) { return (v + 255) & ~int64_t(255); }

static StackWs stack_ws_layout(const tern_moe_layer *L0) {
    StackWs o{};
    int64_t p = 0;
    auto take = [&](int64_t b) {
        const int64_t r = p;
        p = up256_(p + b);
        return r;
    };
    o.bar = take(256);
    o.logits = take((int64_t)L0->E * 8);
    o.H = take((int64_t)L0->k * L0->f * 4);
    o.hist = take((int64_t)(kMaxStackLayers + 1) * L0->d * 2);
    o.idx_hist = take((int64_t)kMaxStackLayers * L0->k * 4);
    o.gate_hist = take((int64_t)kMaxStackLayers * L0->k * 8);
    o.ttrace = take((int64_t)kMaxStackLayers * kMaxTraceCtas * 16 * 8);
    o.total = p;
    return o;
}

size_t stack_persistent_ws_bytes(const tern_moe_layer *L0) { return (size_t)stack_ws_layout(L0).total; }

void stack_persistent_offsets(const tern_moe_layer *L0, int64_t *hist, int64_t *idx_hist, int64_t *gate_hist,
                              int64_t *ttrace) {
    const StackWs o = stack_ws_layout(L0);
    *hist = o.hist;
    *idx_hist = o.idx_hist;
    *gate_hist = o.gate_hist;
    *ttrace = o.ttrace;
}

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

struct StackPlan {
    int P, rb_rows, gu_pairs, dn_rows;
    SmemMap sm;
    const void *fn;
};

static tern_status stack_plan(const tern_moe_layer &L0, int n_layers, tern_act act, StackPlan &pl) {
    if (n_layers > kMaxStackLayers || L0.d != 2048 || L0.k > kSK || L0.f % 64 || L0.f > 2048) return TERN_EUNSUPPORTED;
    const int64_t g = L0.f / 64;
    if ((g & (g - 1)) != 0) return TERN_EUNSUPPORTED;
    pl.P = sm_count();
    if (pl.P <= 0) return TERN_ECUDA;
    if (pl.P > kMaxTraceCtas) pl.P = kMaxTraceCtas;
    pl.rb_rows = (L0.E + pl.P - 1) / pl.P;
    pl.gu_pairs = (int)((L0.k * L0.f + pl.P - 1) / pl.P);
    pl.dn_rows = (int)((L0.d + pl.P - 1) / pl.P);
    if (pl.rb_rows > kStackWarps || pl.dn_rows > 64 || pl.gu_pairs > 64 || L0.k * L0.f > 8 * 4 * kStackThreads)
        return TERN_EUNSUPPORTED;
    const int NL = act == TERN_ACT_INT8 ? 1 : 3;
    pl.sm = smem_map((int)L0.d, (int)L0.f, L0.k, pl.rb_rows, pl.gu_pairs, pl.dn_rows, NL);
    pl.fn = act == TERN_ACT_INT8 ? (const void *)stack_kernel<1> : (const void *)stack_kernel<3>;
    if (cudaFuncSetAttribute(pl.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.sm.total) != cudaSuccess)
        return TERN_ECUDA;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, pl.fn, kStackThreads, pl.sm.total) != cudaSuccess)
        return TERN_ECUDA;
    if (nb < 1) return TERN_EUNSUPPORTED;
    return TERN_OK;
}

bool stack_persistent_supported(const tern_moe_layer *L0, int n_layers, tern_act act) {
    StackPlan pl;
    return stack_plan(*L0, n_layers, act, pl) == TERN_OK;
}

tern_status launch_stack_persistent(const tern_moe_layer *layers, int n_layers, uint16_t *x, float eps, tern_act act,
                                    void *ws, size_t ws_bytes, int *status, cudaStream_t s) {
    const tern_moe_layer &L0 = layers[0];
    StackPlan pl;
    const tern_status pst = stack_plan(L0, n_layers, act, pl);
    if (pst != TERN_OK) return pst;
    const int P = pl.P, rb_rows = pl.rb_rows, gu_pairs = pl.gu_pairs, dn_rows = pl.dn_rows;
    const StackWs o = stack_ws_layout(&L0);
    if (ws_bytes < (size_t)o.total) return TERN_EWORKSPACE;
    if (!status) return TERN_ECUDA;

    StackParams prm;
    memset(&prm, 0, sizeof(prm));
    for (int l = 0; l < n_layers; l++) {
        prm.layer[l].gate = layers[l].gate;
        prm.layer[l].up = layers[l].up;
        prm.layer[l].down = layers[l].down;
        prm.layer[l].sg = layers[l].gate_scale;
        prm.layer[l].su = layers[l].up_scale;
        prm.layer[l].sd = layers[l].down_scale;
        prm.layer[l].router = layers[l].router;
    }
    char *b = static_cast<char *>(ws);
    prm.n_layers = n_layers;
    prm.d = (int)L0.d;
    prm.f = (int)L0.f;
    prm.E = L0.E;
    prm.k = L0.k;
    prm.eps = (double)eps;
    prm.x = x;
    prm.bar = reinterpret_cast<unsigned int *>(b + o.bar);
    prm.logits = reinterpret_cast<double *>(b + o.logits);
    prm.H = reinterpret_cast<float *>(b + o.H);
    prm.hist = reinterpret_cast<uint16_t *>(b + o.hist);
    prm.idx_hist = reinterpret_cast<int32_t *>(b + o.idx_hist);
    prm.gate_hist = reinterpret_cast<double *>(b + o.gate_hist);
    prm.ttrace = reinterpret_cast<unsigned long long *>(b + o.ttrace);
    prm.status = status;
    prm.limit_ns = 1000000000ll;  // every in-kernel wait gives up after one second
    prm.P = P;
    prm.rb_rows = rb_rows;
    prm.gu_pairs = gu_pairs;
    prm.dn_rows = dn_rows;

    const SmemMap sm = pl.sm;
    const void *fn = pl.fn;
    void *args[] = {&prm};
    const cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(P), dim3(kStackThreads), args, sm.total, s);
    return e == cudaSuccess ? TERN_OK : TERN_ECUDA;
}

}  // namespace tern
