// stack.cu -- persistent whole-stack decode for ONE token (batch 1), sm_100a.
//
// Batch-1 decode streams the active weights layer after layer and is bound by memory
// bandwidth ("How a 20B Model Hits 120 tok/s on an iPhone", "Why the number is plausible";
// "A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What
// Ternary Actually Means").  At d = 2048 one layer moves only 7.4 MB, about a microsecond of
// HBM time on a B200, so the chain router -> top-k -> expert rows -> h -> down -> residual
// is bound by latency, not by bytes.  This kernel therefore:
//   * runs the whole stack in ONE launch: one CTA per SM, all co-resident (cooperative
//     launch), no kernel boundary between layers;
//   * exchanges data between CTAs with flag-carrying 64-bit words: {32-bit payload, 32-bit
//     tag}, written and read as single 64-bit accesses (single-copy atomic), where the tag
//     names the launch and the layer.  A consumer polls the data itself, so each exchange
//     costs one L2 round trip instead of a barrier plus a read, and no arrival counter has
//     to be reset between launches;
//   * gives every CTA a fixed share of each layer's bytes and moves it with TMA bulk copies
//     (cp.async.bulk global -> shared, mbarrier completion) as early as the dependencies
//     allow: the next layer's router rows during the current layer; a CTA's gate/up AND down
//     rows together as soon as top-k is known (the down rows do not depend on h);
//   * decodes the packed bytes in registers (one table read + one dp4a per limb per byte).
//
// Per layer l, in every CTA (P = #SMs CTAs):
//   A  x_l (exchange) -> sum of squares and absmax in one block reduction -> n = bf16(x/r),
//      activation limbs; its router rows (prefetched) -> logits -> exchange
//   B  all logits -> top-k + gates -> TMA copies of its gate/up pairs and down rows
//   C  its (slot,row) gate/up pairs -> h = silu(g) * u (fp64 epilogue, one thread per row)
//      -> exchange
//   D  all h -> limbs; its output rows: down for every slot, gate-weighted sum in top-k order
//      (fp64), bf16, residual add -> x_{l+1} -> exchange
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

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
    uint16_t *x;                  // [d] in/out
    unsigned int *ctl;            // [0] CTAs that left this launch, [1] launch epoch
    unsigned long long *xll;      // [d/2]  {two bf16 of x_{l}, tag}
    unsigned long long *lll;      // [2E]   {high / low word of the fp64 logit, tag}
    unsigned long long *hll;      // [k*f]  {fp32 h, tag}
    uint16_t *hist;               // [n_layers+1][d]  x before each layer and after the last
    int32_t *idx_hist;            // [n_layers][k]
    double *gate_hist;            // [n_layers][k]
    int *status;
    long long limit_ns;           // bound on every in-kernel wait
    unsigned long long *ttrace;   // [n_layers][P][16] %globaltimer stamps of every CTA, then
                                  // [n_layers][P][16] clock64 stamps (SM cycles) at the same points
    int P;                        // CTAs
    int rb_rows;                  // max router rows per CTA
    int gu_pairs;                 // max gate/up pairs per CTA
    int dn_rows;                  // max output rows per CTA (even)
};

// ------------------------------------------------------------------ exchange words
// ---- flag-carrying words: one 64-bit access carries payload and tag together
__device__ __forceinline__ void ll_store(unsigned long long *p, uint32_t val, uint32_t tag) {
    const unsigned long long w = ((unsigned long long)tag << 32) | (unsigned long long)val;
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ll_load(const unsigned long long *p) {
    unsigned long long w;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}

// Gather n tagged words (n*8 bytes, 16-byte aligned) from global memory into shared memory
// with one TMA bulk copy, then check every tag in shared memory; re-fetch until all carry
// `tag`.  One bulk copy per CTA replaces thousands of per-thread polls of the same hot L2
// lines (measured on B200: 1.3-1.6 us per 148-CTA exchange instead of 1.5-2.9 us).  Called
// by every thread of the CTA; `phase` is the mbarrier phase counter (same in every thread).
// Returns false (uniformly) on timeout, status set.
__device__ __forceinline__ bool ll_gather(const unsigned long long *src, int n, uint32_t tag,
                                          unsigned long long *dst, uint64_t *mb, uint32_t &phase, long long limit_ns,
                                          int *status) {
    const unsigned long long t0 = gtimer();
    while (true) {
        if (threadIdx.x == 0) {
            mbar_expect_tx(mb, (uint32_t)(n * 8));
            bulk_g2s(dst, src, (uint32_t)(n * 8), mb);
        }
        const bool landed = mbar_wait(mb, phase & 1u, limit_ns, status);
        phase++;
        int mine = landed ? 1 : 0;
        for (int w = threadIdx.x; w < n; w += blockDim.x)
            if ((uint32_t)(dst[w] >> 32) != tag) mine = 0;
        if (__syncthreads_and(mine)) return true;
        // uniform timeout decision: thread 0's clock, broadcast by the barrier below
        const int late = (threadIdx.x == 0) && ((long long)(gtimer() - t0) > limit_ns);
        if (__syncthreads_or(late)) {
            set_status(status, TERN_ETIMEOUT);
            return false;
        }
    }
}

// ------------------------------------------------------------------ shared memory map
struct SmemMap {
    uint32_t lut, rbuf, gbuf, ubuf, dbuf, xs, ns, xl, hl, xch, total;
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
    m.xch = p;  // exchange landing buffer: max(d/2, 2E, k*f) words
    {
        uint32_t nw = (uint32_t)(d / 2);
        if ((uint32_t)(2 * 256) > nw) nw = 2 * 256;
        if ((uint32_t)(k * f) > nw) nw = (uint32_t)(k * f);
        p = align128(p + nw * 8);
    }
    m.total = p;
    return m;
}

// limb words of four consecutive values v[0..3] (one word per limb)
template <int NL>
__device__ __forceinline__ void limb_words(const float (&v)[4], int sh_or_unused, float inv, bool nonzero,
                                           uint32_t (&w)[3]) {
    w[0] = w[1] = w[2] = 0;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        if (NL == 1) {
            w[0] |= ((uint32_t)(nonzero ? quant_one(v[e], inv) : 0) & 0xFFu) << (8 * e);
        } else {
            uint32_t h, m, lo;
            fixed_limbs(v[e], sh_or_unused, h, m, lo);
            w[0] |= h << (8 * e);
            w[1] |= m << (8 * e);
            w[2] |= lo << (8 * e);
        }
    }
}

// ------------------------------------------------------------------ the kernel
template <int NL>
__global__ void __launch_bounds__(kStackThreads, 1) stack_kernel(const __grid_constant__ StackParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_router, mb_gu0, mb_gu1, mb_dn, mb_x;
    __shared__ __align__(8) uint64_t mb_h[kSK];        // per-slot h fetch
    __shared__ int s_hok[kSK][kStackWarps], s_hlate[kSK];
    __shared__ float s_hpart[kSK][kStackWarps];
    __shared__ unsigned int s_hissued[kSK];
    __shared__ double s_red[kStackWarps];
    __shared__ float s_redf[kStackWarps];
    __shared__ double s_part[kStackWarps][kStackWarps];
    __shared__ double s_logit[256];
    __shared__ __align__(16) uint32_t s_gm[32];  // top-k scratch
    __shared__ int s_nc;
    __shared__ ulonglong2 s_cand[256];
    __shared__ int s_idx[kSK];
    __shared__ double s_gate[kSK];
    __shared__ long long s_S[64][2];
    __shared__ double s_ye[64][kSK];
    __shared__ float s_sg[64], s_su[64], s_sd[kSK * 64];
    // the layers' pointers, copied once: a dynamically indexed kernel parameter is a constant
    // cache line fetched from L2 on the critical path of every layer
    __shared__ StackLayerDev s_layer[kMaxStackLayers];

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
    unsigned long long *xch = reinterpret_cast<unsigned long long *>(smem + sm.xch);
    const int xlp = (d / 64) * kSegPad;  // padded words per limb of n
    const int hlp = (f / 64) * kSegPad;  // padded words per limb of one slot's h

    // static shares of this CTA
    const int nr = (E - c + P - 1) / P;  // router rows: c, c+P, ...
    const int NPt = k * f;
    const int p0 = (int)((long long)c * NPt / P), p1 = (int)((long long)(c + 1) * NPt / P);
    const int i0 = 2 * (int)((long long)c * (d / 2) / P), i1 = 2 * (int)((long long)(c + 1) * (d / 2) / P);
    const int nrows = i1 - i0;
    const long long lim = p.limit_ns;
    const uint32_t ep = ld_acquire_gpu(p.ctl + 1);  // launch epoch, advanced by the previous launch
    bool alive = true;
    unsigned int n_rt = 0, n_gu = 0, n_dn = 0;  // phases issued per mbarrier (thread 0)
    uint32_t xph = 0;                            // phase counter of the exchange mbarrier
    uint32_t hph = 0;                            // phase counter of this warp's slot mbarrier
    // gate/up pairs arrive in two halves (first 16 pairs, then the rest) so the dots of the
    // first half overlap the second half's transfer
    const int npairs = p1 - p0;
    const int n0 = npairs < kStackWarps ? npairs : kStackWarps;
    const int n1 = npairs - n0;

    unsigned long long *tt = (tid == 0) ? p.ttrace : nullptr;
    const size_t ctr_off = (size_t)p.n_layers * P * 16;
#define TSTAMP(l, ph)                                              \
    if (tt) {                                                      \
        const size_t o_ = ((size_t)(l) * P + c) * 16 + (ph);       \
        tt[o_] = gtimer();                                         \
        tt[ctr_off + o_] = (unsigned long long)clock64();          \
    }

    lut_fill(lut);
    {
        constexpr int kW = (int)(sizeof(StackLayerDev) / sizeof(uint64_t));
        static_assert(sizeof(StackLayerDev) % sizeof(uint64_t) == 0, "pointer table");
        for (int q = tid; q < p.n_layers * kW; q += kStackThreads)
            reinterpret_cast<uint64_t *>(s_layer)[q] = reinterpret_cast<const uint64_t *>(p.layer)[q];
    }
    if (tid == 0) {
        mbar_init(&mb_router, 1);
        mbar_init(&mb_gu0, 1);
        mbar_init(&mb_gu1, 1);
        mbar_init(&mb_dn, 1);
        mbar_init(&mb_x, 1);
        for (int q = 0; q < kSK; q++) {
            mbar_init(&mb_h[q], 1);
            s_hissued[q] = 0u;
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0 && nr > 0) {  // router rows of layer 0
        mbar_expect_tx(&mb_router, (uint32_t)(nr * d * 2));
        n_rt++;
        for (int r = 0; r < nr; r++)
            bulk_g2s(rbuf + (size_t)r * d, s_layer[0].router + (size_t)(c + r * P) * d, (uint32_t)(d * 2), &mb_router);
    }

    for (int l = 0; l < p.n_layers && alive; l++) {
        const StackLayerDev &Ly = s_layer[l];
        const uint32_t par = (uint32_t)(l & 1);
        const uint32_t tag = (ep << 7) | (uint32_t)(l + 1);  // never 0 (a zeroed workspace holds 0)
        TSTAMP(l, 0)
        if (tid < 3 && c < 32) {
            // one L2 prefetch per 2 MB page of this layer's gate, up and down arrays: the
            // address translations are in place before top-k sends the row copies there
            const uint8_t *base = tid == 0 ? Ly.gate : (tid == 1 ? Ly.up : Ly.down);
            const size_t off = (size_t)c << 21;
            if (off < (size_t)E * f * (d / 4)) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + off));
        }
        if (tid == 0) {
            // this layer's transfer sizes depend only on the CTA's share, not on the routing:
            // register them now so the copies can be issued the moment top-k is known
            mbar_expect_tx(&mb_gu0, (uint32_t)(2 * n0 * (d / 4)));
            mbar_expect_tx(&mb_gu1, (uint32_t)(2 * n1 * (d / 4)));
            mbar_expect_tx(&mb_dn, (uint32_t)(k * nrows * (f / 4)));
            n_gu++;
            n_dn++;
        }
        // ------------------------------------------------------------ A: x_l, norm, limbs
        // thread t owns elements 4t..4t+3 (d = 2048 = 4 * 512)
        float xv[4];
        {
            bool ok = true;
            uint32_t pr[2] = {0, 0};
            if (l == 0) {
                const uint2 v4 = __ldcg(reinterpret_cast<const uint2 *>(p.x) + tid);
                pr[0] = v4.x;
                pr[1] = v4.y;
            } else {
                ok = ll_gather(p.xll, d / 2, tag, xch, &mb_x, xph, lim, p.status);
                pr[0] = (uint32_t)xch[2 * tid];
                pr[1] = (uint32_t)xch[2 * tid + 1];
            }
            alive = __syncthreads_and(ok ? 1 : 0) && alive;
            reinterpret_cast<uint2 *>(xs)[tid] = make_uint2(pr[0], pr[1]);
            xv[0] = bf16_to_f32((uint16_t)(pr[0] & 0xFFFFu));
            xv[1] = bf16_to_f32((uint16_t)(pr[0] >> 16));
            xv[2] = bf16_to_f32((uint16_t)(pr[1] & 0xFFFFu));
            xv[3] = bf16_to_f32((uint16_t)(pr[1] >> 16));
        }
        TSTAMP(l, 1)
        if (l == 0 && c == 0) reinterpret_cast<uint2 *>(p.hist)[tid] = reinterpret_cast<const uint2 *>(xs)[tid];
        double r;
        float amax_n;
        {
            double ss = 0.0;
            float am = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const double v = (double)xv[e];
                ss = fma(v, v, ss);
                am = fmaxf(am, fabsf(xv[e]));
            }
            ss = warp_sum_f64(ss);
            am = warp_max_f32(am);
            if (lane == 0) {
                s_red[warp] = ss;
                s_redf[warp] = am;
            }
            __syncthreads();
            // every thread folds the 16 warp partials in the same order: same r everywhere
            double ts = 0.0;
            float ta = 0.0f;
#pragma unroll
            for (int w = 0; w < kStackWarps; w++) {
                ts += s_red[w];
                ta = fmaxf(ta, s_redf[w]);
            }
            r = sqrt(ts / (double)d + p.eps);
            // rounding is monotone, so max |bf16(x_k / r)| = bf16(max |x_k| / r)
            amax_n = bf16_to_f32(f64_to_bf16_rne((double)ta / r));
        }
        const float s_nq = (NL == 1) ? (amax_n > 0.0f ? __fdiv_rn(amax_n, 127.0f) : 0.0f) : 0.0f;
        const int sh_n = (NL == 1) ? 0 : fixed_shift(amax_n);
        {
            float nv[4];
            uint16_t nb[4];
#pragma unroll
            for (int e = 0; e < 4; e++) {
                nb[e] = f64_to_bf16_rne((double)xv[e] / r);
                nv[e] = bf16_to_f32(nb[e]);
            }
            reinterpret_cast<uint2 *>(ns)[tid] =
                make_uint2((uint32_t)nb[0] | ((uint32_t)nb[1] << 16), (uint32_t)nb[2] | ((uint32_t)nb[3] << 16));
            uint32_t w[3];
            const float inv = (NL == 1 && amax_n > 0.0f) ? quant_inv(amax_n) : 0.0f;
            limb_words<NL>(nv, sh_n, inv, amax_n > 0.0f, w);
            const int pw = padded_word(tid);
            xl[pw] = w[0];
            if (NL > 1) {
                xl[xlp + pw] = w[1];
                xl[2 * xlp + pw] = w[2];
            }
        }
        __syncthreads();
        TSTAMP(l, 2)
        // router rows (prefetched): each row split over kStackWarps / rb_rows warps
        if (nr > 0) {
            const bool okw = mbar_wait(&mb_router, par, lim, p.status);
            alive = __syncthreads_and(okw ? 1 : 0) && alive;
            const int wpr = kStackWarps / p.rb_rows;
            const int rr = warp / wpr, part = warp % wpr;
            double acc = 0.0;
            if (rr < nr) {
                const int per = d / wpr;
                const uint16_t *wrow = rbuf + (size_t)rr * d + part * per;
                const uint16_t *nrow = ns + part * per;
                // bf16 x bf16 has at most 16 significant bits: the product is exact in fp64 and
                // the fma adds it with one rounding
                for (int i = lane; i < per; i += 32)
                    acc = fma((double)bf16_to_f32(wrow[i]), (double)bf16_to_f32(nrow[i]), acc);
            }
            acc = warp_sum_f64(acc);
            if (lane == 0 && rr < nr) s_part[rr][part] = acc;
            __syncthreads();
            if (tid < nr) {
                double sum = 0.0;
                for (int q = 0; q < wpr; q++) sum += s_part[tid][q];
                const unsigned long long b = (unsigned long long)__double_as_longlong(sum);
                const int e = c + tid * P;
                ll_store(p.lll + 2 * e, (uint32_t)(b >> 32), tag);
                ll_store(p.lll + 2 * e + 1, (uint32_t)b, tag);
            }
        }
        TSTAMP(l, 3)
        __syncthreads();
        if (tid == 0 && nr > 0 && l + 1 < p.n_layers) {  // next layer's router rows
            mbar_expect_tx(&mb_router, (uint32_t)(nr * d * 2));
            n_rt++;
            for (int q = 0; q < nr; q++)
                bulk_g2s(rbuf + (size_t)q * d, s_layer[l + 1].router + (size_t)(c + q * P) * d, (uint32_t)(d * 2),
                         &mb_router);
        }
        // ------------------------------------------------------------ B: logits, top-k, copies
        double my_logit = 0.0;  // logit `tid` (E <= 256 on this path)
        {
            const bool ok = ll_gather(p.lll, 2 * E, tag, xch, &mb_x, xph, lim, p.status);
            if (tid < E) {
                my_logit = __longlong_as_double(
                    (long long)(((unsigned long long)(uint32_t)xch[2 * tid] << 32) | (uint32_t)xch[2 * tid + 1]));
                s_logit[tid] = my_logit;
            }
            alive = __syncthreads_and(ok ? 1 : 0) && alive;
        }
        TSTAMP(l, 4)
        // only the expert indices are on the critical path; the gates are needed in the combine
        block_topk_select(my_logit, E, k, s_idx, s_gm, &s_nc, s_cand);
        TSTAMP(l, 5)
        if (warp == 0) {
            // copies: lanes 0..3 first-half gate/up segments, 4..7 second half (each half spans
            // at most two slots x two matrices), lanes 8.. down rows of slot lane-8
            const uint32_t rowb = (uint32_t)(d / 4), rowd = (uint32_t)(f / 4);
            if (lane < 8) {
                const int half = lane >> 2, seg = (lane >> 1) & 1;
                const int h0 = p0 + (half ? n0 : 0), h1 = half ? p1 : p0 + n0;  // pairs of this half
                const int s0 = h0 / f;
                const int e0 = min(h1, (s0 + 1) * f);
                const int a = seg == 0 ? h0 : e0, b = seg == 0 ? e0 : h1;
                if (b > a) {
                    const int s = a / f, j = a % f;
                    const size_t src = ((size_t)s_idx[s] * f + j) * rowb;
                    const int q0 = a - p0;
                    uint64_t *mb = half ? &mb_gu1 : &mb_gu0;
                    if (lane & 1) bulk_g2s(ubuf + (size_t)q0 * rowb, Ly.up + src, (uint32_t)(b - a) * rowb, mb);
                    else bulk_g2s(gbuf + (size_t)q0 * rowb, Ly.gate + src, (uint32_t)(b - a) * rowb, mb);
                }
            } else if (lane < 8 + k && nrows > 0) {
                const int s = lane - 8;
                bulk_g2s(dbuf + (size_t)s * p.dn_rows * rowd, Ly.down + ((size_t)s_idx[s] * d + i0) * rowd,
                         (uint32_t)nrows * rowd, &mb_dn);
            }
        } else {
            // per-row scales of this CTA's rows, fetched while the copies are in flight
            for (int q = tid - 32; q < p1 - p0; q += kStackThreads - 32) {
                const int pp = p0 + q, s2 = pp / f, j = pp % f;
                const size_t o = (size_t)s_idx[s2] * f + j;
                s_sg[q] = __ldg(Ly.sg + o);
                s_su[q] = __ldg(Ly.su + o);
            }
            for (int q = tid - 32; q < k * nrows; q += kStackThreads - 32)
                s_sd[q] = __ldg(Ly.sd + (size_t)s_idx[q / nrows] * d + i0 + q % nrows);
            if (warp == kStackWarps - 1) {
                warp_topk_gates(s_logit, k, s_idx, s_gate, nullptr);
                __syncwarp();
                if (lane < k && c == 0) {
                    p.idx_hist[l * k + lane] = s_idx[lane];
                    p.gate_hist[l * k + lane] = s_gate[lane];
                }
            }
        }
        TSTAMP(l, 6)
        // ------------------------------------------------------------ C: gate/up -> h
        if (p1 > p0) {
            // activation limbs of this lane's segment (G = d/64 = 32 lanes per row)
            SegX<NL> X;
            seg_load_x_padded<NL>(X, xl, xlp, lane % (d / 64));
            const uint32_t lane4 = (uint32_t)lane << 2;
            const int rowb = d / 4;
            for (int half = 0; half < 2; half++) {
                const int qa = half ? n0 : 0, qb = half ? npairs : n0;
                if (qb <= qa) break;
                const bool okw = mbar_wait(half ? &mb_gu1 : &mb_gu0, par, lim, p.status);
                alive = __syncthreads_and(okw ? 1 : 0) && alive;
                if (half == 0) TSTAMP(l, 7)
                for (int q = qa + warp; q < qb; q += kStackWarps) {
                    const uint4 wg = *reinterpret_cast<const uint4 *>(gbuf + (size_t)q * rowb + lane * 16);
                    const uint4 wu = *reinterpret_cast<const uint4 *>(ubuf + (size_t)q * rowb + lane * 16);
                    int ag[NL], au[NL];
#pragma unroll
                    for (int z = 0; z < NL; z++) ag[z] = au[z] = 0;
                    seg_dot<NL>(wg, X, lut, lane4, ag);
                    seg_dot<NL>(wu, X, lut, lane4, au);
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
                        s_S[q][0] = pair_value(NL, ga, gb2);
                        s_S[q][1] = pair_value(NL, ua, ub);
                    }
                }
            }
            __syncthreads();
            TSTAMP(l, 8)
            // SwiGLU epilogue, one thread per row, fp64
            if (tid < p1 - p0) {
                const int q = tid, pp = p0 + q, s = pp / f, j = pp % f;
                const long long Sg = s_S[q][0], Su = s_S[q][1];
                float hv;
                if (NL == 1) {
                    const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg), s_sg[q]), s_nq);
                    const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su), s_su[q]), s_nq);
                    hv = swiglu_f32((double)gv, (double)uv);
                } else {
                    hv = swiglu_f32(ldexp((double)Sg, -sh_n) * (double)s_sg[q], ldexp((double)Su, -sh_n) * (double)s_su[q]);
                }
                ll_store(p.hll + (size_t)s * f + j, __float_as_uint(hv), tag);
            }
        }
        TSTAMP(l, 9)
        // ------------------------------------------------------------ D: down, combine, residual
        {
            // Each slot is owned by wps = 16/k warps.  They fetch that slot's h (f tagged words)
            // with one TMA copy, agree on its tags over a per-slot hardware barrier, build its
            // limbs and run their down rows -- without waiting for the other slots.
            const int G = f / 64;
            const int rpp = 32 / G;
            const int wps = kStackWarps / k;
            const int sl = warp / wps, wi = warp % wps;
            const int nthr = wps * 32;
            const int bar_id = 1 + sl;
            unsigned long long *hb = xch + (size_t)sl * f;
            const int share = f / wps;  // words of the slot this warp checks and converts
            bool okg = true;
            {
                const unsigned long long t0 = gtimer();
                while (true) {
                    if (wi == 0 && lane == 0) {
                        mbar_expect_tx(&mb_h[sl], (uint32_t)(f * 8));
                        bulk_g2s(hb, p.hll + (size_t)sl * f, (uint32_t)(f * 8), &mb_h[sl]);
                        s_hissued[sl]++;
                    }
                    const bool landed = mbar_wait(&mb_h[sl], hph & 1u, lim, p.status);
                    hph++;
                    int mine = landed ? 1 : 0;
                    for (int w = wi * share + lane; w < (wi + 1) * share; w += 32)
                        if ((uint32_t)(hb[w] >> 32) != tag) mine = 0;
                    mine = __all_sync(0xFFFFFFFFu, mine);
                    if (lane == 0) s_hok[sl][wi] = mine;
                    named_bar_sync(bar_id, nthr);
                    int all = 1;
                    for (int q = 0; q < wps; q++) all &= s_hok[sl][q];
                    if (wi == 0 && lane == 0) s_hlate[sl] = (!all) && ((long long)(gtimer() - t0) > lim);
                    named_bar_sync(bar_id, nthr);
                    if (all) break;
                    if (s_hlate[sl]) {
                        set_status(p.status, TERN_ETIMEOUT);
                        okg = false;
                        break;
                    }
                }
            }
            // slot absmax -> shift (bf16 path) or scale (int8 path); identical in the slot's warps
            float m = 0.0f;
            for (int w = wi * share + lane; w < (wi + 1) * share; w += 32)
                m = fmaxf(m, fabsf(__uint_as_float((uint32_t)hb[w])));
            m = warp_max_f32(m);
            if (lane == 0) s_hpart[sl][wi] = m;
            named_bar_sync(bar_id, nthr);
            float a = 0.0f;
            for (int q = 0; q < wps; q++) a = fmaxf(a, s_hpart[sl][q]);
            const int hsh = (NL == 1) ? 0 : fixed_shift(a);
            const float hinv = (NL == 1 && a > 0.0f) ? quant_inv(a) : 0.0f;
            const float hsc = (NL == 1 && a > 0.0f) ? __fdiv_rn(a, 127.0f) : 0.0f;
            // limb words of this warp's share of the slot (4 values per word)
            for (int bw = wi * (share / 4) + lane; bw < (wi + 1) * (share / 4); bw += 32) {
                const float v4[4] = {__uint_as_float((uint32_t)hb[4 * bw]), __uint_as_float((uint32_t)hb[4 * bw + 1]),
                                     __uint_as_float((uint32_t)hb[4 * bw + 2]), __uint_as_float((uint32_t)hb[4 * bw + 3])};
                uint32_t wd[3];
                limb_words<NL>(v4, hsh, hinv, a > 0.0f, wd);
                hl[((size_t)sl * NL + 0) * hlp + padded_word(bw)] = wd[0];
                if (NL > 1) {
                    hl[((size_t)sl * NL + 1) * hlp + padded_word(bw)] = wd[1];
                    hl[((size_t)sl * NL + 2) * hlp + padded_word(bw)] = wd[2];
                }
            }
            named_bar_sync(bar_id, nthr);
            if (warp == 0) TSTAMP(l, 10)
            if (nrows > 0 && !mbar_wait(&mb_dn, par, lim, p.status)) okg = false;
            if (warp == 0) TSTAMP(l, 11)
            if (warp == 0) TSTAMP(l, 12)
            // down rows of this slot: G lanes per row, rpp rows per warp pass
            {
                const int sub = lane / G, gl = lane % G;
                const uint32_t lane4 = (uint32_t)lane << 2;
                SegX<NL> Hx;
                seg_load_x_padded<NL>(Hx, hl + (size_t)sl * NL * hlp, hlp, gl);
                for (int r0 = wi * rpp; r0 < nrows; r0 += wps * rpp) {
                    const int rrow = r0 + sub;
                    const bool valid = rrow < nrows;
                    int acc[NL];
#pragma unroll
                    for (int z = 0; z < NL; z++) acc[z] = 0;
                    const uint4 wd = *reinterpret_cast<const uint4 *>(
                        dbuf + ((size_t)sl * p.dn_rows + (valid ? rrow : 0)) * (f / 4) + gl * 16);
                    seg_dot<NL>(wd, Hx, lut, lane4, acc);
                    int aa, bb;
                    acc_to_pair<NL>(acc, aa, bb);
                    for (int o = G / 2; o > 0; o >>= 1) {
                        aa += __shfl_xor_sync(0xFFFFFFFFu, aa, o);
                        if (NL > 1) bb += __shfl_xor_sync(0xFFFFFFFFu, bb, o);
                    }
                    if (valid && gl == 0) {
                        const long long S = pair_value(NL, aa, bb);
                        const float sd = s_sd[sl * nrows + rrow];
                        double v;
                        if (NL == 1) v = (double)__fmul_rn(__fmul_rn(__int2float_rn((int)S), sd), hsc);
                        else v = ldexp((double)S, -hsh) * (double)sd;
                        s_ye[rrow][sl] = v;
                    }
                }
            }
            alive = __syncthreads_and(okg ? 1 : 0) && alive;
            TSTAMP(l, 13)
            const bool last = (l + 1 == p.n_layers);
            // one output row per thread, fixed top-k order; row pairs leave as one word
            uint16_t xo = 0;
            if (tid < nrows) {
                double y = 0.0;
                for (int q = 0; q < k; q++) y += s_gate[q] * s_ye[tid][q];
                const uint16_t yb = f64_to_bf16_rne(y);
                xo = f64_to_bf16_rne((double)bf16_to_f32(xs[i0 + tid]) + (double)bf16_to_f32(yb));
            }
            const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, (uint32_t)xo, 1);
            if (tid < nrows && (tid & 1) == 0) {
                const uint32_t pr = (uint32_t)xo | (other << 16);
                const int i = i0 + tid;
                reinterpret_cast<uint32_t *>(p.hist + (size_t)(l + 1) * d)[i / 2] = pr;
                if (last) reinterpret_cast<uint32_t *>(p.x)[i / 2] = pr;
                else ll_store(p.xll + i / 2, pr, (ep << 7) | (uint32_t)(l + 2));
            }
            TSTAMP(l, 14)
        }
    }
#undef TSTAMP
    // after a timeout, let this CTA's own copies in flight land (bounded) before leaving
    if (!alive && tid == 0) {
        if (n_rt) mbar_wait(&mb_router, (n_rt - 1) & 1u, lim, p.status);
        if (n_gu) {
            mbar_wait(&mb_gu0, (n_gu - 1) & 1u, lim, p.status);
            mbar_wait(&mb_gu1, (n_gu - 1) & 1u, lim, p.status);
        }
        if (n_dn) mbar_wait(&mb_dn, (n_dn - 1) & 1u, lim, p.status);
        if (xph) mbar_wait(&mb_x, (xph - 1) & 1u, lim, p.status);
        for (int q = 0; q < kSK; q++)
            if (s_hissued[q]) mbar_wait(&mb_h[q], (s_hissued[q] - 1) & 1u, lim, p.status);
    }
    // leave: the last CTA out advances the launch epoch (the next launch's tags differ)
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned int n = atomicAdd(p.ctl, 1u);
        if (n == (unsigned)P - 1) {
            atomicExch(p.ctl, 0u);
            atomicAdd(p.ctl + 1, 1u);
        }
    }
}

// ------------------------------------------------------------------ host side
// Persistent-path workspace: barrier words, logits [E], H [k][f], x history
// [(kMaxStackLayers+1)][d], routing history [kMaxStackLayers][k] (int32 + fp64).
struct StackWs {
    int64_t ctl, xll, lll, hll, hist, idx_hist, gate_hist, ttrace, total;
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
    o.ctl = take(256);
    o.xll = take((int64_t)L0->d / 2 * 8);
    o.lll = take((int64_t)L0->E * 2 * 8);
    o.hll = take((int64_t)L0->k * L0->f * 8);
    o.hist = take((int64_t)(kMaxStackLayers + 1) * L0->d * 2);
    o.idx_hist = take((int64_t)kMaxStackLayers * L0->k * 4);
    o.gate_hist = take((int64_t)kMaxStackLayers * L0->k * 8);
    o.ttrace = take((int64_t)2 * kMaxStackLayers * kMaxTraceCtas * 16 * 8);
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
    pl.dn_rows = 2 * (int)((L0.d / 2 + pl.P - 1) / pl.P);
    // the thread mappings assume d = 4 * threads and k * f = 8 * threads at most, and a CTA's
    // gate/up pairs spanning at most two slots
    if (pl.rb_rows > kStackWarps || pl.dn_rows > 64 || pl.gu_pairs > 64 || pl.gu_pairs > L0.f ||
        L0.k * L0.f > 8 * kStackThreads || (L0.k * L0.f) % 8 || L0.d != 4 * kStackThreads || L0.E > 256 || kStackWarps % L0.k)
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
    prm.ctl = reinterpret_cast<unsigned int *>(b + o.ctl);
    prm.xll = reinterpret_cast<unsigned long long *>(b + o.xll);
    prm.lll = reinterpret_cast<unsigned long long *>(b + o.lll);
    prm.hll = reinterpret_cast<unsigned long long *>(b + o.hll);
    prm.hist = reinterpret_cast<uint16_t *>(b + o.hist);
    prm.idx_hist = reinterpret_cast<int32_t *>(b + o.idx_hist);
    prm.gate_hist = reinterpret_cast<double *>(b + o.gate_hist);
    // phase stamps cost a %globaltimer read and a store each: only when TERNMOE_TRACE=1
    const char *tenv = getenv("TERNMOE_TRACE");
    prm.ttrace = (tenv && tenv[0] == '1') ? reinterpret_cast<unsigned long long *>(b + o.ttrace) : nullptr;
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
