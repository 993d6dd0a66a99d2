// stack.cu -- persistent whole-stack decode for ONE token (batch 1), sm_100a.
//
// Batch-1 decode streams the active weights layer after layer and is bound by memory
// bandwidth ("How a 20B Model Hits 120 tok/s on an iPhone", "Why the number is plausible";
// "A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What
// Ternary Actually Means").  At d = 2048 a layer moves only 7.4 MB, about a microsecond of
// HBM time on a B200, so the chain x -> norm -> router -> top-k -> expert rows -> h -> down
// -> residual is bound by the latency of its steps, not by bytes.  This kernel:
//   * runs the whole stack in ONE launch: P = k * G CTAs, one per SM, co-resident
//     (cooperative launch); no kernel boundary between layers;
//   * is slot-major: CTA (s, c) -- group s, part c of G -- works only on the expert chosen at
//     rank s of the top-k: a contiguous block of its gate/up rows and of its down rows, moved
//     by three bulk copies (TMA, mbarrier completion) the moment top-k is known;
//   * exchanges data between CTAs through flag-carrying 64-bit words {32-bit payload, 32-bit
//     tag} in global memory, stored and polled with single 64-bit relaxed accesses at GPU
//     scope (each word is single-copy atomic, so a reader sees the payload that belongs to
//     the tag it reads; no fence is needed because nothing else is read).  The tag names the
//     launch and the layer.  Four exchanges per layer, three of them inside small groups:
//       logits  every CTA computes <= 2 router rows and publishes them; all CTAs read all;
//       h       the G CTAs of a group publish their h; the group reads the slot's f values;
//       y       the k CTAs with the same part c (one per slot) publish their slot's output
//               rows, rounded to fp32; each reads the k outputs of its rows and sums them;
//       x       the G CTAs of a group publish x' for their rows (+ the sum of squares and
//               the absmax of those rows); the group reads the whole vector;
//     every exchange buffer has two copies (layer parity), see "buffer reuse" below;
//   * prefetches the next layer's experts to L2: with its own n it also computes its router
//     rows of the NEXT layer (fp32, a prediction only), the CTAs exchange these, and group s
//     prefetches its rows of predicted experts s and s + 8 (kPredTop = 12 in all) while the
//     current layer runs.  A prefetch changes no value; it only moves the HBM reads of
//     correctly predicted experts off the critical path;
//   * decodes the packed bytes in registers by integer logic (decode.cuh): no lookup table.
//
// Per layer l, in CTA (s, c):
//   A  x_l (exchange x, or the input at l = 0) -> r = sqrt(sum x^2 / d + eps) from the parts'
//      sums, n = bf16(x / r), activation limbs; router rows -> logits -> publish; the next
//      layer's router rows -> predicted logits -> publish
//   B  all logits -> top-k (one warp) -> bulk copies of this CTA's gate/up and down rows of
//      expert idx[s]; meanwhile other warps load the rows' scales, compute the gates and
//      issue the L2 prefetches of the predicted next-layer experts
//   C  gate/up dots -> h = silu(g) * u (fp64, one thread per row) -> exchange h
//   D  h limbs -> down dots -> y_s rows (fp32) -> exchange y -> y = sum_q g_q y_q in top-k
//      order (fp64) -> x' = bf16(x + bf16(y)) -> exchange x
//
// Buffer reuse.  Each exchange buffer is written at layer l and again at layer l + 2 (same
// parity).  A CTA writes its layer-(l+2) words only after it has read the layer-(l+1) words
// of every other producer of the same exchange, and each of those producers wrote them only
// after reading the layer-l words: so no word is overwritten before every consumer has read
// it.  The tag carries the launch epoch (advanced by the last CTA to leave), so a fresh launch
// never matches words left by an earlier one and the workspace needs no clearing between
// calls.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "cluster.cuh"
#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

namespace tern {

constexpr int kStackWarps = 16;
constexpr int kStackThreads = kStackWarps * 32;
constexpr int kSK = 8;              // max experts per token on this path
constexpr int kMaxTraceCtas = 256;
constexpr int kMaxGroup = 32;       // CTAs per slot group
constexpr int kMaxGU = 32;          // gate/up rows per CTA (two chunks of 16)
constexpr int kMaxDN = 128;         // down rows per CTA
constexpr int kMaxRouterRows = 8;   // router rows per CTA
constexpr int kPredTop = 10;        // at least this many predicted next-layer experts go to L2
constexpr int kMaxPrefetch = 2;     // predicted experts one slot group prefetches (3 warps each)
constexpr int kTracePoints = 24;
constexpr long long kPredictWaitCycles = 10000;  // the prediction exchange is a hint: give up after ~5 us

struct StackParams {
    StackLayerDev layer[kMaxLayers];
    int n_layers, d, f, E, k;
    double eps;
    uint16_t *x;                  // [d] in/out
    unsigned int *ctl;            // [0] CTAs that left this launch, [1] launch epoch
    unsigned long long *xb;       // [2][k][d/2]        {two bf16 of x, tag}
    unsigned long long *xst;      // [2][k][G][4]       {sum x^2 hi, lo, absmax, 0} of each part, tagged
    unsigned long long *lb;       // [2][E][2]          {fp64 logit hi, lo}, tagged
    unsigned long long *pb;       // [2][E]             {fp32 predicted next-layer logit}, tagged
    unsigned long long *hb;       // [2][k][f]          {fp32 h}, tagged
    unsigned long long *yb;       // [2][G][k][kMaxDN]  {fp32 expert output row}, tagged
    uint16_t *hist;               // [n_layers+1][d]  x before each layer and after the last
    int32_t *idx_hist;            // [n_layers][k]
    double *gate_hist;            // [n_layers][k]
    float *y_hist;                // [n_layers][d]    FFN output before the bf16 cast
    float *h_hist;                // [n_layers][k][f] SwiGLU output of each slot
    int *status;
    long long limit_ns;           // bound on every in-kernel wait
    unsigned long long *ttrace;   // [n_layers][P][16] %globaltimer stamps, then the same for clock64
    int P, G;
    int stall_layer;              // test hook: at this layer CTA 0 waits for an h tag nobody writes
    int predict;                  // 1: prefetch predicted next-layer experts to L2
};

// ------------------------------------------------------------------ tagged words
__device__ __forceinline__ unsigned long long tagged(uint32_t payload, uint32_t tag) {
    return ((unsigned long long)tag << 32) | (unsigned long long)payload;
}
__device__ __forceinline__ void st_word(unsigned long long *p, uint32_t payload, uint32_t tag) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(tagged(payload, tag)) : "memory");
}

// Poll the pair of tagged words at src until both carry `tag`; false once `limit` SM cycles
// have passed since t0 (clock64, cheaper than %globaltimer inside a poll loop).
__device__ __forceinline__ bool poll_pair(const unsigned long long *src, uint32_t tag, long long t0, long long limit,
                                          ulonglong2 &out) {
    while (true) {
        out = ld_relaxed_v2(src);
        if ((uint32_t)(out.x >> 32) == tag && (uint32_t)(out.y >> 32) == tag) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// CTA-wide AND over the threads of hardware barrier `id` (nthreads, a multiple of 32)
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------ shared memory map
struct SmemMap {
    uint32_t gbuf, ubuf, dbuf, rbuf0, rbuf1, xs, ns, xl, hl, lg, hv, yv, cand, total;
};

__host__ __device__ inline uint32_t align128(uint32_t v) { return (v + 127u) & ~127u; }

__host__ __device__ inline SmemMap smem_map(int d, int f, int k, int gu_max, int dn_max, int rb_max, int NL) {
    SmemMap m;
    uint32_t p = 0;
    auto take = [&](uint32_t bytes) {
        const uint32_t r = p;
        p = align128(p + bytes);
        return r;
    };
    m.gbuf = take((uint32_t)gu_max * (d / 4));
    m.ubuf = take((uint32_t)gu_max * (d / 4));
    m.dbuf = take((uint32_t)dn_max * (f / 4));
    m.rbuf0 = take((uint32_t)rb_max * d * 2);
    m.rbuf1 = take((uint32_t)rb_max * d * 2);
    m.xs = take((uint32_t)d * 2);
    m.ns = take((uint32_t)d * 2);
    m.xl = take((uint32_t)NL * (d / 64) * kSegPad * 4);
    m.hl = take((uint32_t)NL * (f / 64) * kSegPad * 4);
    m.lg = take(256 * 8);
    m.hv = take((uint32_t)f * 4);
    m.yv = take((uint32_t)k * kMaxDN * 4);
    m.cand = take(256 * 16);
    m.total = p;
    return m;
}

// ------------------------------------------------------------------ the kernel
// PRED: the next-layer prediction side task is compiled in (an option, off by default); the
// default instantiation carries none of its code, which keeps the per-layer code smaller
template <int NL, bool PRED>
__global__ void __launch_bounds__(kStackThreads, 1) stack_kernel(const __grid_constant__ StackParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_r[2], mb_gu0, mb_gu1, mb_dn;
    __shared__ double s_red[kStackWarps];
    __shared__ float s_redf[kStackWarps];
    __shared__ double s_rp[kStackWarps][kMaxRouterRows];
    __shared__ float s_pp[kStackWarps][kMaxRouterRows];
    __shared__ double s_xss[kMaxGroup];
    __shared__ float s_xam[kMaxGroup];
    __shared__ int32_t s_idx[kSK];
    __shared__ __align__(16) uint32_t s_tkm[32];  // top-k scratch
    __shared__ double s_gate[kSK];
    __shared__ long long s_S[kMaxGU][2];
    // scales of this CTA's rows, bulk-copied with the rows: a 16-byte aligned superset of the
    // range, so entry q is at [q + offset], offset < 4
    __shared__ __align__(16) float s_sgb[kMaxGU + 8], s_sub[kMaxGU + 8], s_sdb[kMaxDN + 8];
    __shared__ float s_hmax[kStackWarps];
    __shared__ int32_t s_pf[kMaxPrefetch];  // next-layer experts this CTA prefetches
    __shared__ int s_npf;
    // the layers' pointers, copied once: a dynamically indexed kernel parameter is a constant
    // cache line fetched from L2 on the critical path of every layer
    __shared__ StackLayerDev s_layer[kMaxLayers];

    const int d = p.d, f = p.f, E = p.E, k = p.k, P = p.P, G = p.G;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pid = blockIdx.x, s = pid / G, c = pid % G;
    // this CTA's shares: gate/up rows [j0, j1), down rows [i0, i1) (even bounds), router rows [e0, e1)
    const int j0 = (c * f) / G, j1 = ((c + 1) * f) / G, ngu = j1 - j0;
    const int i0 = 2 * ((c * (d / 2)) / G), i1 = 2 * (((c + 1) * (d / 2)) / G), ndn = i1 - i0;
    const int e0 = (E * pid) / P, e1 = (E * (pid + 1)) / P, nr = e1 - e0;
    const int n0 = ngu < 16 ? ngu : 16, n1 = ngu - n0;  // gate/up rows in the first / second copy
    const int gu_max = (f + G - 1) / G, dn_max = 2 * ((d / 2 + G - 1) / G), rb_max = (E + P - 1) / P;
    const SmemMap sm = smem_map(d, f, k, gu_max, dn_max, rb_max, NL);
    uint8_t *gbuf = smem + sm.gbuf;
    uint8_t *ubuf = smem + sm.ubuf;
    uint8_t *dbuf = smem + sm.dbuf;
    uint16_t *const rbuf0 = reinterpret_cast<uint16_t *>(smem + sm.rbuf0);
    uint16_t *const rbuf1 = reinterpret_cast<uint16_t *>(smem + sm.rbuf1);
    uint16_t *xs = reinterpret_cast<uint16_t *>(smem + sm.xs);
    uint16_t *ns = reinterpret_cast<uint16_t *>(smem + sm.ns);
    uint32_t *xl = reinterpret_cast<uint32_t *>(smem + sm.xl);
    uint32_t *hl = reinterpret_cast<uint32_t *>(smem + sm.hl);
    double *lg = reinterpret_cast<double *>(smem + sm.lg);
    float *hv = reinterpret_cast<float *>(smem + sm.hv);
    float *yv = reinterpret_cast<float *>(smem + sm.yv);
    ulonglong2 *cand = reinterpret_cast<ulonglong2 *>(smem + sm.cand);
    const int xlp = (d / 64) * kSegPad;  // padded words per limb of n
    const int hlp = (f / 64) * kSegPad;  // padded words per limb of h

    const long long lim = p.limit_ns;
    const long long limc = 2 * p.limit_ns;  // the same bound in SM cycles (clocks <= 2 GHz)
    const uint32_t ep = ld_acquire_gpu(p.ctl + 1);  // launch epoch, advanced by the previous launch
    bool alive = true;
    unsigned int n_rt0 = 0, n_rt1 = 0, n_gu = 0, n_dn = 0;  // phases armed per mbarrier (thread 0)

    unsigned long long *tt = (tid == 0) ? p.ttrace : nullptr;
    const size_t ctr_off = (size_t)p.n_layers * P * kTracePoints;
#define TSTAMP(l, ph)                                                  \
    if (tt) {                                                          \
        const size_t o_ = ((size_t)(l) * P + pid) * kTracePoints + (ph); \
        tt[o_] = gtimer();                                             \
        tt[ctr_off + o_] = (unsigned long long)clock64();              \
    }

    {
        constexpr int kW = (int)(sizeof(StackLayerDev) / sizeof(uint64_t));
        static_assert(sizeof(StackLayerDev) % sizeof(uint64_t) == 0, "pointer table");
        for (int q = tid; q < p.n_layers * kW; q += kStackThreads)
            reinterpret_cast<uint64_t *>(s_layer)[q] = reinterpret_cast<const uint64_t *>(p.layer)[q];
    }
    if (tid == 0) {
        mbar_init(&mb_r[0], 1);
        mbar_init(&mb_r[1], 1);
        mbar_init(&mb_gu0, 1);
        mbar_init(&mb_gu1, 1);
        mbar_init(&mb_dn, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // router rows of layers 0 and 1 (buffer l & 1 holds layer l's rows)
    if (tid == 0 && nr > 0) {
        mbar_expect_tx(&mb_r[0], (uint32_t)(nr * d * 2));
        n_rt0++;
        bulk_g2s(rbuf0, s_layer[0].router + (size_t)e0 * d, (uint32_t)(nr * d * 2), &mb_r[0]);
        if (p.n_layers > 1) {
            mbar_expect_tx(&mb_r[1], (uint32_t)(nr * d * 2));
            n_rt1++;
            bulk_g2s(rbuf1, s_layer[1].router + (size_t)e0 * d, (uint32_t)(nr * d * 2), &mb_r[1]);
        }
    }

    for (int l = 0; l < p.n_layers && alive; l++) {
        const StackLayerDev &Ly = s_layer[l];
        const uint32_t par = (uint32_t)(l & 1);
        const uint32_t tag = (ep << 7) | (uint32_t)(l + 1);  // never 0 (a zeroed workspace holds 0)
        const bool has_next = l + 1 < p.n_layers;
        TSTAMP(l, 0)
        // ------------------------------------------------------------ A: x_l, norm, limbs
        // thread t owns elements 4t..4t+3 (d = 4 * threads)
        float xv[4];
        double r;
        float amax;
        {
            bool ok = true;
            uint2 pr;
            if (l == 0) {
                pr = __ldcg(reinterpret_cast<const uint2 *>(p.x) + tid);
            } else {
                const long long t0 = clock64();
                ulonglong2 w;
                ok = poll_pair(p.xb + ((size_t)par * k + s) * (d / 2) + 2 * tid, tag, t0, limc, w);
                pr = make_uint2((uint32_t)w.x, (uint32_t)w.y);
                if (tid < 2 * G) {
                    ulonglong2 st;
                    const bool ok2 = poll_pair(p.xst + (((size_t)par * k + s) * G + (tid >> 1)) * 4 + 2 * (tid & 1), tag,
                                               t0, limc, st);
                    ok = ok && ok2;
                    if (tid & 1) s_xam[tid >> 1] = __uint_as_float((uint32_t)st.x);
                    else s_xss[tid >> 1] = __longlong_as_double((long long)(((unsigned long long)(uint32_t)st.x << 32) |
                                                                            (uint32_t)st.y));
                }
            }
            reinterpret_cast<uint2 *>(xs)[tid] = pr;
            xv[0] = bf16_to_f32((uint16_t)(pr.x & 0xFFFFu));
            xv[1] = bf16_to_f32((uint16_t)(pr.x >> 16));
            xv[2] = bf16_to_f32((uint16_t)(pr.y & 0xFFFFu));
            xv[3] = bf16_to_f32((uint16_t)(pr.y >> 16));
            if (l == 0) {
                double ss = 0.0;
                float am = 0.0f;
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    ss = fma((double)xv[e], (double)xv[e], ss);
                    am = fmaxf(am, fabsf(xv[e]));
                }
                ss = warp_sum_f64(ss);
                am = warp_max_f32(am);
                if (lane == 0) {
                    s_red[warp] = ss;
                    s_redf[warp] = am;
                }
            }
            if (!__syncthreads_and(ok ? 1 : 0)) {
                set_status(p.status, TERN_ETIMEOUT);
                alive = false;
                break;
            }
            // every thread folds the partial sums in the same order: the same r in every CTA
            double ts = 0.0;
            float ta = 0.0f;
            if (l == 0) {
#pragma unroll
                for (int w = 0; w < kStackWarps; w++) {
                    ts += s_red[w];
                    ta = fmaxf(ta, s_redf[w]);
                }
            } else {
                // pairwise tree over the (up to 32) parts, the same order in every thread and CTA
                double v[kMaxGroup];
#pragma unroll
                for (int q = 0; q < kMaxGroup; q++) {
                    v[q] = q < G ? s_xss[q] : 0.0;
                    ta = fmaxf(ta, q < G ? s_xam[q] : 0.0f);
                }
#pragma unroll
                for (int w = kMaxGroup / 2; w > 0; w >>= 1)
#pragma unroll
                    for (int q = 0; q < w; q++) v[q] += v[q + w];
                ts = v[0];
            }
            r = sqrt(ts / (double)d + p.eps);
            amax = ta;
        }
        TSTAMP(l, 1)
        TSTAMP(l, 15)  // r known
        if (l == 0 && pid == 0) reinterpret_cast<uint2 *>(p.hist)[tid] = reinterpret_cast<const uint2 *>(xs)[tid];
        // 1 / r correctly rounded (the same bits as 1.0 / r, without the division routine); rounding
        // is monotone, so max |bf16(x_k / r)| = bf16(max |x_k| / r)
        const double rinv = __drcp_rn(r);
        const float amax_n = bf16_to_f32(bf16_of_quotient((double)amax, r, rinv));
        const float s_nq = (NL == 1) ? (amax_n > 0.0f ? __fdiv_rn(amax_n, 127.0f) : 0.0f) : 0.0f;
        const int sh_n = (NL == 1) ? 0 : fixed_shift(amax_n);
        {
            uint16_t nb[4];
#pragma unroll
            for (int e = 0; e < 4; e++) nb[e] = bf16_of_quotient((double)xv[e], r, rinv);
            reinterpret_cast<uint2 *>(ns)[tid] =
                make_uint2((uint32_t)nb[0] | ((uint32_t)nb[1] << 16), (uint32_t)nb[2] | ((uint32_t)nb[3] << 16));
        }
        TSTAMP(l, 16)  // n known
        // router rows of this layer: thread t multiplies columns 4t..4t+3 (n from shared memory);
        // bf16 x bf16 has at most 16 significant bits, so each product is exact in fp64 and the
        // fma adds it with one rounding (the sums are exact at these magnitudes: the order does
        // not matter)
        if (nr > 0) {
            if (!mbar_wait_sleep(&mb_r[par], (uint32_t)((l >> 1) & 1), lim, p.status)) alive = false;
            const uint2 n2 = reinterpret_cast<const uint2 *>(ns)[tid];
            const double nd[4] = {bf16_to_f64((uint16_t)(n2.x & 0xFFFFu)), bf16_to_f64((uint16_t)(n2.x >> 16)),
                                  bf16_to_f64((uint16_t)(n2.y & 0xFFFFu)), bf16_to_f64((uint16_t)(n2.y >> 16))};
            const uint16_t *rb = par ? rbuf1 : rbuf0;
#pragma unroll 1
            for (int q = 0; q < nr; q += 2) {
                // rows q and q + 1 together (two independent chains); a missing second row is 0
                const uint2 w0 = reinterpret_cast<const uint2 *>(rb + (size_t)q * d)[tid];
                const uint2 w1 = q + 1 < nr ? reinterpret_cast<const uint2 *>(rb + (size_t)(q + 1) * d)[tid]
                                            : make_uint2(0u, 0u);
                double a0 = 0.0, a1 = 0.0;
                a0 = fma(bf16_to_f64((uint16_t)(w0.x & 0xFFFFu)), nd[0], a0);
                a1 = fma(bf16_to_f64((uint16_t)(w1.x & 0xFFFFu)), nd[0], a1);
                a0 = fma(bf16_to_f64((uint16_t)(w0.x >> 16)), nd[1], a0);
                a1 = fma(bf16_to_f64((uint16_t)(w1.x >> 16)), nd[1], a1);
                a0 = fma(bf16_to_f64((uint16_t)(w0.y & 0xFFFFu)), nd[2], a0);
                a1 = fma(bf16_to_f64((uint16_t)(w1.y & 0xFFFFu)), nd[2], a1);
                a0 = fma(bf16_to_f64((uint16_t)(w0.y >> 16)), nd[3], a0);
                a1 = fma(bf16_to_f64((uint16_t)(w1.y >> 16)), nd[3], a1);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    a0 += __shfl_xor_sync(0xFFFFFFFFu, a0, o);
                    a1 += __shfl_xor_sync(0xFFFFFFFFu, a1, o);
                }
                if (lane == 0) {
                    s_rp[warp][q] = a0;
                    if (q + 1 < nr) s_rp[warp][q + 1] = a1;
                }
            }
        }
        TSTAMP(l, 17)  // this warp's router partials written
        if (!__syncthreads_and(alive ? 1 : 0)) break;  // router partials (and n) visible
        if (tid < nr) {
            double sum = 0.0;
            for (int w = 0; w < kStackWarps; w++) sum += s_rp[w][tid];
            const unsigned long long b = (unsigned long long)__double_as_longlong(sum);
            st_relaxed_v2(p.lb + ((size_t)par * E + e0 + tid) * 2, tagged((uint32_t)(b >> 32), tag),
                          tagged((uint32_t)b, tag));
        }
        TSTAMP(l, 2)
        // activation limbs of the gate/up dots (needed only after top-k and the row copies)
        {
            const float inv = (NL == 1 && amax_n > 0.0f) ? quant_inv(amax_n) : 0.0f;
            const uint2 n2 = reinterpret_cast<const uint2 *>(ns)[tid];
            const float v4[4] = {bf16_to_f32((uint16_t)(n2.x & 0xFFFFu)), bf16_to_f32((uint16_t)(n2.x >> 16)),
                                 bf16_to_f32((uint16_t)(n2.y & 0xFFFFu)), bf16_to_f32((uint16_t)(n2.y >> 16))};
            store_limbs4<NL>(xl, xlp, tid, v4, sh_n, inv, amax_n > 0.0f);
        }
        // rbuf[par] is free (this layer's rows are used): fetch the rows of layer l + 2 into it
        if (tid == 0 && nr > 0 && l + 2 < p.n_layers) {
            mbar_expect_tx(&mb_r[par], (uint32_t)(nr * d * 2));
            if (par) n_rt1++;
            else n_rt0++;
            bulk_g2s(par ? rbuf1 : rbuf0, s_layer[l + 2].router + (size_t)e0 * d, (uint32_t)(nr * d * 2), &mb_r[par]);
        }
        TSTAMP(l, 3)
        // ------------------------------------------------------------ B: logits, top-k, copies
        {
            bool ok = true;
            if (tid < E) {
                ulonglong2 w;
                ok = poll_pair(p.lb + ((size_t)par * E + tid) * 2, tag, clock64(), limc, w);
                lg[tid] = __longlong_as_double((long long)(((unsigned long long)(uint32_t)w.x << 32) | (uint32_t)w.y));
            }
            if (!__syncthreads_and(ok ? 1 : 0)) {
                set_status(p.status, TERN_ETIMEOUT);
                alive = false;
                break;
            }
        }
        TSTAMP(l, 4)
        if (warp == 0) {
            warp_topk_filter(lg, E, k, s_idx, cand, s_tkm);
            TSTAMP(l, 18)  // top-k known
            // thread 0 registers the byte counts of this CTA's copies (counted here, so only
            // issued phases are drained after a timeout); warps 0..7 issue them below
            const size_t e = (size_t)s_idx[s];
            // scales: aligned supersets [ga, ga + gn) of rows j0..j1 and [da, da + dn) of i0..i1
            const size_t ga = (e * f + j0) & ~(size_t)3, da = (e * d + i0) & ~(size_t)3;
            const uint32_t gn = (uint32_t)((((e * f + j1) + 3) & ~(size_t)3) - ga);
            const uint32_t dn = ndn > 0 ? (uint32_t)((((e * d + i1) + 3) & ~(size_t)3) - da) : 0u;
            if (lane == 0) {
                mbar_expect_tx(&mb_gu0, (uint32_t)(2 * n0 * (d / 4)) + 8u * gn);
                mbar_expect_tx(&mb_gu1, (uint32_t)(2 * n1 * (d / 4)));
                mbar_expect_tx(&mb_dn, (uint32_t)(ndn * (f / 4)) + 4u * dn);
                n_gu++;
                n_dn++;
            }
        }

        // the copies, one per warp (a warp issues a bulk copy in ~250 cycles; eight from one
        // thread take ~700): warps 0..7 meet at hardware barrier 3 once warp 0 has the experts
        if (warp < 8) {
            named_bar_sync(3, 256);
            if (lane == 0) {
                const size_t e = (size_t)s_idx[s];
                const size_t ga = (e * f + j0) & ~(size_t)3, da = (e * d + i0) & ~(size_t)3;
                const uint32_t gn = (uint32_t)((((e * f + j1) + 3) & ~(size_t)3) - ga);
                const uint32_t dn = ndn > 0 ? (uint32_t)((((e * d + i1) + 3) & ~(size_t)3) - da) : 0u;
                const uint32_t rowg = (uint32_t)(d / 4), rowd = (uint32_t)(f / 4);
                if (warp == 0 && n0 > 0) bulk_g2s(gbuf, Ly.gate + (e * f + j0) * rowg, (uint32_t)n0 * rowg, &mb_gu0);
                if (warp == 1 && n0 > 0) bulk_g2s(ubuf, Ly.up + (e * f + j0) * rowg, (uint32_t)n0 * rowg, &mb_gu0);
                if (warp == 2 && n1 > 0)
                    bulk_g2s(gbuf + (size_t)n0 * rowg, Ly.gate + (e * f + j0 + n0) * rowg, (uint32_t)n1 * rowg, &mb_gu1);
                if (warp == 3 && n1 > 0)
                    bulk_g2s(ubuf + (size_t)n0 * rowg, Ly.up + (e * f + j0 + n0) * rowg, (uint32_t)n1 * rowg, &mb_gu1);
                if (warp == 4 && ndn > 0) bulk_g2s(dbuf, Ly.down + (e * d + i0) * rowd, (uint32_t)ndn * rowd, &mb_dn);
                if (warp == 5) bulk_g2s(s_sgb, Ly.sg + ga, 4u * gn, &mb_gu0);
                if (warp == 6) bulk_g2s(s_sub, Ly.su + ga, 4u * gn, &mb_gu0);
                if (warp == 7 && dn > 0) bulk_g2s(s_sdb, Ly.sd + da, 4u * dn, &mb_dn);
            }
        }
        TSTAMP(l, 5)
        // ------------------------------------------------------------ C: gate/up -> h
        {
            // activation limbs of this lane's segment (d / 64 = 32 segments: lane = segment)
            SegX<NL> X;
            seg_load_x_padded<NL>(X, xl, xlp, lane);
            const int rowb = d / 4;
            bool okc = true;
#pragma unroll 1
            for (int half = 0; half < 2; half++) {
                const int qa = half ? n0 : 0, qb = half ? ngu : n0;
                const int q = qa + warp;
                if (q >= qb) continue;  // no row of this copy for this warp
                // each warp waits for the copy itself: no CTA barrier between the copies and the dots
                if (!mbar_wait_sleep(half ? &mb_gu1 : &mb_gu0, par, lim, p.status)) okc = false;
                if (half == 0) TSTAMP(l, 6)
                {
                    const uint4 wg = *reinterpret_cast<const uint4 *>(gbuf + (size_t)q * rowb + lane * 16);
                    const uint4 wu = *reinterpret_cast<const uint4 *>(ubuf + (size_t)q * rowb + lane * 16);
                    int ag[NL], au[NL];
#pragma unroll
                    for (int z = 0; z < NL; z++) ag[z] = au[z] = 0;
                    seg_dot_alu<NL>(wg, X, ag);
                    seg_dot_alu<NL>(wu, X, au);
                    int ga, gb2, ua, ub;
                    acc_to_pair_x64<NL>(ag, ga, gb2);
                    acc_to_pair_x64<NL>(au, ua, ub);
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
            // warps without rows also take mb_gu0 (the scales the SwiGLU threads read)
            if (warp >= n0 && !mbar_wait_sleep(&mb_gu0, par, lim, p.status)) okc = false;
            if (!__syncthreads_and(okc ? 1 : 0)) {
                alive = false;
                break;
            }
        }
        TSTAMP(l, 7)
        // SwiGLU epilogue, one thread per row, fp64
        const int sgo = (int)(((size_t)s_idx[s] * f + j0) & 3);  // offset of row j0's scale in s_sgb / s_sub
        if (tid < ngu) {
            const int q = tid;
            const long long Sg = s_S[q][0], Su = s_S[q][1];
            float h;
            if (NL == 1) {
                const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg), s_sgb[q + sgo]), s_nq);
                const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su), s_sub[q + sgo]), s_nq);
                h = swiglu_f32((double)gv, (double)uv);
            } else {
                const double p2 = pow2_f64(-sh_n);
                h = swiglu_f32((double)Sg * p2 * (double)s_sgb[q + sgo], (double)Su * p2 * (double)s_sub[q + sgo]);
            }
            st_word(p.hb + ((size_t)par * k + s) * f + j0 + q, __float_as_uint(h), tag);
            p.h_hist[((size_t)l * k + s) * f + j0 + q] = h;
        }
        TSTAMP(l, 8)
        // ------------------------------------------------------------ D: down, combine, residual
        // While warps 0..7 wait for the slot's h: warp 8 computes the gates (needed at the
        // combine); warps 8..15 compute this CTA's router rows of the NEXT layer against n
        // (fp32, a prediction) and publish them.
        if (warp == kStackWarps / 2) {
            warp_topk_gates(lg, k, s_idx, s_gate, nullptr);
            __syncwarp();
            if (lane < k && pid == 0) {
                p.idx_hist[l * k + lane] = s_idx[lane];
                p.gate_hist[l * k + lane] = s_gate[lane];
            }
        }
        const bool predict = PRED && p.predict && has_next && nr > 0;
        if (predict && warp >= kStackWarps / 2) {
            const uint32_t npar = (uint32_t)((l + 1) & 1);
            const bool okr =
                __all_sync(0xFFFFFFFFu, mbar_wait_sleep(&mb_r[npar], (uint32_t)(((l + 1) >> 1) & 1), lim, p.status));
            const int t2 = tid - kStackThreads / 2;  // 256 threads x 8 columns
            const uint4 nv = reinterpret_cast<const uint4 *>(ns)[t2];
#pragma unroll 1
            for (int q = 0; q < nr; q++) {
                if (okr) {
                    const uint4 w = reinterpret_cast<const uint4 *>((npar ? rbuf1 : rbuf0) + (size_t)q * d)[t2];
                    float a = 0.0f;
                    const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, nn[4] = {nv.x, nv.y, nv.z, nv.w};
#pragma unroll
                    for (int z = 0; z < 4; z++) {
                        a = fmaf(__uint_as_float(wv[z] << 16), __uint_as_float(nn[z] << 16), a);
                        a = fmaf(__uint_as_float(wv[z] & 0xFFFF0000u), __uint_as_float(nn[z] & 0xFFFF0000u), a);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
                    if (lane == 0) s_pp[warp - kStackWarps / 2][q] = a;
                }
            }
            named_bar_sync(1, kStackThreads / 2);
            if (t2 < nr && okr) {
                float sum = 0.0f;
                for (int w = 0; w < kStackWarps / 2; w++) sum += s_pp[w][t2];
                st_word(p.pb + (size_t)par * E + e0 + t2, __float_as_uint(sum), tag);
            }
        }
        {
            bool ok = true;
            float m = 0.0f;
            // the test hook makes CTA 0 wait for a tag no producer writes (bounded wait)
            const uint32_t htag = (l == p.stall_layer && pid == 0) ? (tag ^ 0x40000000u) : tag;
            if (2 * tid < f) {
                ulonglong2 w;
                ok = poll_pair(p.hb + ((size_t)par * k + s) * f + 2 * tid, htag, clock64(), limc, w);
                const float h0 = __uint_as_float((uint32_t)w.x), h1 = __uint_as_float((uint32_t)w.y);
                hv[2 * tid] = h0;
                hv[2 * tid + 1] = h1;
                m = fmaxf(fabsf(h0), fabsf(h1));
            }
            m = warp_max_f32(m);
            if (lane == 0) s_hmax[warp] = m;
            if (!__syncthreads_and(ok ? 1 : 0)) {
                set_status(p.status, TERN_ETIMEOUT);
                alive = false;
                break;
            }
        }
        TSTAMP(l, 9)
        float ha = 0.0f;
#pragma unroll
        for (int w = 0; w < kStackWarps; w++) ha = fmaxf(ha, s_hmax[w]);
        const int hsh = (NL == 1) ? 0 : fixed_shift(ha);
        const float hsc = (NL == 1 && ha > 0.0f) ? __fdiv_rn(ha, 127.0f) : 0.0f;
        if (4 * tid < f) {
            const float v4[4] = {hv[4 * tid], hv[4 * tid + 1], hv[4 * tid + 2], hv[4 * tid + 3]};
            const float hinv = (NL == 1 && ha > 0.0f) ? quant_inv(ha) : 0.0f;
            store_limbs4<NL>(hl, hlp, tid, v4, hsh, hinv, ha > 0.0f);
        }
        __syncthreads();
        TSTAMP(l, 10)
        if (ndn > 0 && !mbar_wait_sleep(&mb_dn, par, lim, p.status)) alive = false;
        if (!__syncthreads_and(alive ? 1 : 0)) break;
        TSTAMP(l, 11)
        // down rows: Gf = f / 64 lanes per row, 32 / Gf rows per warp pass
        {
            const int Gf = f / 64;
            const int rpp = 32 / Gf;
            const int sub = lane / Gf, gl = lane % Gf;
            SegX<NL> Hx;
            seg_load_x_padded<NL>(Hx, hl, hlp, gl);
            const int sdo = (int)(((size_t)s_idx[s] * d + i0) & 3);  // offset of row i0's scale in s_sdb
            const uint32_t ytag = tag;
            const int step = kStackWarps * rpp;
            // two rows per lane group at a time (independent chains), then both reductions
#pragma unroll 1
            for (int r0 = warp * rpp; r0 < ndn; r0 += 2 * step) {
                const int ra = r0 + sub, rb2 = r0 + step + sub;
                const bool va = ra < ndn, vb = rb2 < ndn;
                int acca[NL], accb[NL];
#pragma unroll
                for (int z = 0; z < NL; z++) acca[z] = accb[z] = 0;
                const uint4 wa = *reinterpret_cast<const uint4 *>(dbuf + (size_t)(va ? ra : 0) * (f / 4) + gl * 16);
                const uint4 wb = *reinterpret_cast<const uint4 *>(dbuf + (size_t)(vb ? rb2 : 0) * (f / 4) + gl * 16);
                seg_dot_alu<NL>(wa, Hx, acca);
                seg_dot_alu<NL>(wb, Hx, accb);
                int aa, ab, ba, bb;
                acc_to_pair_x64<NL>(acca, aa, ab);
                acc_to_pair_x64<NL>(accb, ba, bb);
                for (int o = Gf / 2; o > 0; o >>= 1) {
                    aa += __shfl_xor_sync(0xFFFFFFFFu, aa, o);
                    ba += __shfl_xor_sync(0xFFFFFFFFu, ba, o);
                    if (NL > 1) {
                        ab += __shfl_xor_sync(0xFFFFFFFFu, ab, o);
                        bb += __shfl_xor_sync(0xFFFFFFFFu, bb, o);
                    }
                }
                if (gl == 0) {
                    const double p2 = pow2_f64(-hsh);
#pragma unroll
                    for (int h2 = 0; h2 < 2; h2++) {
                        const int rr = h2 ? rb2 : ra;
                        if (!(h2 ? vb : va)) continue;
                        const long long S = pair_value(NL, h2 ? ba : aa, h2 ? bb : ab);
                        const float sd = s_sdb[rr + sdo];
                        float v;
                        if (NL == 1) v = __fmul_rn(__fmul_rn(__int2float_rn((int)S), sd), hsc);
                        else v = (float)((double)S * p2 * (double)sd);
                        st_word(p.yb + (((size_t)par * G + c) * k + s) * kMaxDN + rr, __float_as_uint(v), ytag);
                    }
                }
            }
        }
        TSTAMP(l, 12)
        {
            // the k slots' outputs of rows [i0, i1)
            bool ok = true;
            const int half_rows = ndn / 2;
            const long long t0 = clock64();
            for (int t = tid; t < k * half_rows; t += kStackThreads) {
                const int q = t / half_rows, w2 = 2 * (t % half_rows);
                ulonglong2 w;
                if (!poll_pair(p.yb + (((size_t)par * G + c) * k + q) * kMaxDN + w2, tag, t0, limc, w)) {
                    ok = false;
                    break;
                }
                yv[q * kMaxDN + w2] = __uint_as_float((uint32_t)w.x);
                yv[q * kMaxDN + w2 + 1] = __uint_as_float((uint32_t)w.y);
            }
            if (!__syncthreads_and(ok ? 1 : 0)) {
                set_status(p.status, TERN_ETIMEOUT);
                alive = false;
                break;
            }
        }
        TSTAMP(l, 13)
        if (PRED && warp >= kStackWarps / 2 && p.predict && has_next) {
            // The experts predicted for the next layer -> L2 prefetch, by warps 8..15 while warps
            // 0..3 combine.  No exact ranking (a hint needs none): warp 15 takes tau = the
            // kPredTop-th largest of the 32 lane maxima of the predicted logits (lane l holds
            // experts l, l+32, ...), so at least kPredTop experts have a predicted logit >= tau;
            // the c-th of them (lane-major order) belongs to slot group c mod k, and this CTA
            // prefetches its own rows of its group's experts (what it copies if one of them lands
            // in its group).  Warps 8..13 then issue one bulk prefetch each (a warp issues a
            // bulk operation in ~250 cycles; several from one thread serialise).  Only a hint: if
            // the predictions are not all there within a few microseconds, nothing is prefetched.
            // These warps join the CTA again at the next layer's first barrier.
            if (warp == kStackWarps - 1) {
                // the eight words of a lane are loaded together (a global load is a ~700-cycle
                // round trip); only words not yet published are loaded again
                bool ok = true;
                float pv[8];
                unsigned pending = 0;
                const long long t0 = clock64();
                do {
                    unsigned long long w[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const int e = lane + 32 * j;
                        w[j] = 0ull;
                        if (e < E && ((pending >> j) & 1u || pending == 0u))
                            asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w[j]) : "l"(p.pb + (size_t)par * E + e) : "memory");
                    }
                    unsigned still = 0;
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const int e = lane + 32 * j;
                        if (e >= E) {
                            pv[j] = -INFINITY;
                        } else if ((pending >> j) & 1u || pending == 0u) {
                            if ((uint32_t)(w[j] >> 32) == tag) pv[j] = __uint_as_float((uint32_t)w[j]);
                            else still |= 1u << j;
                        }
                    }
                    pending = still ? still : 0u;
                    if (still && clock64() - t0 > kPredictWaitCycles) ok = false;
                    if (!still) break;
                } while (ok);
                int npf = 0;
                if (__all_sync(0xFFFFFFFFu, ok)) {
                    float mx = pv[0];
#pragma unroll
                    for (int j = 1; j < 8; j++) mx = fmaxf(mx, pv[j]);
                    int above4[4] = {0, 0, 0, 0};
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const float o = __shfl_sync(0xFFFFFFFFu, mx, i);
                        above4[i & 3] += (o > mx || (o == mx && i < lane)) ? 1 : 0;
                    }
                    const int above = (above4[0] + above4[1]) + (above4[2] + above4[3]);
                    const int np = E < kPredTop ? E : kPredTop;
                    const unsigned who = __ballot_sync(0xFFFFFFFFu, above == np - 1);
                    const float tau = __shfl_sync(0xFFFFFFFFu, mx, __ffs(who) - 1);
                    unsigned msk[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) msk[j] = __ballot_sync(0xFFFFFFFFu, lane + 32 * j < E && pv[j] >= tau);
                    int count = 0;
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        const int cidx = count + __popc(msk[j] & ((1u << lane) - 1u));
                        if (((msk[j] >> lane) & 1u) && cidx % k == s) {
                            const int slot = cidx / k;
                            if (slot < kMaxPrefetch) s_pf[slot] = lane + 32 * j;
                        }
                        count += __popc(msk[j]);
                    }
                    npf = (count - s + k - 1) / k;  // candidates c < count with c mod k == s
                    if (npf > kMaxPrefetch) npf = kMaxPrefetch;
                    if (npf < 0) npf = 0;
                }
                if (lane == 0) s_npf = npf;
            }
            named_bar_sync(4, kStackThreads / 2);
            const int task = warp - kStackWarps / 2;  // 0..5: expert task / 3, array task % 3
            if (task < 3 * s_npf && lane == 0) {
                const StackLayerDev &Ln = s_layer[l + 1];
                const size_t ee = (size_t)s_pf[task / 3];
                const uint32_t rowg = (uint32_t)(d / 4), rowd = (uint32_t)(f / 4);
                const int a = task % 3;
                if (a == 0 && ngu > 0) {
                    prefetch_l2_bulk(Ln.gate + (ee * f + j0) * rowg, (uint32_t)ngu * rowg);
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(Ln.sg + ee * f + j0));
                }
                if (a == 1 && ngu > 0) {
                    prefetch_l2_bulk(Ln.up + (ee * f + j0) * rowg, (uint32_t)ngu * rowg);
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(Ln.su + ee * f + j0));
                }
                if (a == 2 && ndn > 0) {
                    prefetch_l2_bulk(Ln.down + (ee * d + i0) * rowd, (uint32_t)ndn * rowd);
                    for (int o = 0; o < ndn; o += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(Ln.sd + ee * d + i0 + o));
                }
            }
        }
        {
            const bool last = !has_next;
            const uint32_t ntag = (ep << 7) | (uint32_t)(l + 2);
            const uint32_t npar = (uint32_t)((l + 1) & 1);
            // one output row per thread, fixed top-k order; row pairs leave as one word
            uint16_t xo = 0;
            double sq = 0.0;
            float am = 0.0f;
            if (tid < ndn) {
                double yq[kSK];
#pragma unroll
                for (int q = 0; q < kSK; q++) yq[q] = q < k ? (double)yv[q * kMaxDN + tid] : 0.0;
                double y = 0.0;
#pragma unroll
                for (int q = 0; q < kSK; q++)
                    if (q < k) y += s_gate[q] * yq[q];  // top-k order
                const uint16_t yb = f64_to_bf16_rne(y);
                xo = f64_to_bf16_rne((double)bf16_to_f32(xs[i0 + tid]) + (double)bf16_to_f32(yb));
                const double xv2 = (double)bf16_to_f32(xo);
                sq = xv2 * xv2;
                am = fabsf((float)xv2);
                if (s == 0) {
                    p.hist[(size_t)(l + 1) * d + i0 + tid] = xo;
                    p.y_hist[(size_t)l * d + i0 + tid] = (float)y;
                    if (last) p.x[i0 + tid] = xo;
                }
            }
            const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, (uint32_t)xo, 1);
            if (!last && tid < ndn && (tid & 1) == 0)
                st_word(p.xb + ((size_t)npar * k + s) * (d / 2) + (i0 + tid) / 2, (uint32_t)xo | (other << 16), ntag);
            if (!last && warp < kMaxDN / 32) {
                // sum of squares and absmax of this part (threads < ndn <= kMaxDN = 128: warps
                // 0..3, synchronised by hardware barrier 2 alone)
                sq = warp_sum_f64(sq);
                am = warp_max_f32(am);
                if (lane == 0) {
                    s_red[warp] = sq;
                    s_redf[warp] = am;
                }
                named_bar_sync(2, kMaxDN);
                if (tid == 0) {
                    double ts = 0.0;
                    float ta = 0.0f;
                    for (int w = 0; w < (ndn + 31) / 32; w++) {
                        ts += s_red[w];
                        ta = fmaxf(ta, s_redf[w]);
                    }
                    const unsigned long long b = (unsigned long long)__double_as_longlong(ts);
                    unsigned long long *dst = p.xst + (((size_t)npar * k + s) * G + c) * 4;
                    st_relaxed_v2(dst, tagged((uint32_t)(b >> 32), ntag), tagged((uint32_t)b, ntag));
                    st_relaxed_v2(dst + 2, tagged(__float_as_uint(ta), ntag), tagged(0u, ntag));
                }
            }
        }
        TSTAMP(l, 14)
    }
#undef TSTAMP
    // after a timeout, let this CTA's own copies in flight land (bounded) before leaving
    if (!alive && tid == 0) {
        if (n_rt0) mbar_wait(&mb_r[0], (n_rt0 - 1) & 1u, lim, p.status);
        if (n_rt1) mbar_wait(&mb_r[1], (n_rt1 - 1) & 1u, lim, p.status);
        if (n_gu) {
            mbar_wait(&mb_gu0, (n_gu - 1) & 1u, lim, p.status);
            mbar_wait(&mb_gu1, (n_gu - 1) & 1u, lim, p.status);
        }
        if (n_dn) mbar_wait(&mb_dn, (n_dn - 1) & 1u, lim, p.status);
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
// Persistent-path workspace: control words, exchange buffers, per-layer record, trace.
struct StackWs {
    int64_t ctl, xb, xst, lb, pb, hb, yb, hist, idx_hist, gate_hist, y_hist, h_hist, ttrace, total;
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
    const int64_t d = L0->d, f = L0->f, E = L0->E, k = L0->k;
    o.ctl = take(256);
    o.xb = take(2 * k * (d / 2) * 8);
    o.xst = take(2 * k * kMaxGroup * 4 * 8);
    o.lb = take(2 * E * 2 * 8);
    o.pb = take(2 * E * 8);
    o.hb = take(2 * k * f * 8);
    o.yb = take(2 * kMaxGroup * k * kMaxDN * 8);
    o.hist = take((int64_t)(kMaxLayers + 1) * d * 2);
    o.idx_hist = take((int64_t)kMaxLayers * k * 4);
    o.gate_hist = take((int64_t)kMaxLayers * k * 8);
    o.y_hist = take((int64_t)kMaxLayers * d * 4);
    o.h_hist = take((int64_t)kMaxLayers * k * f * 4);
    o.ttrace = take((int64_t)2 * kMaxLayers * kMaxTraceCtas * kTracePoints * 8);
    o.total = p;
    return o;
}

size_t stack_persistent_ws_bytes(const tern_moe_layer *L0) { return (size_t)stack_ws_layout(L0).total; }

void stack_persistent_offsets(const tern_moe_layer *L0, int64_t *hist, int64_t *idx_hist, int64_t *gate_hist,
                              int64_t *y_hist, int64_t *h_hist, int64_t *ttrace) {
    const StackWs o = stack_ws_layout(L0);
    *hist = o.hist;
    *idx_hist = o.idx_hist;
    *gate_hist = o.gate_hist;
    *y_hist = o.y_hist;
    *h_hist = o.h_hist;
    *ttrace = o.ttrace;
}

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

struct StackPlan {
    int P, G;
    SmemMap sm;
    const void *fn, *fn_pred;  // without / with the next-layer prediction code
};

static tern_status stack_plan(const tern_moe_layer &L0, int n_layers, tern_act act, StackPlan &pl) {
    const int d = (int)L0.d, f = (int)L0.f, E = L0.E, k = L0.k;
    // thread mappings: d = 4 * threads; f / 64 segments per down row, a power of two <= 32;
    // f <= 2 * threads (h gather), E <= 256 (top-k); k <= 8 slot groups
    if (n_layers > kMaxLayers || d != 4 * kStackThreads || k > kSK || f % 64 || f > 2 * kStackThreads || E > 256)
        return TERN_EUNSUPPORTED;
    const int gf = f / 64;
    if (gf < 1 || gf > 32 || (gf & (gf - 1)) != 0) return TERN_EUNSUPPORTED;
    // the scales are bulk-copied in 16-byte aligned blocks (every layer is checked at launch)
    if (((uintptr_t)L0.gate_scale | (uintptr_t)L0.up_scale | (uintptr_t)L0.down_scale) & 15u) return TERN_EUNSUPPORTED;
    const int sms = sm_count();
    if (sms <= 0) return TERN_ECUDA;
    int G = sms / k;
    if (G > kMaxGroup) G = kMaxGroup;
    // shares: <= 32 gate/up rows (two copies of 16), <= 128 down rows, <= 8 router rows per CTA
    if (G < 1 || (f + G - 1) / G > kMaxGU || 2 * ((d / 2 + G - 1) / G) > kMaxDN) return TERN_EUNSUPPORTED;
    const int P = k * G;
    if (P > kMaxTraceCtas || (E + P - 1) / P > kMaxRouterRows) return TERN_EUNSUPPORTED;
    pl.P = P;
    pl.G = G;
    const int NL = act == TERN_ACT_INT8 ? 1 : 3;
    pl.sm = smem_map(d, f, k, (f + G - 1) / G, 2 * ((d / 2 + G - 1) / G), (E + P - 1) / P, NL);
    pl.fn = act == TERN_ACT_INT8 ? (const void *)stack_kernel<1, false> : (const void *)stack_kernel<3, false>;
    pl.fn_pred = act == TERN_ACT_INT8 ? (const void *)stack_kernel<1, true> : (const void *)stack_kernel<3, true>;
    for (const void *fn : {pl.fn, pl.fn_pred}) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.sm.total) != cudaSuccess)
            return TERN_ECUDA;
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kStackThreads, pl.sm.total) != cudaSuccess)
            return TERN_ECUDA;
        if (nb < 1 || nb * sms < P) return TERN_EUNSUPPORTED;
    }
    return TERN_OK;
}

bool stack_persistent_supported(const tern_moe_layer *L0, int n_layers, tern_act act) {
    StackPlan pl;
    return stack_plan(*L0, n_layers, act, pl) == TERN_OK;
}

int stack_persistent_ctas(const tern_moe_layer *L0, int n_layers, tern_act act) {
    StackPlan pl;
    return stack_plan(*L0, n_layers, act, pl) == TERN_OK ? pl.P : 0;
}

tern_status launch_stack_persistent(const tern_moe_layer *layers, int n_layers, uint16_t *x, float eps, tern_act act,
                                    void *ws, size_t ws_bytes, int *status, int stall_layer, long long limit_ns,
                                    cudaStream_t s) {
    const tern_moe_layer &L0 = layers[0];
    StackPlan pl;
    const tern_status pst = stack_plan(L0, n_layers, act, pl);
    if (pst != TERN_OK) return pst;
    const StackWs o = stack_ws_layout(&L0);
    if (ws_bytes < (size_t)o.total) return TERN_EWORKSPACE;
    if (!status) return TERN_ECUDA;
    // the scales are bulk-copied in 16-byte aligned blocks: the arrays must start 16-byte aligned
    for (int l = 0; l < n_layers; l++)
        if (((uintptr_t)layers[l].gate_scale | (uintptr_t)layers[l].up_scale | (uintptr_t)layers[l].down_scale) & 15u)
            return TERN_EUNSUPPORTED;

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
    prm.xb = reinterpret_cast<unsigned long long *>(b + o.xb);
    prm.xst = reinterpret_cast<unsigned long long *>(b + o.xst);
    prm.lb = reinterpret_cast<unsigned long long *>(b + o.lb);
    prm.pb = reinterpret_cast<unsigned long long *>(b + o.pb);
    prm.hb = reinterpret_cast<unsigned long long *>(b + o.hb);
    prm.yb = reinterpret_cast<unsigned long long *>(b + o.yb);
    prm.hist = reinterpret_cast<uint16_t *>(b + o.hist);
    prm.idx_hist = reinterpret_cast<int32_t *>(b + o.idx_hist);
    prm.gate_hist = reinterpret_cast<double *>(b + o.gate_hist);
    prm.y_hist = reinterpret_cast<float *>(b + o.y_hist);
    prm.h_hist = reinterpret_cast<float *>(b + o.h_hist);
    // phase stamps cost a %globaltimer read and a store each: only when TERNMOE_TRACE=1
    const char *tenv = getenv("TERNMOE_TRACE");
    prm.ttrace = (tenv && tenv[0] == '1') ? reinterpret_cast<unsigned long long *>(b + o.ttrace) : nullptr;
    // L2 prefetch of predicted next-layer experts: only when TERNMOE_PREDICT=1 (measured: the
    // prediction's own cost still exceeds the row-wait time it saves)
    const char *penv = getenv("TERNMOE_PREDICT");
    prm.predict = (penv && penv[0] == '1') ? 1 : 0;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.P = pl.P;
    prm.G = pl.G;
    prm.stall_layer = stall_layer;

    void *args[] = {&prm};
    const cudaError_t e = cudaLaunchCooperativeKernel(prm.predict ? pl.fn_pred : pl.fn, dim3(pl.P), dim3(kStackThreads),
                                                      args, pl.sm.total, s);
    return e == cudaSuccess ? TERN_OK : TERN_ECUDA;
}

}  // namespace tern
