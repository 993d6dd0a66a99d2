// stack_batch.cu -- whole-stack decode for a small batch (2 <= T <= 16 tokens) in ONE
// cooperative launch, sm_100a.
//
// Several tokens decoded together share the experts they select: the pages' batch-1 argument
// ("A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What
// Ternary Actually Means") counts the active experts' bytes once per token, and the MoE
// discussion ("iPhone Runs a 20B Model at 120 tok/s", "MoE Is the Other Half of the Story
// Behind the 20B Figure") notes that the selected experts' weights are scattered.  Here every
// selected expert's rows are read from HBM once per step and applied to every token routed to
// it, and the per-stage kernels' launch and fixed costs are replaced by four grid-wide
// barriers per layer inside one launch:
//   A  every CTA: r and n of every token, the activation limbs of every token (shared
//      memory), its 1-2 router rows for every token (exact fp64) -> logits to global
//   -- barrier --
//   B  every CTA: top-k and gates of every token (one warp per token, the same in every CTA),
//      the distinct experts (ascending) and their (token, slot) lists
//   C  gate/up work items = (distinct expert, block of 16 rows), a contiguous range per CTA;
//      each item's rows come by bulk copy into a ring of stages, one row per warp, applied to
//      every token of that expert -> h (fp32) of each (token, slot)
//   -- barrier --
//   D  down work items = (distinct expert, block of 512 / (f/64) rows); per expert the h limbs
//      of its (token, slot) pairs are built once in shared memory -> each pair's output rows
//      (fp32)
//   -- barrier --
//   E  rows split over the CTAs: y = sum_q g_q y_q in top-k order (fp64), x' = bf16(x +
//      bf16(y)) for every token, in place in x
//   -- barrier (before the next layer) --
// The arithmetic is the batch-1 kernel's (stack.cu) operation for operation, so a token's
// result does not depend on the other tokens of the batch.
#include <cuda_runtime.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include "cluster.cuh"
#include "kernels.h"
#include "tern_common.cuh"
#include "tma.cuh"

namespace tern {

constexpr int kBWarps = 16;
constexpr int kBThreads = kBWarps * 32;
constexpr int kBMaxT = 16;
constexpr int kBMaxK = 8;
constexpr int kBMaxPairs = kBMaxT * kBMaxK;
constexpr int kBMaxE = 256;
constexpr int kBGuRows = 16;        // gate/up rows per work item: one per warp
constexpr int kBMaxRouterRows = 2;  // router rows per CTA
constexpr int kBMaxStages = 8;
constexpr int kBTopkCand = 256;     // candidate entries per top-k warp
constexpr int kBTracePoints = 16;   // per layer and CTA: see the stamps in the kernel
constexpr int kBMaxCtas = 256;

struct BatchParams {
    StackLayerDev layer[kMaxLayers];
    int n_layers, d, f, E, k, T;
    double eps;
    uint16_t *x;            // [T][d] in/out; also x between layers (rows updated in place)
    unsigned int *ctl;      // [0] barrier arrivals, [1] CTAs that left
    double *lg;             // [T][E] router logits of the current layer
    float *yb;              // [T*k][d] output rows of each (token, slot)'s expert (fp32)
    uint16_t *hist;         // [n_layers+1][T][d] x entering each layer, and the final x
    int32_t *idx_hist;      // [n_layers][T][k]
    double *gate_hist;      // [n_layers][T][k]
    float *y_hist;          // [n_layers][T][d]    FFN output before its bf16 cast
    float *h_hist;          // [n_layers][T][k][f] SwiGLU output; also the h exchange buffer
    int *status;
    long long limit_cycles; // bound on every in-kernel poll (SM cycles)
    long long limit_ns;     // the same bound for mbarrier waits (%globaltimer)
    unsigned long long *ttrace;  // [n_layers][P][kBTracePoints] clock64 stamps, or null
    int P;                  // CTAs
    int stall_layer;        // test hook: at this layer CTA 0 does not arrive at the barrier after phase C
    int stages;             // ring stages
    uint32_t stage_bytes;
};

// dynamic shared memory: activation limbs of every token (reused for the h limbs of one
// expert's pairs in phase D), then the ring of row stages (reused for the logits and the
// top-k candidates in phase B, and for the reductions of phase A)
struct BatchSmem {
    uint32_t xl, ring, total;
};

__host__ __device__ inline uint32_t batch_align128(uint32_t v) { return (v + 127u) & ~127u; }

__host__ __device__ inline BatchSmem batch_smem(int d, int E, int T, int NL, int stages, uint32_t stage_bytes) {
    BatchSmem m;
    m.xl = 0;
    m.ring = batch_align128((uint32_t)T * NL * (d / 64) * kSegPad * 4);
    m.total = m.ring + (uint32_t)stages * stage_bytes;
    (void)E;
    return m;
}

// ring bytes phase B needs: T x E logits (fp64), then T x 256 candidates (16 bytes each)
__host__ __device__ inline uint32_t batch_topk_bytes(int E, int T) {
    return batch_align128((uint32_t)T * E * 8) + (uint32_t)T * kBTopkCand * 16;
}

// phase A scratch inside the ring: [T][16] partial sums of squares (fp64), [T][16] partial
// maxima, [T][16][2] router partials (fp64)
constexpr uint32_t kBScratchRed = kBMaxT * kBWarps * 8;
constexpr uint32_t kBScratchRedf = kBMaxT * kBWarps * 4;
constexpr uint32_t kBScratchRp = kBMaxT * kBWarps * kBMaxRouterRows * 8;
constexpr uint32_t kBScratchBytes = kBScratchRed + kBScratchRedf + kBScratchRp;

__device__ __forceinline__ void unpack_bf16x4(uint2 pr, float (&v)[4]) {
    v[0] = bf16_to_f32((uint16_t)(pr.x & 0xFFFFu));
    v[1] = bf16_to_f32((uint16_t)(pr.x >> 16));
    v[2] = bf16_to_f32((uint16_t)(pr.y & 0xFFFFu));
    v[3] = bf16_to_f32((uint16_t)(pr.y >> 16));
}

// ------------------------------------------------------------------ the kernel
template <int NL>
__global__ void __launch_bounds__(kBThreads, 1) stack_batch_kernel(const __grid_constant__ BatchParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t mb_full[kBMaxStages];
    __shared__ double s_r[kBMaxT], s_rinv[kBMaxT];
    __shared__ int s_tsh[kBMaxT];      // bf16 activations: fixed-point shift of n_t
    __shared__ float s_tsc[kBMaxT];    // int8 activations: scale of n_t (absmax / 127)
    __shared__ float s_tam[kBMaxT];    // absmax of n_t
    __shared__ int32_t s_idx[kBMaxPairs];
    __shared__ double s_gate[kBMaxPairs];
    __shared__ __align__(16) uint32_t s_tkm[kBWarps][32];
    __shared__ int s_cnt[kBMaxE], s_rank[kBMaxE];
    __shared__ int s_uexp[kBMaxPairs], s_ustart[kBMaxPairs + 1], s_plist[kBMaxPairs];
    __shared__ int s_U;
    __shared__ int s_rng[4];           // this CTA's item ranges: C [0, 1), D [2, 3)
    __shared__ int s_hsh[kBMaxT];      // h limbs of the current expert's pairs: shift / int8 scale
    __shared__ float s_hsc[kBMaxT];
    __shared__ int s_flag;
    __shared__ StackLayerDev s_ly;     // this layer's pointers

    const int d = p.d, f = p.f, E = p.E, k = p.k, T = p.T, P = p.P;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, pid = blockIdx.x;
    const int npair = T * k;
    const BatchSmem sm = batch_smem(d, E, T, NL, p.stages, p.stage_bytes);
    uint32_t *xl = reinterpret_cast<uint32_t *>(smem + sm.xl);  // [T][NL][xlp] limbs of n_t
    uint32_t *hl = xl;                                            // [m][NL][hlp] (phase D)
    unsigned char *ring = smem + sm.ring;
    const int xlp = (d / 64) * kSegPad;
    const int hlp = (f / 64) * kSegPad;
    const int e0 = (E * pid) / P, nr = (E * (pid + 1)) / P - e0;   // router rows
    const int r0 = (d * pid) / P, nrow = (d * (pid + 1)) / P - r0;  // combine rows
    const int Gf = f / 64, rpp = 32 / Gf, rb_dn = kBWarps * rpp;     // down: lanes per row, rows per item
    const int nb_gu = f / kBGuRows, nb_dn = d / rb_dn;              // items per expert
    const uint32_t rowg = (uint32_t)(d / 4), rowd = (uint32_t)(f / 4);
    GridSync gs;
    gs.arrive = p.ctl;
    gs.leave = p.ctl + 1;
    gs.status = p.status;
    gs.nblocks = (unsigned)P;
    gs.epoch = 0u;
    gs.limit = p.limit_cycles;
    unsigned long long *tt = (tid == 0) ? p.ttrace : nullptr;
#define BSTAMP(l, ph_)                                                                         \
    if (tt) tt[((size_t)(l) * P + pid) * kBTracePoints + (ph_)] = (unsigned long long)clock64();
    bool alive = true;
    uint32_t ph = 0u;    // per stage: parity of its next completion
    // the current phase's items [dr_c0 + ...): issued up to dr_hi, consumed up to dr_lo (the
    // same in every thread); after a timeout, the copies of items [dr_lo, dr_hi) may be in flight
    int dr_c0 = 0, dr_lo = 0, dr_hi = 0;

    if (tid == 0) {
        for (int q = 0; q < p.stages; q++) mbar_init(&mb_full[q], 1);
        fence_mbar_init();
    }
    if (pid == 0)
        for (int q = tid; q < T * d / 4; q += kBThreads)
            reinterpret_cast<uint2 *>(p.hist)[q] = __ldcg(reinterpret_cast<const uint2 *>(p.x) + q);
    __syncthreads();

    for (int l = 0; l < p.n_layers && alive; l++) {
        const bool has_next = l + 1 < p.n_layers;
        if (tid < (int)(sizeof(StackLayerDev) / 8))
            reinterpret_cast<unsigned long long *>(&s_ly)[tid] = reinterpret_cast<const unsigned long long *>(&p.layer[l])[tid];
        BSTAMP(l, 0)
        // ------------------------------------------------------------ A: norm, limbs, router
        double *s_red = reinterpret_cast<double *>(ring);
        float *s_redf = reinterpret_cast<float *>(ring + kBScratchRed);
        double *s_rp = reinterpret_cast<double *>(ring + kBScratchRed + kBScratchRedf);
        // x of every token into shared memory (after the phase A scratch); thread t holds
        // elements 4t .. 4t + 3 of each token (d = 4 * threads)
        uint2 *xsh = reinterpret_cast<uint2 *>(ring + kBScratchBytes);  // [T][d / 4]
#pragma unroll
        for (int t0 = 0; t0 < kBMaxT; t0 += 8) {
            uint2 xr[8];  // eight loads in flight at a time
#pragma unroll
            for (int t = 0; t < 8; t++)
                if (t0 + t < T) xr[t] = __ldcg(reinterpret_cast<const uint2 *>(p.x + (size_t)(t0 + t) * d) + tid);
#pragma unroll
            for (int t = 0; t < 8; t++)
                if (t0 + t < T) xsh[(t0 + t) * (d / 4) + tid] = xr[t];
        }
        // sums of squares and maxima, four tokens at a time (a loop, not unrolled: one copy of
        // the code for any T)
#pragma unroll 1
        for (int t0 = 0; t0 < T; t0 += 4) {
            double ss[4];
            float am[4];
#pragma unroll
            for (int tt = 0; tt < 4; tt++) {
                float xv[4];
                unpack_bf16x4(t0 + tt < T ? xsh[(t0 + tt) * (d / 4) + tid] : make_uint2(0u, 0u), xv);
                ss[tt] = 0.0;
                am[tt] = 0.0f;
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    ss[tt] = fma((double)xv[e], (double)xv[e], ss[tt]);
                    am[tt] = fmaxf(am[tt], fabsf(xv[e]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int tt = 0; tt < 4; tt++) {
                    ss[tt] += __shfl_xor_sync(0xFFFFFFFFu, ss[tt], o);
                    am[tt] = fmaxf(am[tt], __shfl_xor_sync(0xFFFFFFFFu, am[tt], o));
                }
            if (lane == 0)
#pragma unroll
                for (int tt = 0; tt < 4; tt++)
                    if (t0 + tt < T) {
                        s_red[(t0 + tt) * kBWarps + warp] = ss[tt];
                        s_redf[(t0 + tt) * kBWarps + warp] = am[tt];
                    }
        }
        __syncthreads();
        BSTAMP(l, 8)
        if (tid < T) {
            // the warps' partial sums in warp order: the same r in every CTA
            double ts = 0.0;
            float ta = 0.0f;
            for (int w = 0; w < kBWarps; w++) {
                ts += s_red[tid * kBWarps + w];
                ta = fmaxf(ta, s_redf[tid * kBWarps + w]);
            }
            const double r = sqrt(ts / (double)d + p.eps);
            s_r[tid] = r;
            const double rinv = __drcp_rn(r);  // correctly rounded: the same bits as 1.0 / r
            s_rinv[tid] = rinv;
            // rounding is monotone, so max |bf16(x_k / r)| = bf16(max |x_k| / r)
            const float amax_n = bf16_to_f32(bf16_of_quotient((double)ta, r, rinv));
            s_tam[tid] = amax_n;
            s_tsh[tid] = (NL == 1) ? 0 : fixed_shift(amax_n);
            s_tsc[tid] = (NL == 1 && amax_n > 0.0f) ? __fdiv_rn(amax_n, 127.0f) : 0.0f;
        }
        __syncthreads();
        BSTAMP(l, 9)
        {
            // this thread's four columns of the CTA's router rows
            uint2 rw[kBMaxRouterRows];
#pragma unroll
            for (int q = 0; q < kBMaxRouterRows; q++)
                rw[q] = q < nr ? __ldg(reinterpret_cast<const uint2 *>(s_ly.router + (size_t)(e0 + q) * d) + tid)
                               : make_uint2(0u, 0u);
#pragma unroll 1
            for (int t0 = 0; t0 < T; t0 += 4) {
                {
                    double part[4][kBMaxRouterRows];
#pragma unroll
                    for (int tt = 0; tt < 4; tt++) {
                        const int t = t0 + tt;
#pragma unroll
                        for (int q = 0; q < kBMaxRouterRows; q++) part[tt][q] = 0.0;
                        if (t < T) {
                            float xv[4];
                            unpack_bf16x4(xsh[t * (d / 4) + tid], xv);
                            const double r = s_r[t], rinv = s_rinv[t];
                            uint16_t nb[4];
#pragma unroll
                            for (int e = 0; e < 4; e++) nb[e] = bf16_of_quotient((double)xv[e], r, rinv);
                            const float amax_n = s_tam[t];
                            const float inv = (NL == 1 && amax_n > 0.0f) ? quant_inv(amax_n) : 0.0f;
                            const float v4[4] = {bf16_to_f32(nb[0]), bf16_to_f32(nb[1]), bf16_to_f32(nb[2]),
                                                 bf16_to_f32(nb[3])};
                            store_limbs4<NL>(xl + (size_t)t * NL * xlp, xlp, tid, v4, s_tsh[t], inv, amax_n > 0.0f);
                            const double nd[4] = {bf16_to_f64(nb[0]), bf16_to_f64(nb[1]), bf16_to_f64(nb[2]),
                                                  bf16_to_f64(nb[3])};
                            // bf16 x bf16 products are exact in fp64; the fma adds each with one
                            // rounding, in the same order as the batch-1 kernel
#pragma unroll
                            for (int q = 0; q < kBMaxRouterRows; q++) {
                                double a = 0.0;
                                a = fma(bf16_to_f64((uint16_t)(rw[q].x & 0xFFFFu)), nd[0], a);
                                a = fma(bf16_to_f64((uint16_t)(rw[q].x >> 16)), nd[1], a);
                                a = fma(bf16_to_f64((uint16_t)(rw[q].y & 0xFFFFu)), nd[2], a);
                                a = fma(bf16_to_f64((uint16_t)(rw[q].y >> 16)), nd[3], a);
                                part[tt][q] = a;
                            }
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                        for (int tt = 0; tt < 4; tt++)
#pragma unroll
                            for (int q = 0; q < kBMaxRouterRows; q++)
                                part[tt][q] += __shfl_xor_sync(0xFFFFFFFFu, part[tt][q], o);
                    if (lane == 0)
#pragma unroll
                        for (int tt = 0; tt < 4; tt++)
#pragma unroll
                            for (int q = 0; q < kBMaxRouterRows; q++)
                                if (t0 + tt < T) s_rp[((t0 + tt) * kBWarps + warp) * kBMaxRouterRows + q] = part[tt][q];
                }
            }
        }
        BSTAMP(l, 10)
        __syncthreads();
        if (tid < T * nr) {
            const int t = tid / nr, q = tid % nr;
            double sum = 0.0;
            for (int w = 0; w < kBWarps; w++) sum += s_rp[(t * kBWarps + w) * kBMaxRouterRows + q];
            p.lg[(size_t)t * E + e0 + q] = sum;
        }
        BSTAMP(l, 1)
        if (!grid_sync(gs, &s_flag)) {
            alive = false;
            break;
        }
        // ------------------------------------------------------------ B: top-k, gates, grouping
        {
            double *s_lg = reinterpret_cast<double *>(ring);
            ulonglong2 *cand = reinterpret_cast<ulonglong2 *>(ring + batch_align128((uint32_t)T * E * 8));
            for (int q = tid; q < T * E; q += kBThreads) s_lg[q] = __ldcg(p.lg + q);
            __syncthreads();
            BSTAMP(l, 11)
            if (warp < T) {
                warp_topk_filter(s_lg + (size_t)warp * E, E, k, s_idx + warp * k, cand + (size_t)warp * kBTopkCand,
                                 s_tkm[warp]);
                warp_topk_gates(s_lg + (size_t)warp * E, k, s_idx + warp * k, s_gate + warp * k, nullptr);
                __syncwarp();
                if (pid == 0 && lane < k) {
                    p.idx_hist[((size_t)l * T + warp) * k + lane] = s_idx[warp * k + lane];
                    p.gate_hist[((size_t)l * T + warp) * k + lane] = s_gate[warp * k + lane];
                }
            }
            __syncthreads();
            BSTAMP(l, 12)
            // how many (token, slot) pairs chose each expert
            if (tid < E) s_cnt[tid] = 0;
            __syncthreads();
            if (tid < npair) atomicAdd(&s_cnt[s_idx[tid]], 1);
            __syncthreads();
            // the distinct experts in ascending order and where their pair lists start: lane l
            // of warp 0 takes experts 8l .. 8l + 7 (E <= 256), then an exclusive scan
            if (warp == 0) {
                int pc = 0, sc = 0;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int e = 8 * lane + j;
                    const int c = e < E ? s_cnt[e] : 0;
                    pc += c > 0 ? 1 : 0;
                    sc += c;
                }
                int ipc = pc, isc = sc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int a = __shfl_up_sync(0xFFFFFFFFu, ipc, o), b = __shfl_up_sync(0xFFFFFFFFu, isc, o);
                    if (lane >= o) {
                        ipc += a;
                        isc += b;
                    }
                }
                int rk = ipc - pc, st = isc - sc;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const int e = 8 * lane + j;
                    const int c = e < E ? s_cnt[e] : 0;
                    if (c > 0) {
                        s_rank[e] = rk;
                        s_uexp[rk] = e;
                        s_ustart[rk] = st;
                        rk++;
                        st += c;
                    }
                }
                if (lane == 31) {
                    s_U = ipc;
                    s_ustart[ipc] = isc;
                }
            }
            __syncthreads();
            // each expert's pairs in pair order (token-major): warp 0 walks the pairs 32 at a time;
            // equal experts within a chunk are ranked by lane, and s_cnt (no longer needed as a
            // count) carries each expert's running fill across chunks
            if (warp == 0) {
                for (int e = lane; e < E; e += 32) s_cnt[e] = 0;
                __syncwarp();
                for (int q0 = 0; q0 < npair; q0 += 32) {
                    const int q = q0 + lane;
                    const bool v = q < npair;
                    const int e = v ? s_idx[q] : -1 - lane;  // distinct values for lanes past the end
                    const unsigned m = __match_any_sync(0xFFFFFFFFu, e);
                    const int before = __popc(m & ((1u << lane) - 1u));
                    const int base = v ? s_cnt[e] : 0;
                    __syncwarp();
                    if (v) {
                        s_plist[s_ustart[s_rank[e]] + base + before] = q;
                        if (lane == __ffs(m) - 1) s_cnt[e] = base + __popc(m);
                    }
                    __syncwarp();
                }
            }
            // this CTA's work items in phases C and D: contiguous ranges of equal weight, an
            // item weighing 1 + the pairs of its expert (its rows' load and decode, then one dot
            // per pair); item j of expert u starts at weight nb * (pairs before u + u) + j * (m_u + 1)
            if (warp == 0) {
                const int Us = s_U;
                const int nbs[2] = {nb_gu, nb_dn};
#pragma unroll
                for (int ph2 = 0; ph2 < 2; ph2++) {
                    const int nb = nbs[ph2];
                    const int W = nb * (npair + Us);
                    const int lo = (int)(((long long)W * pid) / P), hi = (int)(((long long)W * (pid + 1)) / P);
                    int clo = 0, chi = 0;  // items starting below lo / below hi
                    for (int u = lane; u < Us; u += 32) {
                        const int m1 = s_ustart[u + 1] - s_ustart[u] + 1, base = nb * (s_ustart[u] + u);
                        clo += lo <= base ? 0 : min(nb, (lo - base + m1 - 1) / m1);
                        chi += hi <= base ? 0 : min(nb, (hi - base + m1 - 1) / m1);
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        clo += __shfl_xor_sync(0xFFFFFFFFu, clo, o);
                        chi += __shfl_xor_sync(0xFFFFFFFFu, chi, o);
                    }
                    if (lane == 0) {
                        s_rng[2 * ph2] = clo;
                        s_rng[2 * ph2 + 1] = chi;
                    }
                }
            }
            __syncthreads();
        }
        BSTAMP(l, 2)
        long long wait_c = 0, wait_d = 0;  // thread 0, traced calls: cycles spent waiting for row copies
        // ------------------------------------------------------------ C: gate/up -> h
        {
            const int c0 = s_rng[0], c1 = s_rng[1];
            // item i -> stage (i - c0) mod stages: gate rows, then up rows, of 16 rows
            auto issue = [&](int i) {
                const int st = (i - c0) % p.stages;
                const int u = i / nb_gu, jb = (i % nb_gu) * kBGuRows;
                const size_t e = (size_t)s_uexp[u];
                unsigned char *dst = ring + (size_t)st * p.stage_bytes;
                const uint32_t bytes = (uint32_t)kBGuRows * rowg, sb = (uint32_t)kBGuRows * 4u;
                mbar_expect_tx(&mb_full[st], 2u * bytes + 2u * sb);
                bulk_g2s(dst, s_ly.gate + (e * f + jb) * rowg, bytes, &mb_full[st]);
                bulk_g2s(dst + bytes, s_ly.up + (e * f + jb) * rowg, bytes, &mb_full[st]);
                bulk_g2s(dst + 2 * bytes, s_ly.sg + e * f + jb, sb, &mb_full[st]);
                bulk_g2s(dst + 2 * bytes + sb, s_ly.su + e * f + jb, sb, &mb_full[st]);
            };
            // the first stages, one item per warp (a lane issues a bulk copy in ~250 cycles; one
            // thread issuing them all would hold its warp for microseconds)
            dr_c0 = c0;
            dr_lo = c0;
            dr_hi = min(c1, c0 + p.stages);
            if (lane == 0 && warp < p.stages && c0 + warp < c1) issue(c0 + warp);
            // the next layer's router rows of this CTA, into L2 ahead of use
            if (tid == 32 * (kBWarps - 1) && has_next && nr > 0)
                prefetch_l2_bulk(p.layer[l + 1].router + (size_t)e0 * d, (uint32_t)(nr * d * 2));
            for (int i = c0; i < c1; i++) {
                const int st = (i - c0) % p.stages;
                const long long tw0 = tt ? clock64() : 0;
                const bool okw = mbar_wait(&mb_full[st], (ph >> st) & 1u, p.limit_ns, p.status);
                if (tt) wait_c += clock64() - tw0;
                if (okw) {
                    ph ^= 1u << st;
                    dr_lo = i + 1;
                }
                const int u = i / nb_gu, j = (i % nb_gu) * kBGuRows + warp;
                const int pa = s_ustart[u], m = s_ustart[u + 1] - pa;
                if (okw) {
                    const unsigned char *stg = ring + (size_t)st * p.stage_bytes;
                    const uint4 wg = *reinterpret_cast<const uint4 *>(stg + (size_t)warp * rowg + lane * 16);
                    const uint4 wu = *reinterpret_cast<const uint4 *>(stg + (size_t)(kBGuRows + warp) * rowg + lane * 16);
                    const float *ssc = reinterpret_cast<const float *>(stg + 2 * (size_t)kBGuRows * rowg);
                    const float sgv = ssc[warp], suv = ssc[kBGuRows + warp];
                    // the dots of each pair; every lane gets the sums (xor reduction) and lane q
                    // keeps pair q's, so the pairs' SwiGLU epilogues run side by side (m <= 16)
                    long long Sg_q = 0, Su_q = 0;
                    for (int q = 0; q < m; q++) {
                        const int t = s_plist[pa + q] / k;
                        SegX<NL> X;
                        seg_load_x_padded<NL>(X, xl + (size_t)t * NL * xlp, xlp, lane);
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
                        if (lane == q) {
                            Sg_q = pair_value(NL, ga, gb2);
                            Su_q = pair_value(NL, ua, ub);
                        }
                    }
                    if (lane < m) {
                        const int pr = s_plist[pa + lane], t = pr / k;
                        float h;
                        if (NL == 1) {
                            const float gv = __fmul_rn(__fmul_rn(__int2float_rn((int)Sg_q), sgv), s_tsc[t]);
                            const float uv = __fmul_rn(__fmul_rn(__int2float_rn((int)Su_q), suv), s_tsc[t]);
                            h = swiglu_f32((double)gv, (double)uv);
                        } else {
                            const double p2 = pow2_f64(-s_tsh[t]);
                            h = swiglu_f32((double)Sg_q * p2 * (double)sgv, (double)Su_q * p2 * (double)suv);
                        }
                        p.h_hist[((size_t)l * npair + pr) * f + j] = h;
                    }
                }
                // the stage is free once every warp is past it
                if (!__syncthreads_and(okw ? 1 : 0)) {
                    alive = false;
                    break;
                }
                // refill: one warp's lane per item, rotating, so no warp carries every issue
                if (i + p.stages < c1) {
                    if (tid == 32 * ((i - c0) % kBWarps)) issue(i + p.stages);
                    dr_hi = i + p.stages + 1;
                }
            }
        }
        if (!alive) break;
        BSTAMP(l, 3)
        if (!grid_sync(gs, &s_flag, !(l == p.stall_layer && pid == 0))) {
            alive = false;
            break;
        }
        BSTAMP(l, 4)
        // ------------------------------------------------------------ D: down -> output rows
        {
            const int c0 = s_rng[2], c1 = s_rng[3];
            auto issue = [&](int i) {
                const int st = (i - c0) % p.stages;
                const int u = i / nb_dn, ib = (i % nb_dn) * rb_dn;
                const size_t e = (size_t)s_uexp[u];
                const uint32_t bytes = (uint32_t)rb_dn * rowd, sb = (uint32_t)rb_dn * 4u;
                mbar_expect_tx(&mb_full[st], bytes + sb);
                bulk_g2s(ring + (size_t)st * p.stage_bytes, s_ly.down + (e * d + ib) * rowd, bytes, &mb_full[st]);
                bulk_g2s(ring + (size_t)st * p.stage_bytes + bytes, s_ly.sd + e * d + ib, sb, &mb_full[st]);
            };
            dr_c0 = c0;
            dr_lo = c0;
            dr_hi = min(c1, c0 + p.stages);
            if (lane == 0 && warp < p.stages && c0 + warp < c1) issue(c0 + warp);
            const int sub = lane / Gf, gl = lane % Gf;
            int cur_u = -1;
            for (int i = c0; i < c1; i++) {
                const int u = i / nb_dn;
                const int pa = s_ustart[u], m = s_ustart[u + 1] - pa;
                if (u != cur_u) {
                    // h limbs of this expert's pairs: warp w builds pair w's (m <= T <= 16)
                    __syncthreads();  // the previous expert's limbs are no longer read
                    if (warp < m) {
                        const int pr = s_plist[pa + warp];
                        const float *hrow = p.h_hist + ((size_t)l * npair + pr) * f;
                        const int per4 = f / 128;  // float4 groups per lane (f / 32 values)
                        float hv[16];
                        float mx = 0.0f;
#pragma unroll
                        for (int g = 0; g < 4; g++) {
                            if (g < per4) {
                                const float4 v = __ldcg(reinterpret_cast<const float4 *>(hrow) + lane * per4 + g);
                                hv[4 * g] = v.x;
                                hv[4 * g + 1] = v.y;
                                hv[4 * g + 2] = v.z;
                                hv[4 * g + 3] = v.w;
                                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                            }
                        }
                        mx = warp_max_f32(mx);
                        const int hsh = (NL == 1) ? 0 : fixed_shift(mx);
                        const float hinv = (NL == 1 && mx > 0.0f) ? quant_inv(mx) : 0.0f;
#pragma unroll
                        for (int g = 0; g < 4; g++) {
                            if (g < per4) {
                                const float v4[4] = {hv[4 * g], hv[4 * g + 1], hv[4 * g + 2], hv[4 * g + 3]};
                                store_limbs4<NL>(hl + (size_t)warp * NL * hlp, hlp, lane * per4 + g, v4, hsh, hinv,
                                                 mx > 0.0f);
                            }
                        }
                        if (lane == 0) {
                            s_hsh[warp] = hsh;
                            s_hsc[warp] = (NL == 1 && mx > 0.0f) ? __fdiv_rn(mx, 127.0f) : 0.0f;
                        }
                    }
                    __syncthreads();
                    cur_u = u;
                }
                const int st = (i - c0) % p.stages;
                const long long tw0 = tt ? clock64() : 0;
                const bool okw = mbar_wait(&mb_full[st], (ph >> st) & 1u, p.limit_ns, p.status);
                if (tt) wait_d += clock64() - tw0;
                if (okw) {
                    ph ^= 1u << st;
                    dr_lo = i + 1;
                }
                if (okw) {
                    const int r = warp * rpp + sub, row = (i % nb_dn) * rb_dn + r;
                    const uint4 wd = *reinterpret_cast<const uint4 *>(ring + (size_t)st * p.stage_bytes + (size_t)r * rowd +
                                                                      gl * 16);
                    const float sdv = reinterpret_cast<const float *>(ring + (size_t)st * p.stage_bytes + (size_t)rb_dn * rowd)[r];
                    for (int q = 0; q < m; q++) {
                        SegX<NL> Hx;
                        seg_load_x_padded<NL>(Hx, hl + (size_t)q * NL * hlp, hlp, gl);
                        int acc[NL];
#pragma unroll
                        for (int z = 0; z < NL; z++) acc[z] = 0;
                        seg_dot_alu<NL>(wd, Hx, acc);
                        int a, b;
                        acc_to_pair_x64<NL>(acc, a, b);
                        for (int o = Gf / 2; o > 0; o >>= 1) {
                            a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
                            if (NL > 1) b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
                        }
                        if (gl == 0) {
                            const long long S = pair_value(NL, a, b);
                            float v;
                            if (NL == 1) v = __fmul_rn(__fmul_rn(__int2float_rn((int)S), sdv), s_hsc[q]);
                            else v = (float)((double)S * pow2_f64(-s_hsh[q]) * (double)sdv);
                            p.yb[(size_t)s_plist[pa + q] * d + row] = v;
                        }
                    }
                }
                if (!__syncthreads_and(okw ? 1 : 0)) {
                    alive = false;
                    break;
                }
                if (i + p.stages < c1) {
                    if (tid == 32 * ((i - c0) % kBWarps)) issue(i + p.stages);
                    dr_hi = i + p.stages + 1;
                }
            }
        }
        if (!alive) break;
        BSTAMP(l, 5)
        if (!grid_sync(gs, &s_flag)) {
            alive = false;
            break;
        }
        BSTAMP(l, 6)
        // ------------------------------------------------------------ E: combine, residual
        // y = sum_q g_q y_q in top-k order (fp64), x' = bf16(x + bf16(y)); rows [r0, r0 + nrow)
        for (int w = tid; w < T * nrow; w += kBThreads) {
            const int t = w / nrow, i = r0 + w % nrow;
            double y = 0.0;
#pragma unroll
            for (int q = 0; q < kBMaxK; q++)
                if (q < k) y += s_gate[t * k + q] * (double)__ldcg(p.yb + (size_t)(t * k + q) * d + i);
            const uint16_t x0 = __ldcg(reinterpret_cast<const unsigned short *>(p.x) + (size_t)t * d + i);
            const uint16_t xo = f64_to_bf16_rne((double)bf16_to_f32(x0) + (double)bf16_to_f32(f64_to_bf16_rne(y)));
            p.x[(size_t)t * d + i] = xo;
            p.hist[((size_t)(l + 1) * T + t) * d + i] = xo;
            p.y_hist[((size_t)l * T + t) * d + i] = (float)y;
        }
        BSTAMP(l, 7)
        if (tt) {
            tt[((size_t)l * P + pid) * kBTracePoints + 13] = (unsigned long long)wait_c;
            tt[((size_t)l * P + pid) * kBTracePoints + 14] = (unsigned long long)wait_d;
        }
        if (has_next && !grid_sync(gs, &s_flag)) {
            alive = false;
            break;
        }
    }
    // after a timeout, let this CTA's own copies in flight land (bounded) before leaving
    if (!alive && tid == 0)
        for (int i = dr_lo; i < dr_hi; i++) {
            const int q = (i - dr_c0) % p.stages;
            mbar_wait(&mb_full[q], (ph >> q) & 1u, p.limit_ns, p.status);
        }
    grid_exit(gs);
#undef BSTAMP
}

// ------------------------------------------------------------------ host side
// Workspace of the small-batch path: control words, logits, expert output rows, per-layer record.
struct BatchWs {
    int64_t ctl, lg, yb, hist, idx, gates, y32, h32, trace, total;
};

static inline int64_t bup256(int64_t v) { return (v + 255) & ~int64_t(255); }

static BatchWs batch_ws_layout(const tern_moe_layer *L0, int64_t T) {
    BatchWs o{};
    int64_t q = 0;
    auto take = [&](int64_t b) {
        const int64_t r = q;
        q = bup256(q + b);
        return r;
    };
    const int64_t d = L0->d, f = L0->f, E = L0->E, k = L0->k;
    o.ctl = take(256);
    o.lg = take(T * E * 8);
    o.yb = take(T * k * d * 4);
    o.hist = take((int64_t)(kMaxLayers + 1) * T * d * 2);
    o.idx = take((int64_t)kMaxLayers * T * k * 4);
    o.gates = take((int64_t)kMaxLayers * T * k * 8);
    o.y32 = take((int64_t)kMaxLayers * T * d * 4);
    o.h32 = take((int64_t)kMaxLayers * T * k * f * 4);
    o.trace = take((int64_t)kMaxLayers * kBMaxCtas * kBTracePoints * 8);
    o.total = q;
    return o;
}

size_t stack_batch_ws_bytes(const tern_moe_layer *L0, int64_t T) { return (size_t)batch_ws_layout(L0, T).total; }

void stack_batch_offsets(const tern_moe_layer *L0, int64_t T, int64_t *hist, int64_t *idx, int64_t *gates,
                         int64_t *y32, int64_t *h32, int64_t *trace) {
    const BatchWs o = batch_ws_layout(L0, T);
    *trace = o.trace;
    *hist = o.hist;
    *idx = o.idx;
    *gates = o.gates;
    *y32 = o.y32;
    *h32 = o.h32;
}

struct BatchPlan {
    int P, stages;
    uint32_t stage_bytes;
    BatchSmem sm;
    const void *fn;
};

static tern_status batch_plan(const tern_moe_layer &L0, int n_layers, int64_t T, tern_act act, BatchPlan &pl) {
    const int d = (int)L0.d, f = (int)L0.f, E = L0.E, k = L0.k;
    // thread mappings: d = 4 * threads and d / 64 = 32 segments (one per lane) per gate/up row;
    // f / 32 values of h per lane in groups of four (f % 128 == 0, f <= 512); f / 64 lanes per
    // down row (a power of two); one top-k warp per token (E <= 256, k <= 8)
    if (T < 2 || T > kBMaxT || n_layers < 1 || n_layers > kMaxLayers) return TERN_EUNSUPPORTED;
    // the scales are bulk-copied with their rows in 16-byte blocks (every layer is checked at launch)
    if (((uintptr_t)L0.gate_scale | (uintptr_t)L0.up_scale | (uintptr_t)L0.down_scale) & 15u) return TERN_EUNSUPPORTED;
    if (d != 4 * kBThreads || k > kBMaxK || E > kBMaxE || f % 128 || f > 512) return TERN_EUNSUPPORTED;
    const int Gf = f / 64;
    if ((Gf & (Gf - 1)) != 0) return TERN_EUNSUPPORTED;
    int dev = 0, sms = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TERN_ECUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TERN_ECUDA;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return TERN_ECUDA;
    const int P = sms;
    if (P < 1 || P > kBMaxCtas || (E + P - 1) / P > kBMaxRouterRows) return TERN_EUNSUPPORTED;
    const int NL = act == TERN_ACT_INT8 ? 1 : 3;
    pl.fn = act == TERN_ACT_INT8 ? (const void *)stack_batch_kernel<1> : (const void *)stack_batch_kernel<3>;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, pl.fn) != cudaSuccess) return TERN_ECUDA;
    const int rb_dn = kBWarps * (32 / Gf);
    // a stage: gate and up rows of a gate/up item and their scales, or the rows of a down item
    // and their scales
    const uint32_t stage = (uint32_t)std::max(2 * kBGuRows * (d / 4) + 2 * kBGuRows * 4, rb_dn * (f / 4) + rb_dn * 4);
    const BatchSmem base = batch_smem(d, E, (int)T, NL, 0, stage);
    const long long room = (long long)optin - (long long)fa.sharedSizeBytes - (long long)base.ring;
    int stages = room > 0 ? (int)(room / stage) : 0;
    if (stages > kBMaxStages) stages = kBMaxStages;
    // the ring also holds phase B's logits and candidates, and phase A's partial sums and x
    const uint32_t ring_min = std::max(batch_topk_bytes(E, (int)T), kBScratchBytes + (uint32_t)T * d * 2);
    while (stages < kBMaxStages && (uint32_t)stages * stage < ring_min) stages++;
    if ((uint32_t)stages * stage < ring_min) return TERN_EUNSUPPORTED;
    if (stages < 2 || (long long)stages * stage > room) return TERN_EUNSUPPORTED;
    pl.P = P;
    pl.stages = stages;
    pl.stage_bytes = stage;
    pl.sm = batch_smem(d, E, (int)T, NL, stages, stage);
    if (cudaFuncSetAttribute(pl.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.sm.total) != cudaSuccess)
        return TERN_ECUDA;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, pl.fn, kBThreads, pl.sm.total) != cudaSuccess)
        return TERN_ECUDA;
    if (nb < 1) return TERN_EUNSUPPORTED;
    return TERN_OK;
}

bool stack_batch_supported(const tern_moe_layer *L0, int n_layers, int64_t T, tern_act act) {
    BatchPlan pl;
    return batch_plan(*L0, n_layers, T, act, pl) == TERN_OK;
}

tern_status launch_stack_batch(const tern_moe_layer *layers, int n_layers, uint16_t *x, int64_t T, float eps,
                               tern_act act, void *ws, size_t ws_bytes, int *status, long long limit_ns,
                               cudaStream_t s, int stall_layer) {
    const tern_moe_layer &L0 = layers[0];
    BatchPlan pl;
    const tern_status pst = batch_plan(L0, n_layers, T, act, pl);
    if (pst != TERN_OK) return pst;
    const BatchWs o = batch_ws_layout(&L0, T);
    if (ws_bytes < (size_t)o.total) return TERN_EWORKSPACE;
    if (!status) return TERN_ECUDA;
    for (int l = 0; l < n_layers; l++)
        if (((uintptr_t)layers[l].gate_scale | (uintptr_t)layers[l].up_scale | (uintptr_t)layers[l].down_scale) & 15u)
            return TERN_EUNSUPPORTED;
    BatchParams prm;
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
    prm.T = (int)T;
    prm.eps = (double)eps;
    prm.x = x;
    prm.ctl = reinterpret_cast<unsigned int *>(b + o.ctl);
    prm.lg = reinterpret_cast<double *>(b + o.lg);
    prm.yb = reinterpret_cast<float *>(b + o.yb);
    prm.hist = reinterpret_cast<uint16_t *>(b + o.hist);
    prm.idx_hist = reinterpret_cast<int32_t *>(b + o.idx);
    prm.gate_hist = reinterpret_cast<double *>(b + o.gates);
    prm.y_hist = reinterpret_cast<float *>(b + o.y32);
    prm.h_hist = reinterpret_cast<float *>(b + o.h32);
    // phase stamps: only when TERNMOE_TRACE=1
    const char *tenv = getenv("TERNMOE_TRACE");
    prm.ttrace = (tenv && tenv[0] == '1') ? reinterpret_cast<unsigned long long *>(b + o.trace) : nullptr;
    prm.status = status;
    prm.limit_ns = limit_ns;
    prm.limit_cycles = 2 * limit_ns;  // SM clocks <= 2 GHz
    prm.P = pl.P;
    prm.stages = pl.stages;
    prm.stall_layer = stall_layer;
    prm.stage_bytes = pl.stage_bytes;
    void *args[] = {&prm};
    const cudaError_t e = cudaLaunchCooperativeKernel(pl.fn, dim3(pl.P), dim3(kBThreads), args, pl.sm.total, s);
    return e == cudaSuccess ? TERN_OK : TERN_ECUDA;
}

}  // namespace tern
