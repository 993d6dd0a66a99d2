// flashhead.cu -- approximate output head: score 4-bit cluster centroids, keep the top
// clusters, project only their tokens (sm_100a).
//
// "A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "The
// Architecture: Designed for the Hardware": the projection to a ~151,000-token vocabulary is
// the most expensive part of decode; clustering the vocabulary into 4,748 groups, scoring
// 4-bit centroids and computing full-precision projections only for the top 512 clusters
// turns O(hidden x vocab) into much less.  Layout: the vocabulary is stored cluster-major
// (cluster c = tokens c*cs .. c*cs+cs-1); a centroid is the mean of its cluster's bf16 rows,
// stored as symmetric int4 in [-7, 7] (two per byte, element 2j in the low nibble) with one
// fp64 scale = absmax / 7.  Scores and candidate logits are fp64 sums of exact products
// (int4 x bf16 and bf16 x bf16 products fit fp64), one fused multiply-add each.
//
// Kernels: centroid (offline preparation), score (warp per cluster), select (one CTA: radix
// select of the top clusters then their ranks, or for more than 1,024 of them a bitonic sort
// by (score desc, index asc)), logits (warp per candidate token),
// best (one CTA, candidate with the largest logit, ties to the lower token id).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ternmoe.h"
#include "tern_common.cuh"

namespace {

using namespace tern;

constexpr int kFhWarps = 8;
constexpr int kFhMaxClusters = 8192;
constexpr int kFhSelectThreads = 1024;
constexpr int64_t kFhMaxD = 8192;

__device__ __forceinline__ double bf16_f64(uint16_t b) { return (double)bf16_to_f32(b); }

__device__ __forceinline__ double block_max_f64(double v, double *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double m = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) m = fmax(m, red[w]);
    __syncthreads();
    return m;
}

// centroid element k of cluster c: the exact mean of its cs rows (sums of bf16 values fit fp64)
__device__ __forceinline__ double centroid_at(const uint16_t *W, int64_t d, int cs, int c, int64_t k) {
    double s = 0.0;
    for (int r = 0; r < cs; r++) s += bf16_f64(W[((int64_t)c * cs + r) * d + k]);
    return s / (double)cs;
}

__device__ __forceinline__ int quant4_one(double v, double scale) {
    if (!(scale > 0.0)) return 0;
    double q = rint(v / scale);
    q = q > 7.0 ? 7.0 : (q < -7.0 ? -7.0 : q);
    return (int)q;
}

__global__ void fh_centroid_kernel(const uint16_t *__restrict__ W, int64_t d, int cs, uint8_t *__restrict__ C4,
                                   double *__restrict__ scale) {
    __shared__ double red[32];
    const int c = blockIdx.x;
    double m = 0.0;
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x) m = fmax(m, fabs(centroid_at(W, d, cs, c, k)));
    const double sc = block_max_f64(m, red) / 7.0;
    if (threadIdx.x == 0) scale[c] = sc;
    for (int64_t j = threadIdx.x; j < d / 2; j += blockDim.x) {
        const int q0 = quant4_one(centroid_at(W, d, cs, c, 2 * j), sc);
        const int q1 = quant4_one(centroid_at(W, d, cs, c, 2 * j + 1), sc);
        C4[(int64_t)c * (d / 2) + j] = (uint8_t)(((uint32_t)q0 & 0xFu) | (((uint32_t)q1 & 0xFu) << 4));
    }
}

__device__ __forceinline__ void stage_x64(const uint16_t *x, int64_t d, double *xs) {
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x) xs[k] = bf16_f64(x[k]);
    __syncthreads();
}

__global__ void __launch_bounds__(kFhWarps * 32) fh_score_kernel(const uint8_t *__restrict__ C4,
                                                                  const double *__restrict__ scale,
                                                                  const uint16_t *__restrict__ x, int64_t d, int nc,
                                                                  double *__restrict__ scores) {
    extern __shared__ double xs[];
    stage_x64(x, d, xs);
    const int lane = threadIdx.x & 31;
    const int c = blockIdx.x * kFhWarps + (threadIdx.x >> 5);
    if (c >= nc) return;
    const uint8_t *row = C4 + (int64_t)c * (d / 2);
    double acc = 0.0;
    for (int64_t j = lane; j < d / 2; j += 32) {
        const int b = row[j];
        const int lo = (b & 0x7) - (b & 0x8), hi = ((b >> 4) & 0x7) - ((b >> 4) & 0x8);  // sign-extended nibbles
        acc = fma((double)lo, xs[2 * j], acc);
        acc = fma((double)hi, xs[2 * j + 1], acc);
    }
    acc = warp_sum_f64(acc);
    if (lane == 0) scores[c] = acc * scale[c];
}

__device__ __forceinline__ bool fh_before(unsigned long long ka, int ia, unsigned long long kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

__global__ void __launch_bounds__(kFhSelectThreads) fh_select_kernel(const double *__restrict__ scores, int nc, int N,
                                                                      int top_c, int32_t *__restrict__ sel) {
    extern __shared__ unsigned long long sk[];  // [N] keys, then [N] indices
    int *si = reinterpret_cast<int *>(sk + N);
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
        sk[i] = (i < nc) ? f64_order_key(scores[i]) : 0ull;  // padding sorts last
        si[i] = (i < nc) ? i : 0x7FFFFFFF;
    }
    __syncthreads();
    for (int size = 2; size <= N; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < N; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool up = (i & size) == 0;
                    const bool first = fh_before(sk[i], si[i], sk[j], si[j]);
                    if (up != first) {
                        const unsigned long long tk = sk[i];
                        sk[i] = sk[j];
                        sk[j] = tk;
                        const int ti = si[i];
                        si[i] = si[j];
                        si[j] = ti;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int q = threadIdx.x; q < top_c; q += blockDim.x) sel[q] = si[q];
}

// Top top_c clusters (top_c <= kFhRadixMax) without sorting all of them, one CTA:
//  1. tau = the top_c-th largest order key: MSB-first radix select, 8 passes of 8-bit digits,
//     each a 256-bin histogram (shared atomics) of the keys that match the digits chosen so
//     far, then one warp finds the bin where the count from the top reaches the rank sought;
//  2. every key above tau is kept, and of the keys equal to tau the `need` ones with the
//     lowest indices (a block scan in index order);
//  3. each kept cluster's output position = how many kept clusters come before it (larger
//     key, or the same key and a lower index).
constexpr int kFhRadixMax = 1024;

__global__ void __launch_bounds__(kFhSelectThreads) fh_select_radix_kernel(const double *__restrict__ scores, int nc,
                                                                            int top_c, int32_t *__restrict__ sel) {
    constexpr int J = kFhMaxClusters / kFhSelectThreads;  // clusters per thread
    __shared__ int s_hist[256];
    __shared__ int s_bin, s_need, s_cnt;
    __shared__ int s_wsum[kFhSelectThreads / 32];
    __shared__ unsigned long long s_k[kFhRadixMax];
    __shared__ int s_i[kFhRadixMax];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned long long key[J];
#pragma unroll
    for (int j = 0; j < J; j++) {
        const int i = tid + j * kFhSelectThreads;
        key[j] = i < nc ? f64_order_key(scores[i]) : 0ull;
    }
    unsigned long long prefix = 0ull, mask = 0ull;
    int need = top_c;  // rank sought among the keys that match the prefix (1 = largest)
    for (int shift = 56; shift >= 0; shift -= 8) {
        if (tid < 256) s_hist[tid] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < J; j++)
            if (tid + j * kFhSelectThreads < nc && (key[j] & mask) == prefix)
                atomicAdd(&s_hist[(int)((key[j] >> shift) & 255ull)], 1);
        __syncthreads();
        if (warp == 0) {
            // lane l holds bins 255 - 8l .. 248 - 8l (from the top)
            int c[8], tot = 0;
#pragma unroll
            for (int q = 0; q < 8; q++) {
                c[q] = s_hist[255 - 8 * lane - q];
                tot += c[q];
            }
            int incl = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            const int excl = incl - tot;
            if (excl < need && need <= incl) {
                int cum = excl;
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    if (cum < need && cum + c[q] >= need) {
                        s_bin = 255 - 8 * lane - q;
                        s_need = need - cum;
                    }
                    cum += c[q];
                }
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)s_bin << shift;
        mask |= 255ull << shift;
        need = s_need;
        __syncthreads();
    }
    const unsigned long long tau = prefix;  // need = clusters with key tau to keep
    if (tid == 0) s_cnt = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < J; j++) {
        const int i = tid + j * kFhSelectThreads;
        if (i < nc && key[j] > tau) s_i[atomicAdd(&s_cnt, 1)] = i;
    }
    // the ties, in index order (item (tid, j) has index j * threads + tid)
    int base = 0;
#pragma unroll
    for (int j = 0; j < J; j++) {
        const int i = tid + j * kFhSelectThreads;
        const bool eq = i < nc && key[j] == tau;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, eq);
        if (lane == 0) s_wsum[warp] = __popc(bal);
        __syncthreads();
        int before = 0, all = 0;
        for (int w = 0; w < kFhSelectThreads / 32; w++) {
            before += w < warp ? s_wsum[w] : 0;
            all += s_wsum[w];
        }
        const int r = base + before + __popc(bal & ((1u << lane) - 1u));
        if (eq && r < need) s_i[atomicAdd(&s_cnt, 1)] = i;
        base += all;
        __syncthreads();
    }
    for (int t = tid; t < top_c; t += kFhSelectThreads) s_k[t] = f64_order_key(scores[s_i[t]]);
    __syncthreads();
    for (int t = tid; t < top_c; t += kFhSelectThreads) {
        const unsigned long long kt = s_k[t];
        const int it = s_i[t];
        int r = 0;
        for (int u = 0; u < top_c; u++) r += fh_before(s_k[u], s_i[u], kt, it) ? 1 : 0;
        sel[r] = it;
    }
}

// acc + w * x for bf16 w and x, with one rounding (as fma in fp64): the product of two bf16
// values (8 significant bits each) is exact in fp32 unless it leaves fp32's normal range, so it
// is formed there and added in fp64; the rare product outside that range takes the fp64 path
__device__ __forceinline__ double fh_add_prod(double acc, float w, float x) {
    const float p = __fmul_rn(w, x);
    const float ap = fabsf(p);
    if ((ap >= 1.17549435e-38f && ap <= 3.40282347e38f) || w == 0.0f || x == 0.0f) return acc + (double)p;
    return fma((double)w, (double)x, acc);
}

__global__ void __launch_bounds__(kFhWarps * 32) fh_logits_kernel(const uint16_t *__restrict__ W,
                                                                   const uint16_t *__restrict__ x, int64_t d, int cs,
                                                                   const int32_t *__restrict__ sel, int ncand,
                                                                   int32_t *__restrict__ ids,
                                                                   double *__restrict__ logits) {
    // x in fp32 (exact): each lane reads four consecutive values per step, one 16-byte load,
    // consecutive lanes consecutive addresses (no bank conflict)
    extern __shared__ float xsf[];
    for (int64_t k = threadIdx.x; k < d; k += blockDim.x) xsf[k] = bf16_to_f32(x[k]);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int q = blockIdx.x * kFhWarps + (threadIdx.x >> 5);
    if (q >= ncand) return;
    const int v = sel[q / cs] * cs + q % cs;
    const uint2 *row = reinterpret_cast<const uint2 *>(W + (int64_t)v * d);
    const float4 *x4 = reinterpret_cast<const float4 *>(xsf);
    double acc = 0.0;
    for (int64_t ch = lane; ch < d / 4; ch += 32) {
        const uint2 wv = __ldg(row + ch);
        const float4 xv = x4[ch];
        acc = fh_add_prod(acc, bf16_to_f32((uint16_t)(wv.x & 0xFFFFu)), xv.x);
        acc = fh_add_prod(acc, bf16_to_f32((uint16_t)(wv.x >> 16)), xv.y);
        acc = fh_add_prod(acc, bf16_to_f32((uint16_t)(wv.y & 0xFFFFu)), xv.z);
        acc = fh_add_prod(acc, bf16_to_f32((uint16_t)(wv.y >> 16)), xv.w);
    }
    acc = warp_sum_f64(acc);
    if (lane == 0) {
        ids[q] = v;
        logits[q] = acc;
    }
}

__global__ void __launch_bounds__(1024) fh_best_kernel(const int32_t *__restrict__ ids,
                                                       const double *__restrict__ logits, int n,
                                                       int32_t *__restrict__ best) {
    __shared__ unsigned long long s_k[32];
    __shared__ int s_i[32];
    unsigned long long bk = 0ull;
    int bi = 0x7FFFFFFF;
    for (int q = threadIdx.x; q < n; q += blockDim.x) {
        const unsigned long long k = f64_order_key(logits[q]);
        const int id = ids[q];
        if (fh_before(k, id, bk, bi)) {
            bk = k;
            bi = id;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long ok = __shfl_xor_sync(0xFFFFFFFFu, bk, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (fh_before(ok, oi, bk, bi)) {
            bk = ok;
            bi = oi;
        }
    }
    if ((threadIdx.x & 31) == 0) {
        s_k[threadIdx.x >> 5] = bk;
        s_i[threadIdx.x >> 5] = bi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); w++)
            if (fh_before(s_k[w], s_i[w], bk, bi)) {
                bk = s_k[w];
                bi = s_i[w];
            }
        best[0] = bi;
    }
}

inline bool fh_aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

bool fh_shape_ok(int64_t d, int32_t nc, int32_t cs) {
    return d >= 64 && d <= kFhMaxD && d % 64 == 0 && nc >= 1 && nc <= kFhMaxClusters && cs >= 1 && cs <= 1024;
}

}  // namespace

extern "C" tern_status flash_head_centroids(const uint16_t *W, int64_t d, int32_t n_clusters, int32_t cluster_size,
                                            uint8_t *C4, double *c_scale, void *stream) {
    if (!W || !C4 || !c_scale || !fh_shape_ok(d, n_clusters, cluster_size)) return TERN_EINVAL;
    if (!fh_aligned(W, 16) || !fh_aligned(c_scale, 8)) return TERN_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    fh_centroid_kernel<<<n_clusters, 256, 0, s>>>(W, d, cluster_size, C4, c_scale);
    return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ECUDA;
}

extern "C" tern_status flash_head(const uint8_t *C4, const double *c_scale, const uint16_t *W, const uint16_t *x,
                                  int64_t d, int32_t n_clusters, int32_t cluster_size, int32_t top_c, double *scores,
                                  int32_t *sel_clusters, int32_t *cand_ids, double *cand_logits, int32_t *best_id,
                                  void *stream) {
    if (!C4 || !c_scale || !W || !x || !scores || !sel_clusters || !cand_ids || !cand_logits || !best_id)
        return TERN_EINVAL;
    if (!fh_shape_ok(d, n_clusters, cluster_size) || top_c < 1 || top_c > n_clusters) return TERN_EINVAL;
    if ((int64_t)top_c * cluster_size > (1ll << 30)) return TERN_EINVAL;
    if (!fh_aligned(W, 16) || !fh_aligned(x, 2) || !fh_aligned(c_scale, 8) || !fh_aligned(scores, 8) ||
        !fh_aligned(sel_clusters, 4) || !fh_aligned(cand_ids, 4) || !fh_aligned(cand_logits, 8) ||
        !fh_aligned(best_id, 4))
        return TERN_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t xs_bytes = (size_t)d * sizeof(double);  // x as fp64, up to 64 KB
    cudaFuncSetAttribute(fh_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)xs_bytes);

    fh_score_kernel<<<(n_clusters + kFhWarps - 1) / kFhWarps, kFhWarps * 32, xs_bytes, s>>>(C4, c_scale, x, d,
                                                                                           n_clusters, scores);
    if (cudaGetLastError() != cudaSuccess) return TERN_ECUDA;
    if (top_c <= kFhRadixMax) {
        fh_select_radix_kernel<<<1, kFhSelectThreads, 0, s>>>(scores, n_clusters, top_c, sel_clusters);
    } else {
        int N = 1;
        while (N < n_clusters) N <<= 1;
        const size_t sel_bytes = (size_t)N * (sizeof(unsigned long long) + sizeof(int));
        cudaFuncSetAttribute(fh_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_bytes);
        fh_select_kernel<<<1, kFhSelectThreads, sel_bytes, s>>>(scores, n_clusters, N, top_c, sel_clusters);
    }
    if (cudaGetLastError() != cudaSuccess) return TERN_ECUDA;
    const int ncand = top_c * cluster_size;
    fh_logits_kernel<<<(ncand + kFhWarps - 1) / kFhWarps, kFhWarps * 32, (size_t)d * sizeof(float), s>>>(W, x, d, cluster_size,
                                                                                       sel_clusters, ncand, cand_ids,
                                                                                       cand_logits);
    if (cudaGetLastError() != cudaSuccess) return TERN_ECUDA;
    fh_best_kernel<<<1, 1024, 0, s>>>(cand_ids, cand_logits, ncand, best_id);
    return cudaGetLastError() == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
