// tern_common.cuh -- device helpers shared by the sm_100a kernels of libternmoe.
//
// Ternary decode without unpacking: a packed byte holds four 2-bit codes (00 -> 0,
// 01 -> +1, 10 -> -1, little-endian along K).  Each byte is turned into four signed int8
// lanes by ONE shared-memory table read (a 256-entry table replicated per lane so every
// lane reads its own bank), and the four products with activations happen in ONE dp4a.
// This is the integer-unit form of "negate, zero, or pass through" ("A 20B AI Model Trained
// in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What Ternary Actually
// Means"): the weights are never widened to bf16 and no floating-point multiply is issued
// per weight.
//
// Activations enter as integer "limbs":
//   int8 path: one signed limb (the quantised value);
//   bf16/fp32 path: a 24-bit fixed-point value x_int = rint(x * 2^s) with s chosen per
//     vector so that |x_int| < 2^23, split into hi (signed 8 bit), mid and lo (unsigned
//     8 bit): x_int = hi*65536 + mid*256 + lo.  The dot is then exact in integers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ternmoe.h"
#include "decode.cuh"

namespace tern {

constexpr int kWarp = 32;

// ------------------------------------------------------------------ device status word
// A per-device int owned by the library (first error wins; read and cleared by
// tern_stream_status()); kernels receive its address.
__device__ __forceinline__ void set_status(int *st, int code) {
    if (st) atomicCAS(st, 0, code);
}

// ---------------------------------------------------------------------------- bf16 / fp64
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Nearest bf16 (ties to even) of a double.  Two roundings are exact here when the first is
// round-to-odd and keeps at least two more bits than the second (fp32 keeps 16 more than
// bf16): truncate to fp32, set the last fp32 bit if anything was cut off (round to odd),
// then round the fp32 value to nearest-even bf16 with an integer add.  Finite inputs of any
// magnitude below fp32 overflow (values that would round past bf16 max become inf).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
    float f = __double2float_rz(v);
    if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// bf16 -> fp64 by moving bits (normal values); zero, subnormal, inf and nan go through fp32
__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
    const uint32_t e = (b >> 7) & 0xFFu;
    if (e == 0u || e == 0xFFu) return (double)bf16_to_f32(b);
    const unsigned long long bits = ((unsigned long long)(b & 0x8000u) << 48) |
                                    ((unsigned long long)(e + 896u) << 52) | ((unsigned long long)(b & 0x7Fu) << 45);
    return __longlong_as_double((long long)bits);
}

// 2^e as a double, exact, for -1022 <= e <= 1023 (multiplying an integer-valued double by it
// is exact, like ldexp, as long as the product stays in the normal range)
__device__ __forceinline__ double pow2_f64(int e) {
    return __longlong_as_double((long long)(unsigned long long)(1023 + e) << 52);
}

// bf16(x / r), nearest even, as f64_to_bf16_rne(x / r), from q = x * rinv (rinv = 1 / r rounded):
// q is within a few units in the last place of the exact quotient, so its bf16 rounding is the
// quotient's unless q lies within 8 units of a point halfway between two bf16 values (or outside
// the normal bf16 range); those take the exact division.  The rounding itself is integer
// arithmetic on q's bits: the top 19 bits (sign, exponent, 7 mantissa bits) plus one when the
// 45 bits below exceed the halfway point or equal it with an odd last kept bit.
// the exact path, out of line: it is rare, and an inlined fp64 division per call site would
// multiply the code of loops that call this many times
static __device__ __noinline__ uint16_t bf16_of_exact_quotient(double x, double r) { return f64_to_bf16_rne(x / r); }

__device__ __forceinline__ uint16_t bf16_of_quotient(double x, double r, double rinv) {
    const double q = x * rinv;
    const unsigned long long b = (unsigned long long)__double_as_longlong(q);
    const unsigned long long low = b & ((1ull << 45) - 1), half = 1ull << 44;
    const long long dist = (long long)low - (long long)half;
    const uint32_t e11 = (uint32_t)(b >> 52) & 0x7FFu;
    if (dist >= -8 && dist <= 8) return bf16_of_exact_quotient(x, r);  // near a tie: exact path
    if (e11 < 1023 - 126 + 1 || e11 > 1023 + 127 - 1) return bf16_of_exact_quotient(x, r);  // not a normal bf16
    uint32_t t = (uint32_t)(b >> 45);                                   // sign | e11 | 7 mantissa bits
    t += (dist > 0) ? 1u : 0u;                                          // no ties here (|dist| > 8)
    const uint32_t sign = (t >> 18) & 1u, e = (t >> 7) & 0x7FFu, m = t & 0x7Fu;
    return (uint16_t)((sign << 15) | ((e - 896u) << 7) | m);
}

// ---------------------------------------------------------------------------- dp4a
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
    return __dp4a((int)a, (int)b, c);
}
// a: signed int8x4 (ternary weights), b: unsigned 8-bit limbs
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// -------------------------------------------------------------------- decode table
// Entry b (a packed byte) holds the four weights of b as signed int8 lanes (byte j = code j),
// replicated in 32 lane-private columns: entry stride 256 bytes, lane l reads column l, so
// lanes never share a bank.  The stride lets ONE byte-permute build the whole shared-memory
// offset of a lookup: (packed byte << 8) | (lane << 2).
constexpr int kLutStrideWords = 64;
constexpr int kLutWords = 256 * kLutStrideWords;
constexpr int kLutBytes = kLutWords * 4;  // 64 KB (columns 32..63 unused)

__device__ __forceinline__ uint32_t decode_byte(uint32_t b) {
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const uint32_t c = (b >> (2 * j)) & 3u;
        const uint32_t v = (c == 1u) ? 0x01u : (c == 2u) ? 0xFFu : 0x00u;
        out |= v << (8 * j);
    }
    return out;
}

__device__ __forceinline__ void lut_fill(uint32_t *lut) {
    for (int i4 = threadIdx.x; i4 < 256 * 8; i4 += blockDim.x) {
        const uint32_t b = (uint32_t)i4 >> 3;
        const uint32_t v = decode_byte(b);
        reinterpret_cast<uint4 *>(lut + b * kLutStrideWords)[i4 & 7] = make_uint4(v, v, v, v);
    }
}

// ------------------------------------------------------------------- segment dot
// A "segment" is 64 consecutive codes = 16 packed bytes (one uint4).  xw[l][b] holds limb l
// of the four activations that meet byte b of the segment.
template <int NL>
struct SegX {
    uint32_t w[NL][16];
};

// lane4 = lane * 4 (the lane's column offset in bytes)
template <int NL>
__device__ __forceinline__ void seg_dot(const uint4 wb, const SegX<NL> &x, const uint32_t *lut, uint32_t lane4,
                                        int (&acc)[NL]) {
    const char *lb = reinterpret_cast<const char *>(lut);
    const uint32_t words[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int q = 0; q < 4; q++) {
#pragma unroll
        for (int i = 0; i < 4; i++) {
            // result byte 0 = lane4, byte 1 = packed byte i, bytes 2-3 = 0 (byte 1 of lane4)
            const uint32_t off = __byte_perm(words[q], lane4, 0x5504u | ((uint32_t)i << 4));
            const uint32_t wv = *reinterpret_cast<const uint32_t *>(lb + off);
            const int bb = 4 * q + i;
            if (NL == 1) {
                acc[0] = dp4a_ss(wv, x.w[0][bb], acc[0]);
            } else {
                acc[0] = dp4a_ss(wv, x.w[0][bb], acc[0]);   // hi limb: signed
                acc[1] = dp4a_su(wv, x.w[1][bb], acc[1]);   // mid limb: unsigned
                acc[2] = dp4a_su(wv, x.w[2][bb], acc[2]);   // lo limb: unsigned
            }
        }
    }
}

// The same segment dot without a table (decode.cuh): x holds the limbs in position-major
// order (word 4q+j of limb l = the four activations of position j of packed word q).  Every
// dp4a term is 64 times a weight-activation product, so acc is 64 times the limb dot; use
// acc_to_pair_x64 to reduce it.
template <int NL>
__device__ __forceinline__ void seg_dot_alu(const uint4 wb, const SegX<NL> &x, int (&acc)[NL]) {
    const uint32_t words[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint32_t sgn = tern_signed_fields(words[q]);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t m = tern_position_lanes(sgn, j);
            const int bb = 4 * q + j;
            acc[0] = dp4a_ss(m, x.w[0][bb], acc[0]);
            if (NL > 1) {
                acc[1] = dp4a_su(m, x.w[1][bb], acc[1]);
                acc[2] = dp4a_su(m, x.w[2][bb], acc[2]);
            }
        }
    }
}

// load the limbs of one segment from a limb-word array laid out [NL][n/4] (u32 words)
template <int NL>
__device__ __forceinline__ void seg_load_x(SegX<NL> &x, const uint32_t *limbw, int64_t words_per_limb,
                                           int64_t seg) {
#pragma unroll
    for (int l = 0; l < NL; l++) {
        const uint4 *p = reinterpret_cast<const uint4 *>(limbw + (int64_t)l * words_per_limb + seg * 16);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const uint4 t = __ldg(p + v);
            x.w[l][4 * v + 0] = t.x;
            x.w[l][4 * v + 1] = t.y;
            x.w[l][4 * v + 2] = t.z;
            x.w[l][4 * v + 3] = t.w;
        }
    }
}

// same, from shared memory
template <int NL>
__device__ __forceinline__ void seg_load_x_smem(SegX<NL> &x, const uint32_t *limbw, int words_per_limb, int seg) {
#pragma unroll
    for (int l = 0; l < NL; l++) {
        const uint4 *p = reinterpret_cast<const uint4 *>(limbw + l * words_per_limb + seg * 16);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const uint4 t = p[v];
            x.w[l][4 * v + 0] = t.x;
            x.w[l][4 * v + 1] = t.y;
            x.w[l][4 * v + 2] = t.z;
            x.w[l][4 * v + 3] = t.w;
        }
    }
}

// Padded limb layout in shared memory: the 16 words of segment g start at word 20*g, so the
// 128-bit loads of 8 lanes reading 8 different segments fall in 8 different bank groups.
constexpr int kSegPad = 20;
__device__ __forceinline__ int padded_word(int w) { return (w >> 4) * kSegPad + (w & 15); }

template <int NL>
__device__ __forceinline__ void seg_load_x_padded(SegX<NL> &x, const uint32_t *limbw, int words_per_limb_padded,
                                                  int seg) {
#pragma unroll
    for (int l = 0; l < NL; l++) {
        const uint4 *p = reinterpret_cast<const uint4 *>(limbw + l * words_per_limb_padded + seg * kSegPad);
#pragma unroll
        for (int v = 0; v < 4; v++) {
            const uint4 t = p[v];
            x.w[l][4 * v + 0] = t.x;
            x.w[l][4 * v + 1] = t.y;
            x.w[l][4 * v + 2] = t.z;
            x.w[l][4 * v + 3] = t.w;
        }
    }
}

// Per-lane partial sums -> at most two int32 for the cross-lane reduction.
// NL == 3: hi stays separate, (mid*256 + lo) is combined; both fit int32 for <= 256 codes
// per lane and 32 lanes.
template <int NL>
__device__ __forceinline__ void acc_to_pair(const int (&acc)[NL], int &a, int &b) {
    if (NL == 1) {
        a = acc[0];
        b = 0;
    } else {
        a = acc[0];
        b = acc[1] * 256 + acc[2];
    }
}

// acc_to_pair for accumulators of seg_dot_alu (64 times the limb dot; exact shift)
template <int NL>
__device__ __forceinline__ void acc_to_pair_x64(const int (&acc)[NL], int &a, int &b) {
    if (NL == 1) {
        a = acc[0] >> 6;
        b = 0;
    } else {
        a = acc[0] >> 6;
        b = (acc[1] >> 6) * 256 + (acc[2] >> 6);
    }
}

__device__ __forceinline__ long long pair_value(int NLv, int a, int b) {
    return NLv == 1 ? (long long)a : (long long)a * 65536ll + (long long)b;
}

// xor-reduce within aligned groups of G lanes
template <int G>
__device__ __forceinline__ int group_sum(int v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Two rows at once: vA, vB are a lane's partials of rows A and B in its aligned group of G
// lanes (G >= 2).  The first level trades halves (one shuffle serves both rows), the rest
// reduce within half groups.  Afterwards the group's lane 0 holds row A's sum and its lane
// G/2 holds row B's.
template <int G>
__device__ __forceinline__ int group_sum2(int vA, int vB) {
    const int lane = threadIdx.x & 31;
    const bool upper = (lane & (G / 2)) != 0;
    int v = (upper ? vB : vA) + __shfl_xor_sync(0xFFFFFFFFu, upper ? vA : vB, G / 2);
#pragma unroll
    for (int o = G / 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// block-wide max of non-negative floats (all threads get the result); red >= 32 floats
__device__ __forceinline__ float block_max_f32(float v, float *red) {
    v = warp_max_f32(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    const int nw = (blockDim.x + 31) >> 5;
    float r = (l < nw) ? red[l] : 0.0f;
    r = warp_max_f32(r);
    return r;
}

// ------------------------------------------------------- fixed-point activation limbs
// Shift s such that |x| * 2^s < 2^23 for every element (s = 22 - floor(log2(absmax))).
__device__ __forceinline__ int fixed_shift(float absmax) {
    if (!(absmax > 0.0f)) return 0;
    const int be = (__float_as_int(absmax) >> 23) & 0xFF;  // biased exponent
    if (be == 0) return 22 - ilogbf(absmax);               // subnormal absmax
    return 22 - (be - 127);
}

// x_int = rint(x * 2^s) split into three bytes: hi (signed), mid, lo (unsigned).  x * 2^s is
// a power-of-two scale, exact unless it lands below the fp32 normal range, where it rounds
// to zero either way.
__device__ __forceinline__ void fixed_limbs(float x, int s, uint32_t &hi, uint32_t &mid, uint32_t &lo) {
    const bool fast = (s >= -126 && s <= 127);
    const float sx = fast ? __fmul_rn(x, __int_as_float((127 + s) << 23)) : scalbnf(x, s);
    const int xi = __float2int_rn(sx);
    hi = (uint32_t)(xi >> 16) & 0xFFu;
    mid = (uint32_t)(xi >> 8) & 0xFFu;
    lo = (uint32_t)xi & 0xFFu;
}

// ---------------------------------------------------------------------------- top-k
// Order-preserving 64-bit key of a finite double (larger double -> larger unsigned key;
// -0.0 and +0.0 map to the same key).
__device__ __forceinline__ unsigned long long f64_order_key(double v) {
    if (v == 0.0) v = 0.0;  // fold -0.0 into +0.0
    const unsigned long long u = (unsigned long long)__double_as_longlong(v);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

template <int J>
__device__ __forceinline__ void topk_cas(unsigned long long (&key)[J], int (&ix)[J], int a, int b) {
    // afterwards (key[a], ix[a]) ranks first: larger key, then lower index
    const bool sw = (key[b] > key[a]) || (key[b] == key[a] && ix[b] < ix[a]);
    const unsigned long long ka = key[a], kb = key[b];
    const int ia = ix[a], ib = ix[b];
    key[a] = sw ? kb : ka;
    key[b] = sw ? ka : kb;
    ix[a] = sw ? ib : ia;
    ix[b] = sw ? ia : ib;
}

// One warp selects the top k (k <= 8) of E fp64 logits: descending value, ties to the lower
// index.  Lane l owns experts l, l+32, ...; each lane sorts its candidates once (Batcher's
// network for 8), then every round the best lane head wins; the winning lane writes
// idx_out[r] and pops its head.  Heads tie on the high key word only when two logits share
// sign, exponent and 20 leading mantissa bits; then the low word, then the index decide.
// idx_out must be visible to the whole warp afterwards (shared or global memory).
template <int J>
__device__ __forceinline__ void warp_topk_select(const double *lg, int E, int k, int32_t *idx_out) {
    const int lane = threadIdx.x & 31;
    unsigned long long key[J];
    int ix[J];
#pragma unroll
    for (int j = 0; j < J; j++) {
        const int e = lane + 32 * j;
        key[j] = (e < E) ? f64_order_key(lg[e]) : 0ull;  // 0 = below every finite logit
        ix[j] = (e < E) ? e : 0x7FFFFFFF;
    }
    if (J == 8) {
        topk_cas<J>(key, ix, 0, 1); topk_cas<J>(key, ix, 2, 3); topk_cas<J>(key, ix, 4, 5); topk_cas<J>(key, ix, 6, 7);
        topk_cas<J>(key, ix, 0, 2); topk_cas<J>(key, ix, 1, 3); topk_cas<J>(key, ix, 4, 6); topk_cas<J>(key, ix, 5, 7);
        topk_cas<J>(key, ix, 1, 2); topk_cas<J>(key, ix, 5, 6);
        topk_cas<J>(key, ix, 0, 4); topk_cas<J>(key, ix, 1, 5); topk_cas<J>(key, ix, 2, 6); topk_cas<J>(key, ix, 3, 7);
        topk_cas<J>(key, ix, 2, 4); topk_cas<J>(key, ix, 3, 5);
        topk_cas<J>(key, ix, 1, 2); topk_cas<J>(key, ix, 3, 4); topk_cas<J>(key, ix, 5, 6);
    } else {
#pragma unroll
        for (int a = 0; a < J; a++)
#pragma unroll
            for (int b = 0; b < J - 1 - a; b++) topk_cas<J>(key, ix, b, b + 1);
    }
    for (int r = 0; r < k; r++) {
        const unsigned hi = (unsigned)(key[0] >> 32);
        const unsigned mhi = __reduce_max_sync(0xFFFFFFFFu, hi);
        unsigned cand = __ballot_sync(0xFFFFFFFFu, hi == mhi);
        if (__popc(cand) > 1) {
            const unsigned lo = (unsigned)key[0];
            const unsigned mlo = __reduce_max_sync(0xFFFFFFFFu, hi == mhi ? lo : 0u);
            const bool c2 = (hi == mhi) && (lo == mlo);
            const unsigned mi = __reduce_min_sync(0xFFFFFFFFu, c2 ? (unsigned)ix[0] : 0xFFFFFFFFu);
            cand = __ballot_sync(0xFFFFFFFFu, c2 && (unsigned)ix[0] == mi);
        }
        if (lane == __ffs(cand) - 1) {
            // finite logits always select a valid expert; NaN inputs must still not index out of range
            idx_out[r] = (ix[0] >= 0 && ix[0] < E) ? ix[0] : r;
#pragma unroll
            for (int j = 0; j < J - 1; j++) {
                key[j] = key[j + 1];
                ix[j] = ix[j + 1];
            }
            key[J - 1] = 0ull;
            ix[J - 1] = 0x7FFFFFFF;
        }
    }
    __syncwarp();
}

// Top-k expert indices of E <= 256 logits by a whole CTA (blockDim.x >= 256), through a
// filter instead of k rounds of warp-wide maxima.  Order: larger logit first, equal logits
// by lower index.  Thread t < E holds logit t (`mine`); every thread of the block calls this.
//  1. h_t = high word of t's order key (sign, exponent, 20 leading mantissa bits); the
//     32 groups of 8 consecutive logits each take their largest h;
//  2. tau = the k-th largest group maximum (groups ordered by maximum, then group number);
//  3. every logit with h_t >= tau is a candidate.  At least k groups hold a logit with
//     h >= tau, so the k best logits are all candidates -- typically a few more than k pass;
//  4. each candidate's rank = the number of candidates ordered before it (full 64-bit key,
//     then index); ranks below k land in idx_out.
// Shared scratch: s_gm[32] (16-byte aligned), *s_nc, s_cand[256].  Ends with a CTA barrier:
// idx_out (shared memory) is then visible to every thread.
__device__ __forceinline__ void block_topk_select(double mine, int E, int k, int32_t *idx_out, uint32_t *s_gm,
                                                  int *s_nc, ulonglong2 *s_cand) {
    const int tid = threadIdx.x, lane = tid & 31;
    const bool has = tid < E;
    const unsigned long long key = has ? f64_order_key(mine) : 0ull;
    const uint32_t h = (uint32_t)(key >> 32);
    uint32_t gm = h;
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 1));
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 2));
    gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 4));
    if (tid < 256 && (tid & 7) == 0) s_gm[tid >> 3] = gm;
    if (tid == 0) *s_nc = 0;
    __syncthreads();
    if (tid < 256) {
        // every warp finds tau itself: lane g ranks group g
        const uint32_t m = s_gm[lane];
        int above = 0;
#pragma unroll
        for (int q4 = 0; q4 < 8; q4++) {
            const uint4 v = reinterpret_cast<const uint4 *>(s_gm)[q4];
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int z = 0; z < 4; z++) above += (vv[z] > m || (vv[z] == m && 4 * q4 + z < lane)) ? 1 : 0;
        }
        const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
        const uint32_t tau = __shfl_sync(0xFFFFFFFFu, m, __ffs(who) - 1);
        // slot order is irrelevant: ranks come from comparisons, not positions
        if (has && h >= tau) s_cand[atomicAdd(s_nc, 1)] = make_ulonglong2(key, (unsigned long long)tid);
    }
    __syncthreads();
    const int nc = *s_nc;
    for (int i = tid; i < nc; i += blockDim.x) {
        const ulonglong2 me = s_cand[i];
        int r = 0;
        for (int q = 0; q < nc; q++) {
            const ulonglong2 o = s_cand[q];
            r += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
        }
        if (r < k) idx_out[r] = (int)me.y;
    }
    __syncthreads();
}

// One warp selects the top k (k <= 8) of E <= 256 fp64 logits held in shared memory `lg`:
// larger logit first, equal logits by lower index.  Lane l owns experts l, l+32, ..., l+224.
//  1. h = high word of each order key (sign, exponent, 20 leading mantissa bits); each lane
//     takes the largest h of its eight;
//  2. tau = the k-th largest lane maximum (lanes ordered by maximum, then lane number).  At
//     least k logits have h >= tau, and a logit with h < tau is below at least k others, so the
//     k best logits all have h >= tau;
//  3. the logits with h >= tau (typically a few more than k) are compacted into `cand`;
//  4. each candidate's rank = the number of candidates ordered before it (full 64-bit key, then
//     index); ranks below k land in idx_out.
// cand: shared scratch of 256 entries; s_m: 32 words of shared scratch, 16-byte aligned (both
// private to the calling warp, so several warps may run it at once); idx_out: shared memory;
// k <= 32.  No CTA barrier: only the calling warp takes part, and it ends with __syncwarp.
static __device__ __noinline__ void warp_topk_filter(const double *lg, int E, int k, int32_t *idx_out,
                                                     ulonglong2 *cand, uint32_t *s_m) {
    // Written for a short dependency chain: tau from the 32 lane maxima read back from shared
    // memory as broadcasts (eight 16-byte loads instead of 32 shuffles), the eight ballots issued
    // before their prefix sums, and the candidate ranking loading four candidates per step.
    const int lane = threadIdx.x & 31;
    unsigned long long key[8];
    uint32_t hi[8];
#pragma unroll
    for (int j = 0; j < 8; j++) {
        const int e = lane + 32 * j;
        key[j] = e < E ? f64_order_key(lg[e]) : 0ull;  // 0 = below every finite logit
        hi[j] = (uint32_t)(key[j] >> 32);
    }
    const uint32_t m = max(max(max(hi[0], hi[1]), max(hi[2], hi[3])), max(max(hi[4], hi[5]), max(hi[6], hi[7])));
    s_m[lane] = m;
    __syncwarp();
    int above4[4] = {0, 0, 0, 0};
#pragma unroll
    for (int q4 = 0; q4 < 8; q4++) {
        const uint4 v = reinterpret_cast<const uint4 *>(s_m)[q4];
        above4[0] += (v.x > m || (v.x == m && 4 * q4 + 0 < lane)) ? 1 : 0;
        above4[1] += (v.y > m || (v.y == m && 4 * q4 + 1 < lane)) ? 1 : 0;
        above4[2] += (v.z > m || (v.z == m && 4 * q4 + 2 < lane)) ? 1 : 0;
        above4[3] += (v.w > m || (v.w == m && 4 * q4 + 3 < lane)) ? 1 : 0;
    }
    const int above = (above4[0] + above4[1]) + (above4[2] + above4[3]);
    const unsigned who = __ballot_sync(0xFFFFFFFFu, above == k - 1);
    const uint32_t tau = s_m[__ffs(who) - 1];
    unsigned msk[8];
#pragma unroll
    for (int j = 0; j < 8; j++) msk[j] = __ballot_sync(0xFFFFFFFFu, lane + 32 * j < E && hi[j] >= tau);
    const unsigned below = (1u << lane) - 1u;
    int base = 0;
#pragma unroll
    for (int j = 0; j < 8; j++) {
        if ((msk[j] >> lane) & 1u) cand[base + __popc(msk[j] & below)] = make_ulonglong2(key[j], (unsigned long long)(lane + 32 * j));
        base += __popc(msk[j]);
    }
    const int nc = base;
    __syncwarp();
    for (int i = lane; i < nc; i += 32) {
        const ulonglong2 me = cand[i];
        int r4[4] = {0, 0, 0, 0};
        int q = 0;
        for (; q + 4 <= nc; q += 4) {
#pragma unroll
            for (int z = 0; z < 4; z++) {
                const ulonglong2 o = cand[q + z];
                r4[z] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
            }
        }
        for (; q < nc; q++) {
            const ulonglong2 o = cand[q];
            r4[0] += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
        }
        const int r = (r4[0] + r4[1]) + (r4[2] + r4[3]);
        if (r < k) idx_out[r] = (int)me.y;
    }
    __syncwarp();
}

// Renormalised gates of the selected experts: g_i = exp(l_i - l_0) / sum_j exp(l_j - l_0),
// lanes 0..k-1 each one exp in fp64, the sum taken in top-k order.
static __device__ __noinline__ void warp_topk_gates(const double *lg, int k, const int32_t *idx, double *g64, float *g32) {
    const int lane = threadIdx.x & 31;
    const double my_l = (lane < k) ? lg[idx[lane]] : 0.0;
    const double l0 = __shfl_sync(0xFFFFFFFFu, my_l, 0);
    const double ev = (lane < k) ? exp(my_l - l0) : 0.0;
    double z = 0.0;
    for (int r = 0; r < k; r++) z += __shfl_sync(0xFFFFFFFFu, ev, r);  // top-k order
    if (lane < k) {
        const double g = ev / z;
        if (g64) g64[lane] = g;
        if (g32) g32[lane] = (float)g;
    }
}

template <int J>
__device__ __forceinline__ void warp_topk(const double *lg, int E, int k, int32_t *idx_out, double *g64, float *g32) {
    warp_topk_select<J>(lg, E, k, idx_out);
    warp_topk_gates(lg, k, idx_out, g64, g32);
}

// ----------------------------------------------------------- absmax int8 quantisation
// q = clamp(rint(x * (127/absmax)), -127, 127) in fp32, ties to even; s = absmax/127
__device__ __forceinline__ float quant_inv(float absmax) { return __fdiv_rn(127.0f, absmax); }
__device__ __forceinline__ int quant_one(float x, float inv) {
    int q = __float2int_rn(__fmul_rn(x, inv));
    return q > 127 ? 127 : (q < -127 ? -127 : q);
}

// ----------------------------------------------------------------- SwiGLU epilogue
__device__ __forceinline__ float swiglu_f32(double g, double u) {
    return (float)(g / (1.0 + exp(-g)) * u);
}

// 4x4 byte transpose, into the position-major order of the table-free decode: P_j holds byte j
// of N0, N1, N2, N3 (in that byte order)
__device__ __forceinline__ void bytes_transpose4(uint32_t n0, uint32_t n1, uint32_t n2, uint32_t n3, uint32_t &p0,
                                                 uint32_t &p1, uint32_t &p2, uint32_t &p3) {
    const uint32_t t0 = __byte_perm(n0, n1, 0x5140u), t1 = __byte_perm(n2, n3, 0x5140u);
    const uint32_t t2 = __byte_perm(n0, n1, 0x7362u), t3 = __byte_perm(n2, n3, 0x7362u);
    p0 = __byte_perm(t0, t1, 0x5410u);
    p1 = __byte_perm(t0, t1, 0x7632u);
    p2 = __byte_perm(t2, t3, 0x5410u);
    p3 = __byte_perm(t2, t3, 0x7632u);
}

// Limb bytes of four consecutive values v[0..3] (elements 4t..4t+3 of a vector whose limbs go
// to `limbs`, laid out [NL][segments][kSegPad words], position-major inside each segment):
// element 4t+e lands in byte (t & 3) of word 4 * ((t >> 2) & 3) + e of segment t >> 4.
template <int NL>
__device__ __forceinline__ void store_limbs4(uint32_t *limbs, int seg_words_per_limb, int t, const float (&v)[4], int sh,
                                             float inv, bool nonzero) {
    uint8_t *lb = reinterpret_cast<uint8_t *>(limbs);
    const int g = t >> 4, q = (t >> 2) & 3, b = t & 3;
#pragma unroll
    for (int e = 0; e < 4; e++) {
        const int w = g * kSegPad + 4 * q + e;
        if (NL == 1) {
            lb[4 * w + b] = (uint8_t)((nonzero ? quant_one(v[e], inv) : 0) & 0xFF);
        } else {
            uint32_t hi, mid, lo;
            fixed_limbs(v[e], sh, hi, mid, lo);
            lb[4 * w + b] = (uint8_t)hi;
            lb[4 * (seg_words_per_limb + w) + b] = (uint8_t)mid;
            lb[4 * (2 * seg_words_per_limb + w) + b] = (uint8_t)lo;
        }
    }
}

// --------------------------------------------------------- bounded grid-wide barrier
// Monotonic arrival counter: barrier number n waits until the counter reaches n * nblocks.
// The counter is reset to zero by the last block to leave the kernel (see grid_exit), so it
// is zero at every launch.  Waits give up after `limit` SM cycles (clock64): the status word
// is set to TERN_ETIMEOUT and false is returned; the caller then leaves the kernel.  Stores a
// block made before the barrier are visible to every block after it: the block barrier orders
// them before thread 0's release add, and each block's thread 0 acquires before its block
// barrier releases the other threads.
struct GridSync {
    unsigned int *arrive;   // monotonic arrivals
    unsigned int *leave;    // blocks that finished
    int *status;            // device status word
    unsigned int nblocks;
    unsigned int epoch;     // barriers passed by this block
    long long limit;        // SM cycles
};

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_gpu_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// returns false on timeout (all threads of the block get the same answer); arrive = false (a
// test hook) waits without arriving, so this barrier and every block waiting at it time out
__device__ __forceinline__ bool grid_sync(GridSync &gs, int *flag_smem, bool arrive = true) {
    __syncthreads();
    if (threadIdx.x == 0) {
        gs.epoch++;
        const unsigned int target = gs.epoch * gs.nblocks;
        if (arrive) red_release_gpu_add(gs.arrive, 1u);
        const long long t0 = clock64();
        int ok = 1;
        while ((int)(ld_acquire_gpu(gs.arrive) - target) < 0) {
            if (clock64() - t0 > gs.limit) {
                ok = 0;
                set_status(gs.status, TERN_ETIMEOUT);
                break;
            }
        }
        *flag_smem = ok;
    }
    __syncthreads();
    const bool ok = *flag_smem != 0;
    __syncthreads();
    if (threadIdx.x != 0) gs.epoch++;
    return ok;
}

// last block out resets both counters so the next launch starts from zero
__device__ __forceinline__ void grid_exit(GridSync &gs) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned int n = atomicAdd(gs.leave, 1u);
        if (n == gs.nblocks - 1) {
            atomicExch(gs.arrive, 0u);
            atomicExch(gs.leave, 0u);
        }
    }
}

}  // namespace tern
