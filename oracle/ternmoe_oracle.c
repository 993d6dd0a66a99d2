/*
 * ternmoe_oracle.c -- plain, slow, obviously-correct CPU oracle for ternary-weight
 * MoE FFN decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and the
 * CPU-baseline leg of the benchmark may load this code.  It shares no code, header,
 * table or constant with the CUDA library; it is compiled by gcc with
 * -O2 -ffp-contract=off (no fused multiply-adds, no fast-math), single-threaded.  The
 * benchmark also times a second build of this same file with -fopenmp: the `omp` pragmas
 * below then split independent rows (router rows, gate/up rows, down rows) across the
 * host's cores.  Every value is still computed by one thread in the same order, so both
 * builds return identical results; the pragmas change the timing only.
 *
 * What it computes (sources are the five web pages on the Maple-Preview model):
 *  - ternary weights w in {-1,0,+1}, four 2-bit codes per byte ("How a 20B Model
 *    Hits 120 tok/s on an iPhone", "Why the number is plausible"; "A 20B AI Model
 *    Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini",
 *    "What Ternary Actually Means").  The pages do not disclose the code assignment
 *    ("iPhone Runs a 20B Model at 120 tok/s", "What a Credible Reproduction Report
 *    Should Disclose"); this oracle fixes 00 -> 0, 01 -> +1, 10 -> -1, code k%4 of a
 *    row in bits 2(k%4)..2(k%4)+1 of byte k/4 (little-endian along K).  Code 11 is
 *    never produced and decodes to 0 (reported).
 *  - a dot product with a ternary row needs no multiply: "negate, zero, or pass
 *    through" ("A 20B AI Model...", "What Ternary Actually Means").  The oracle takes
 *    that literally: sum of x over the +1 codes minus sum over the -1 codes, then
 *    one per-row fp32 scale.
 *  - a learned router picks 8 of 256 experts per token ("iPhone Runs a 20B Model",
 *    "MoE Is the Other Half of the Story Behind the 20B Figure"; "A 20B AI Model...",
 *    "The Architecture: Designed for the Hardware").  The pages do not say how the
 *    gate weights are normalised; the reading taken here: softmax over all experts,
 *    top-k by logit with ties to the lower index, gates renormalised over the
 *    selected k (the unselected experts cancel, so g_i = exp(l_i - l_max) / sum).
 *  - the expert body is not described on the pages; the reading taken here is a
 *    SwiGLU expert: h = silu(s_g * (G x)) * (s_u * (U x)), y_e = s_d * (D h), and
 *    the layer output is sum_i g_i y_{e_i} in top-k order.
 *  - a decode step streams the active weights layer after layer ("How a 20B
 *    Model...", "Why the number is plausible"); the 24-layer stack applies
 *    x' = bf16(x + bf16(FFN(bf16(RMSNorm(x))))) with RMSNorm(x) = x / sqrt(mean x^2 + eps)
 *    and no learned gain.
 *
 * Precision: integer work is exact (int64, checked to fit int32 where the method
 * keeps int32).  Floating-point sums of bf16 / fp32 terms are computed twice: in fp64
 * in index order and exactly as an __int128 fixed-point sum; the returned value is
 * the exact sum rounded once to fp64, and every function returns how many sums the
 * plain fp64 loop did NOT reproduce exactly (expected: 0).  The int8 path follows
 * fp32 operations one by one where floating point decides an integer (absmax
 * quantisation), so both sides take that decision in the same precision.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERANGE 1

/* ------------------------------------------------------------------ bf16 */

static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* nearest bf16 (ties to even) of a finite double */
static uint16_t f64_to_bf16(double v) {
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e = ilogb(a);
    if (e < -126) e = -126;
    int step = e - 7;                     /* bf16 keeps 8 significant bits */
    double q = nearbyint(ldexp(a, -step)); /* default mode: ties to even */
    double r = ldexp(q, step);
    if (r >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    float rf = (float)r; /* exact: at most 9 significant bits */
    uint32_t u;
    memcpy(&u, &rf, 4);
    return (uint16_t)(sign | (u >> 16));
}

uint16_t or_f64_to_bf16(double v) { return f64_to_bf16(v); }
double or_bf16_to_f64(uint16_t b) { return bf16_to_f64(b); }

/* ------------------------------------------------- exact fixed-point sums */

typedef struct {
    __int128 acc;
    int ok;
} xsum;

#define XQ 96 /* resolution 2^-96; magnitudes below 2^30 */

static void xs_init(xsum *s) {
    s->acc = 0;
    s->ok = 1;
}

static void xs_add(xsum *s, double v) {
    double t = ldexp(v, XQ);
    if (!(fabs(t) < 0x1p124) || t != trunc(t)) {
        s->ok = 0;
        return;
    }
    s->acc += (__int128)t;
}

/* exact sum rounded once to double */
static double xs_value(const xsum *s) { return ldexp((double)s->acc, -XQ); }

/* ------------------------------------------------------------- the format */

static int code_to_weight(unsigned c) {
    switch (c) {
    case 0: return 0;
    case 1: return 1;
    case 2: return -1;
    default: return 0; /* 11: never produced */
    }
}

/* Pack int8 weights [M,K] into bytes [M,K/4].  Returns the number of entries not
 * in {-1,0,+1} (those are packed as code 00). */
int64_t or_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *out) {
    int64_t bad = 0;
    for (int64_t m = 0; m < M; m++) {
        for (int64_t b = 0; b < K / 4; b++) {
            unsigned byte = 0;
            for (int j = 0; j < 4; j++) {
                int v = w[m * K + 4 * b + j];
                unsigned code;
                if (v == 0) code = 0;
                else if (v == 1) code = 1;
                else if (v == -1) code = 2;
                else {
                    code = 0;
                    bad++;
                }
                byte |= code << (2 * j);
            }
            out[m * (K / 4) + b] = (uint8_t)byte;
        }
    }
    return bad;
}

/* Unpack bytes [M,K/4] into int8 weights [M,K].  Returns the number of 11 codes. */
int64_t or_unpack(const uint8_t *p, int64_t M, int64_t K, int8_t *w) {
    int64_t bad = 0;
    for (int64_t m = 0; m < M; m++)
        for (int64_t k = 0; k < K; k++) {
            unsigned c = (p[m * (K / 4) + k / 4] >> (2 * (k % 4))) & 3u;
            if (c == 3) bad++;
            w[m * K + k] = (int8_t)code_to_weight(c);
        }
    return bad;
}

/* ------------------------------------------------ base-3 packing: five weights per byte
 * The pages give the information content of a ternary weight, log2(3) ~ 1.585 bits ("How a
 * 20B Model Hits 120 tok/s on an iPhone", "Why the number is plausible"; "A 20B AI Model
 * Trained in Ternary...", "What Ternary Actually Means").  3^5 = 243 <= 256, so five weights
 * fit one byte: 1.6 bits per weight.  Reading taken here: weight w[5b+i] contributes the digit
 * t_i in {0,1,2} -- the same code as the 2-bit format (0 -> 0, 1 -> +1, 2 -> -1) -- and byte b
 * of a row holds t_0 + 3 t_1 + 9 t_2 + 27 t_3 + 81 t_4 (little-endian along K).  Positions past
 * K hold digit 0; each row is padded with zero bytes to a multiple of 16 bytes.  Bytes 243..255
 * are never produced and decode to five zeros (reported). */
int64_t or_tern5_row_bytes(int64_t K) {
    const int64_t b = (K + 4) / 5;
    return (b + 15) / 16 * 16;
}

int64_t or_pack5(const int8_t *w, int64_t M, int64_t K, uint8_t *out) {
    const int64_t rb = or_tern5_row_bytes(K);
    int64_t bad = 0;
    for (int64_t m = 0; m < M; m++)
        for (int64_t b = 0; b < rb; b++) {
            unsigned value = 0, place = 1;
            for (int i = 0; i < 5; i++) {
                const int64_t k = 5 * b + i;
                unsigned digit = 0;
                if (k < K) {
                    const int v = w[m * K + k];
                    if (v == 1) digit = 1;
                    else if (v == -1) digit = 2;
                    else if (v != 0) bad++;
                }
                value += digit * place;
                place *= 3;
            }
            out[m * rb + b] = (uint8_t)value;
        }
    return bad;
}

/* Returns the number of bytes >= 243 among the bytes that hold weights of [0, K). */
int64_t or_unpack5(const uint8_t *p, int64_t M, int64_t K, int8_t *w) {
    const int64_t rb = or_tern5_row_bytes(K);
    int64_t bad = 0;
    for (int64_t m = 0; m < M; m++)
        for (int64_t b = 0; b * 5 < K; b++) {
            unsigned value = p[m * rb + b];
            if (value >= 243) {
                bad++;
                value = 0;
            }
            for (int i = 0; i < 5; i++) {
                const int64_t k = 5 * b + i;
                if (k < K) w[m * K + k] = (int8_t)code_to_weight(value % 3);
                value /= 3;
            }
        }
    return bad;
}

static int weight_at(const uint8_t *row, int64_t k) {
    return code_to_weight((row[k / 4] >> (2 * (k % 4))) & 3u);
}

/* ------------------------------------------------------ ternary dot products */

/* sum over +1 codes minus sum over -1 codes of integer activations */
static int64_t tern_dot_i64(const uint8_t *row, const int8_t *q, int64_t K) {
    int64_t plus = 0, minus = 0;
    for (int64_t k = 0; k < K; k++) {
        int w = weight_at(row, k);
        if (w == 1) plus += q[k];
        else if (w == -1) minus += q[k];
    }
    return plus - minus;
}

/* same with real activations; exact sum, rounded once.  *inexact += 1 when the
 * plain fp64 loop differs from the exact value; *unchecked += 1 when a term did not
 * fit the fixed-point grid (then the plain fp64 value is returned). */
static double tern_dot_f64(const uint8_t *row, const double *x, int64_t K, int64_t *inexact,
                           int64_t *unchecked) {
    double plus = 0.0, minus = 0.0;
    xsum ex;
    xs_init(&ex);
    for (int64_t k = 0; k < K; k++) {
        int w = weight_at(row, k);
        if (w == 1) {
            plus += x[k];
            xs_add(&ex, x[k]);
        } else if (w == -1) {
            minus += x[k];
            xs_add(&ex, -x[k]);
        }
    }
    double plain = plus - minus;
    if (!ex.ok) {
        (*unchecked)++;
        return plain;
    }
    double exact = xs_value(&ex);
    if (exact != plain) (*inexact)++;
    return exact;
}

/* ----------------------------------------------------------- ternary GEMV */

/* int8 activations: acc[t,m] = sum_k w[m,k] q[t,k] (int32), y = (fp32)acc * s[m]
 * (one fp32 rounding), then * x_scale[t] when x_scale is given.
 * Returns OR_ERANGE if an accumulator does not fit int32. */
int or_gemv_i8(const uint8_t *Wp, const float *s, int64_t M, int64_t K, int64_t T, const int8_t *q,
               const float *x_scale, int32_t *acc, float *y) {
    int rc = OR_OK;
    for (int64_t t = 0; t < T; t++)
        for (int64_t m = 0; m < M; m++) {
            int64_t a = tern_dot_i64(Wp + m * (K / 4), q + t * K, K);
            if (a > INT32_MAX || a < INT32_MIN) rc = OR_ERANGE;
            if (acc) acc[t * M + m] = (int32_t)a;
            volatile float v = (float)(int32_t)a;
            v = v * s[m];
            if (x_scale) v = v * x_scale[t];
            if (y) y[t * M + m] = v;
        }
    return rc;
}

/* bf16 activations: y[t,m] = s[m] * (sum_{+1} x - sum_{-1} x), in fp64 with the sum
 * exact.  Returns the number of sums the plain fp64 loop did not reproduce. */
int64_t or_gemv_bf16(const uint8_t *Wp, const float *s, int64_t M, int64_t K, int64_t T,
                     const uint16_t *x, double *y) {
    int64_t inexact = 0, unchecked = 0;
    double *xf = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t t = 0; t < T; t++) {
        for (int64_t k = 0; k < K; k++) xf[k] = bf16_to_f64(x[t * K + k]);
        for (int64_t m = 0; m < M; m++)
            y[t * M + m] = tern_dot_f64(Wp + m * (K / 4), xf, K, &inexact, &unchecked) * (double)s[m];
    }
    free(xf);
    return inexact + unchecked;
}

/* ------------------------------------------------ absmax int8 quantisation */

/* Symmetric per-vector absmax quantisation in fp32 (pages silent; the reading
 * taken: s = absmax/127, q = clamp(rint(x * (127/absmax)), -127, 127), ties to
 * even; an all-zero vector gives q = 0, s = 0). */
void or_quant_absmax(const float *x, int64_t n, int8_t *q, float *s) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        for (int64_t i = 0; i < n; i++) q[i] = 0;
        *s = 0.0f;
        return;
    }
    volatile float inv = 127.0f / amax;
    for (int64_t i = 0; i < n; i++) {
        volatile float p = x[i] * inv;
        float r = rintf(p);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[i] = (int8_t)r;
    }
    volatile float sc = amax / 127.0f;
    *s = sc;
}

/* ---------------------------------------------------------------- RMSNorm */

/* n = bf16( x / sqrt(mean(x^2) + eps) ), every step in fp64; mean(x^2) from an exact
 * sum of squares.  Returns 1 if the plain fp64 sum of squares was not exact. */
int64_t or_rmsnorm(const uint16_t *x, int64_t d, double eps, uint16_t *n) {
    double plain = 0.0;
    xsum ex;
    xs_init(&ex);
    for (int64_t k = 0; k < d; k++) {
        double v = bf16_to_f64(x[k]);
        plain += v * v;
        xs_add(&ex, v * v);
    }
    int64_t bad = 0;
    double ss = plain;
    if (ex.ok) {
        ss = xs_value(&ex);
        if (ss != plain) bad = 1;
    } else bad = 1;
    double r = sqrt(ss / (double)d + eps);
    for (int64_t k = 0; k < d; k++) n[k] = f64_to_bf16(bf16_to_f64(x[k]) / r);
    return bad;
}

/* ------------------------------------------------------------------ router */

/* logits[t,e] = sum_k Wg[e,k] x[t,k] (exact, rounded once to fp64); top-k by logit
 * descending with ties to the lower expert index; gates renormalised over the
 * selected experts: g_i = exp(l_i - l_0) / sum_j exp(l_j - l_0) summed in top-k
 * order.  Returns the number of logits the plain fp64 loop did not reproduce. */
int64_t or_route(const uint16_t *Wg, const uint16_t *x, int64_t T, int64_t d, int32_t E, int32_t k,
                 double *logits, int32_t *idx, double *gates) {
    int64_t bad = 0;
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    char *taken = (char *)malloc((size_t)E);
    for (int64_t t = 0; t < T; t++) {
#pragma omp parallel for reduction(+ : bad) schedule(static)
        for (int32_t e = 0; e < E; e++) {
            double plain = 0.0;
            xsum ex;
            xs_init(&ex);
            for (int64_t c = 0; c < d; c++) {
                double p = bf16_to_f64(Wg[(int64_t)e * d + c]) * bf16_to_f64(x[t * d + c]); /* exact */
                plain += p;
                xs_add(&ex, p);
            }
            double v = plain;
            if (ex.ok) {
                v = xs_value(&ex);
                if (v != plain) bad++;
            } else bad++;
            l[e] = v;
            if (logits) logits[t * E + e] = v;
        }
        memset(taken, 0, (size_t)E);
        for (int32_t i = 0; i < k; i++) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep lower index */
            }
            taken[best] = 1;
            idx[t * k + i] = best;
        }
        double l0 = l[idx[t * k]];
        double z = 0.0;
        double *ev = (double *)malloc(sizeof(double) * (size_t)k);
        for (int32_t i = 0; i < k; i++) {
            ev[i] = exp(l[idx[t * k + i]] - l0);
            z += ev[i];
        }
        for (int32_t i = 0; i < k; i++) gates[t * k + i] = ev[i] / z;
        free(ev);
    }
    free(l);
    free(taken);
    return bad;
}

/* ------------------------------------------------------------- MoE FFN layer */

typedef struct {
    const uint8_t *gate;       /* [E][f][d/4] */
    const uint8_t *up;         /* [E][f][d/4] */
    const uint8_t *down;       /* [E][d][f/4] */
    const float *gate_scale;   /* [E][f] */
    const float *up_scale;     /* [E][f] */
    const float *down_scale;   /* [E][d] */
    const uint16_t *router;    /* [E][d] bf16 */
    int64_t d, f;
    int32_t E, k;
} or_layer;

/* Optional intermediate outputs (any pointer may be NULL). */
typedef struct {
    int32_t *idx;     /* [T][k] */
    double *gates;    /* [T][k] */
    double *logits;   /* [T][E] */
    float *h;         /* [T][k][f] SwiGLU output rounded to fp32 */
    int32_t *acc_g;   /* [T][k][f] int8 path only */
    int32_t *acc_u;   /* [T][k][f] */
    int8_t *qx;       /* [T][d] */
    float *sx;        /* [T] */
    int8_t *qh;       /* [T][k][f] */
    float *sh;        /* [T][k] */
    int32_t *acc_d;   /* [T][k][d] */
    double *ye;       /* [T][k][d] per-expert down output, before the gate */
} or_trace;

#define OR_ACT_BF16 0
#define OR_ACT_INT8 1

static double silu_times(double g, double u) { return g / (1.0 + exp(-g)) * u; }

/* One MoE FFN layer for T tokens.
 *   act = OR_ACT_BF16: x and h enter the ternary dots as real numbers (exact sums);
 *   act = OR_ACT_INT8: x is absmax-quantised per token, h per (token, expert); the
 *     dots are int32; g = ((fp32)acc_g * s_g) * s_x in fp32, likewise u; h is the
 *     fp64 SwiGLU of those fp32 values rounded to fp32; y_e = ((fp32)acc_d * s_d) * s_h.
 * Both paths: y = sum_i gates_i * y_e_i in fp64 in top-k order; y_bf16 = nearest-even
 * bf16 of y; y64 = y.
 * Teacher forcing: if qh_in/sh_in (int8) or h_in (bf16) are given, the down stage
 * consumes them instead of this oracle's own values.
 * Returns the number of inexact plain-fp64 sums (expected 0) + 1e6 * int32 overflows. */
int64_t or_moe_ffn(const or_layer *L, const uint16_t *x, int64_t T, int act, uint16_t *y_bf16,
                   double *y64, or_trace *tr, const int8_t *qh_in, const float *sh_in,
                   const float *h_in) {
    const int64_t d = L->d, f = L->f;
    const int32_t E = L->E, k = L->k;
    int64_t bad = 0, unchecked = 0;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * k));
    double *gates = (double *)malloc(sizeof(double) * (size_t)(T * k));
    double *logits = (double *)malloc(sizeof(double) * (size_t)(T * E));
    bad += or_route(L->router, x, T, d, E, k, logits, idx, gates);
    double *xf = (double *)malloc(sizeof(double) * (size_t)d);
    float *x32 = (float *)malloc(sizeof(float) * (size_t)d);
    int8_t *qx = (int8_t *)malloc((size_t)d);
    float *h = (float *)malloc(sizeof(float) * (size_t)f);
    double *hd = (double *)malloc(sizeof(double) * (size_t)f);
    int8_t *qh = (int8_t *)malloc((size_t)f);
    double *y = (double *)malloc(sizeof(double) * (size_t)d);

    for (int64_t t = 0; t < T; t++) {
        float sx = 0.0f;
        for (int64_t c = 0; c < d; c++) {
            xf[c] = bf16_to_f64(x[t * d + c]);
            x32[c] = (float)xf[c];
        }
        if (act == OR_ACT_INT8) {
            or_quant_absmax(x32, d, qx, &sx);
            if (tr && tr->qx) memcpy(tr->qx + t * d, qx, (size_t)d);
            if (tr && tr->sx) tr->sx[t] = sx;
        }
        for (int64_t c = 0; c < d; c++) y[c] = 0.0;
        for (int32_t i = 0; i < k; i++) {
            const int32_t e = idx[t * k + i];
            const int64_t slot = t * k + i;
            /* gate / up rows, SwiGLU */
#pragma omp parallel for reduction(+ : bad, unchecked) schedule(static)
            for (int64_t j = 0; j < f; j++) {
                const uint8_t *grow = L->gate + ((int64_t)e * f + j) * (d / 4);
                const uint8_t *urow = L->up + ((int64_t)e * f + j) * (d / 4);
                float sg = L->gate_scale[(int64_t)e * f + j];
                float su = L->up_scale[(int64_t)e * f + j];
                if (act == OR_ACT_INT8) {
                    int64_t ag = tern_dot_i64(grow, qx, d);
                    int64_t au = tern_dot_i64(urow, qx, d);
                    if (ag > INT32_MAX || ag < INT32_MIN || au > INT32_MAX || au < INT32_MIN) bad += 1000000;
                    if (tr && tr->acc_g) tr->acc_g[slot * f + j] = (int32_t)ag;
                    if (tr && tr->acc_u) tr->acc_u[slot * f + j] = (int32_t)au;
                    volatile float g = (float)(int32_t)ag;
                    g = g * sg;
                    g = g * sx;
                    volatile float u = (float)(int32_t)au;
                    u = u * su;
                    u = u * sx;
                    h[j] = (float)silu_times((double)g, (double)u);
                } else {
                    double g = tern_dot_f64(grow, xf, d, &bad, &unchecked) * (double)sg;
                    double u = tern_dot_f64(urow, xf, d, &bad, &unchecked) * (double)su;
                    h[j] = (float)silu_times(g, u);
                }
            }
            if (tr && tr->h) memcpy(tr->h + slot * f, h, sizeof(float) * (size_t)f);
            /* down rows */
            float sh = 0.0f;
            if (act == OR_ACT_INT8) {
                or_quant_absmax(h, f, qh, &sh);
                if (tr && tr->qh) memcpy(tr->qh + slot * f, qh, (size_t)f);
                if (tr && tr->sh) tr->sh[slot] = sh;
                if (qh_in) {
                    memcpy(qh, qh_in + slot * f, (size_t)f);
                    sh = sh_in[slot];
                }
            } else {
                const float *hs = h_in ? h_in + slot * f : h;
                for (int64_t j = 0; j < f; j++) hd[j] = (double)hs[j];
            }
#pragma omp parallel for reduction(+ : bad, unchecked) schedule(static)
            for (int64_t c = 0; c < d; c++) {
                const uint8_t *drow = L->down + ((int64_t)e * d + c) * (f / 4);
                float sd = L->down_scale[(int64_t)e * d + c];
                double ye;
                if (act == OR_ACT_INT8) {
                    int64_t ad = tern_dot_i64(drow, qh, f);
                    if (ad > INT32_MAX || ad < INT32_MIN) bad += 1000000;
                    if (tr && tr->acc_d) tr->acc_d[slot * d + c] = (int32_t)ad;
                    volatile float v = (float)(int32_t)ad;
                    v = v * sd;
                    v = v * sh;
                    ye = (double)v;
                } else {
                    ye = tern_dot_f64(drow, hd, f, &bad, &unchecked) * (double)sd;
                }
                if (tr && tr->ye) tr->ye[slot * d + c] = ye;
                y[c] += gates[t * k + i] * ye;
            }
        }
        for (int64_t c = 0; c < d; c++) {
            if (y_bf16) y_bf16[t * d + c] = f64_to_bf16(y[c]);
            if (y64) y64[t * d + c] = y[c];
        }
    }
    if (tr && tr->idx) memcpy(tr->idx, idx, sizeof(int32_t) * (size_t)(T * k));
    if (tr && tr->gates) memcpy(tr->gates, gates, sizeof(double) * (size_t)(T * k));
    if (tr && tr->logits) memcpy(tr->logits, logits, sizeof(double) * (size_t)(T * E));
    free(idx); free(gates); free(logits); free(xf); free(x32); free(qx);
    free(h); free(hd); free(qh); free(y);
    return bad + unchecked;
}

/* One layer of the residual stack: n = RMSNorm(x) in bf16, y = FFN(n) in bf16,
 * x_out = bf16(x + y).  n_out / y_out (bf16) and y64 are optional. */
int64_t or_stack_layer(const or_layer *L, const uint16_t *x, int64_t T, double eps, int act,
                       uint16_t *x_out, uint16_t *n_out, uint16_t *y_out, double *y64,
                       or_trace *tr) {
    const int64_t d = L->d;
    int64_t bad = 0;
    uint16_t *n = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(T * d));
    uint16_t *y = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(T * d));
    for (int64_t t = 0; t < T; t++) bad += or_rmsnorm(x + t * d, d, eps, n + t * d);
    bad += or_moe_ffn(L, n, T, act, y, y64, tr, NULL, NULL, NULL);
    for (int64_t i = 0; i < T * d; i++) x_out[i] = f64_to_bf16(bf16_to_f64(x[i]) + bf16_to_f64(y[i]));
    if (n_out) memcpy(n_out, n, sizeof(uint16_t) * (size_t)(T * d));
    if (y_out) memcpy(y_out, y, sizeof(uint16_t) * (size_t)(T * d));
    free(n);
    free(y);
    return bad;
}
