/*
 * ternmoe.h -- C ABI of libternmoe.so: ternary-weight mixture-of-experts FFN decode on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (from the web pages on the Maple-Preview model):
 *   - weights are ternary, every weight -1, 0 or +1 ("How a 20B Model Hits 120 tok/s on an
 *     iPhone", lead and "Why the number is plausible"), packed four 2-bit codes per byte
 *     and used without unpacking ("A 20B AI Model Trained in Ternary Just Hit 218
 *     Tokens/Second on a $599 Mac Mini", "What Ternary Actually Means" and "The
 *     Architecture: Designed for the Hardware"), so a dot product is adds and subtracts of
 *     activations followed by one per-row scale;
 *   - batch-1 decode is a sequence of matrix-vector products bound by memory bandwidth
 *     (same page, "What Ternary Actually Means");
 *   - a learned router picks 8 of 256 experts per token ("iPhone Runs a 20B Model at 120
 *     tok/s", "MoE Is the Other Half of the Story Behind the 20B Figure"; "A 20B AI Model...",
 *     "The Architecture: Designed for the Hardware"), 24 layers deep.
 *
 * Packed format (the pages leave the encoding undisclosed -- "iPhone Runs a 20B Model...",
 * "What a Credible Reproduction Report Should Disclose"; this library fixes it):
 *   code 00 -> 0, 01 -> +1, 10 -> -1 (11 is never written and reads as 0);
 *   weight k of row m is in bits 2(k%4)..2(k%4)+1 of byte m*(K/4) + k/4;
 *   one fp32 scale per output row.
 *
 * Conventions for every call below
 *   - All array pointers are DEVICE pointers owned by the caller; the library never frees
 *     them.  bf16 values travel as uint16_t bit patterns.  Row-major layouts.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls
 *     enqueue work and return without waiting, except tern_pack / tern_unpack and
 *     tern5_pack / tern5_unpack (they wait for their own kernel to report invalid codes) and
 *     tern_stream_status.
 *   - Arguments are checked on the host before anything is enqueued; a failed check returns
 *     TERN_EINVAL / TERN_EALIGN / TERN_EWORKSPACE and enqueues nothing.  A CUDA launch
 *     error returns TERN_ECUDA.  No C++ exception crosses the ABI.
 *   - K (the reduction length of a ternary matrix) must be a multiple of 64 so packed rows
 *     are whole 16-byte vectors; K <= 2048, or a multiple of 2048 up to 16384 (the base-3
 *     calls take any K up to 16384: their rows are padded to 16 bytes).  Packed
 *     arrays and activations must be 16-byte aligned, scales 4-byte aligned.
 *   - The library allocates no device memory on these paths: scratch space is the
 *     caller's `workspace`.  A workspace must be zero-filled once before its first use
 *     (cudaMemset); every successful call leaves its control words zero again.  Calls that
 *     share a workspace must not overlap on the GPU.
 */
#ifndef TERNMOE_H
#define TERNMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TERNMOE_ABI_VERSION 3

typedef enum {
    TERN_OK = 0,
    TERN_EINVAL = 1,      /* bad shape, null pointer, k > E, unsupported size */
    TERN_EALIGN = 2,      /* pointer not aligned as required */
    TERN_ECODE = 3,       /* pack: weight outside {-1,0,1}; unpack: code 11 present */
    TERN_ECUDA = 4,       /* a CUDA runtime call or launch failed */
    TERN_ETIMEOUT = 5,    /* a bounded in-kernel wait gave up (device status word) */
    TERN_EWORKSPACE = 6,  /* workspace null or smaller than the query says */
    TERN_EUNSUPPORTED = 7 /* valid request this build does not implement */
} tern_status;

typedef enum {
    TERN_ACT_BF16 = 0, /* bf16 activations; exact integer dot on a 24-bit fixed-point grid */
    TERN_ACT_INT8 = 1  /* int8 activations (per-vector absmax quantisation), int32 accumulate */
} tern_act;

/* One MoE FFN layer (device pointers). E experts, each a SwiGLU expert with ternary gate and
 * up matrices [f][d] and a ternary down matrix [d][f]; router W_g [E][d] in bf16.
 * The pages do not describe the expert body; this library takes the SwiGLU reading. */
typedef struct {
    const uint8_t *gate;       /* [E][f][d/4] packed */
    const uint8_t *up;         /* [E][f][d/4] packed */
    const uint8_t *down;       /* [E][d][f/4] packed */
    const float *gate_scale;   /* [E][f] */
    const float *up_scale;     /* [E][f] */
    const float *down_scale;   /* [E][d] */
    const uint16_t *router;    /* [E][d] bf16 */
    int64_t d, f;              /* hidden and expert width; multiples of 64 */
    int32_t E, k;              /* experts, experts per token: 1 <= k <= 8, k <= E <= 1024 */
} tern_moe_layer;

/* Byte offsets, inside the workspace of moe_ffn_decode, of the intermediates the last call
 * left there (for inspection and parity checks; -1 = not produced on this path). */
typedef struct {
    int64_t logits;   /* double [T][E] router logits */
    int64_t idx;      /* int32 [T][k] selected experts, descending logit, ties -> lower index */
    int64_t gates64;  /* double [T][k] renormalised gates */
    int64_t gates32;  /* float [T][k] the same rounded to fp32 */
    int64_t h;        /* float [T][k][f] SwiGLU output of each (token, slot) */
    int64_t qx;       /* int8 [T][d] quantised layer input (int8 path) */
    int64_t sx;       /* float [T] its scale (int8 path) */
    int64_t qh;       /* int8 [T][k][f] quantised h (int8 path) */
    int64_t sh;       /* float [T][k] its scale (int8 path) */
    int64_t acc_g;    /* int32 [T][k][f] gate accumulators (int8 path) */
    int64_t acc_u;    /* int32 [T][k][f] up accumulators (int8 path) */
    int64_t acc_d;    /* int32 [T][k][d] down accumulators (int8 path) */
    int64_t ye;       /* double [T][k][d] expert outputs before the gate */
    int64_t n_unique; /* int32: number of distinct experts selected by the step */
    int64_t total;    /* bytes needed */
} tern_ffn_layout;

/* Human-readable name of a status code (static string). */
const char *tern_status_str(tern_status s);

/* TERNMOE_ABI_VERSION of the loaded library. */
int32_t tern_abi_version(void);

/* Pack int8 weights w [M][K] (values -1, 0, +1) into packed [M][K/4].
 * Waits for its kernel; returns TERN_ECODE if any weight is outside {-1,0,1} (that weight
 * is written as code 00).  K % 4 == 0. */
tern_status tern_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, void *stream);

/* Unpack packed [M][K/4] into int8 w [M][K].  Waits; returns TERN_ECODE if a code 11 was
 * found (written as 0).  K % 4 == 0. */
tern_status tern_unpack(const uint8_t *packed, int64_t M, int64_t K, int8_t *w, void *stream);

/* Ternary GEMV for T tokens:  S[t,m] = sum_k w[m,k] x[t,k]  (adds/subtracts only), then
 *   act = TERN_ACT_INT8: x is int8 [T][K]; acc[t,m] = S (int32, exact; acc may be NULL);
 *        y[t,m] = ((float)S * row_scale[m]) * x_scale[t]   (x_scale may be NULL: no factor);
 *   act = TERN_ACT_BF16: x is bf16 [T][K]; y[t,m] = row_scale[m] * S, where S is summed
 *        exactly on a 24-bit fixed-point grid per token (every bf16 within 2^15 of the
 *        token's absmax is exact; smaller ones round to the grid), scaled in fp64 and
 *        rounded to fp32; acc must be NULL.
 * Wp [M][K/4], row_scale [M], y [T][M].  1 <= T <= 64. */
tern_status tern_gemv(const uint8_t *Wp, const float *row_scale, int64_t M, int64_t K, tern_act act,
                      const void *x, const float *x_scale, int64_t T, int32_t *acc, float *y,
                      void *stream);

/* Base-3 packed format: five ternary weights per byte, 1.6 bits per weight (a ternary weight
 * carries log2(3) ~ 1.585 bits: "How a 20B Model Hits 120 tok/s on an iPhone", "Why the
 * number is plausible").  Byte b of a row holds t0 + 3 t1 + 9 t2 + 27 t3 + 81 t4, where t_i is
 * the 2-bit code of weight 5b+i (0 -> 0, 1 -> +1, 2 -> -1); positions past K and the row's
 * padding bytes are 0.  A row takes tern5_row_bytes(K) bytes: ceil(K/5) rounded up to a
 * multiple of 16 (416 bytes for K = 2048, against 512 for four codes per byte).
 * Returns 0 for K < 1. */
int64_t tern5_row_bytes(int64_t K);

/* Pack int8 w [M][K] (values in {-1,0,1}) into packed [M][tern5_row_bytes(K)].  Waits for its
 * kernel; returns TERN_ECODE if any weight is outside {-1,0,1} (packed as 0).  Any K >= 1. */
tern_status tern5_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, void *stream);

/* Unpack into int8 w [M][K].  Waits; returns TERN_ECODE if a byte holding weights is >= 243
 * (its five weights are written as 0). */
tern_status tern5_unpack(const uint8_t *packed, int64_t M, int64_t K, int8_t *w, void *stream);

/* The ternary GEMV of tern_gemv on base-3 packed rows W5 [M][tern5_row_bytes(K)]: same
 * arguments, same arithmetic and results (exact integer sums).  1 <= K <= 16384; W5 16-byte
 * aligned, x 2-byte aligned. */
tern_status tern5_gemv(const uint8_t *W5, const float *row_scale, int64_t M, int64_t K, tern_act act,
                       const void *x, const float *x_scale, int64_t T, int32_t *acc, float *y,
                       void *stream);

/* Per-vector absmax int8 quantisation of bf16 rows x [T][n]:  s[t] = absmax/127,
 * q = clamp(rint(x * (127/absmax)), -127, 127) in fp32, ties to even; a zero row gives
 * q = 0, s = 0.  (The pages are silent on activation precision; this is the int8 reading.) */
tern_status tern_quant_absmax(const uint16_t *x, int64_t T, int64_t n, int8_t *q, float *s,
                              void *stream);

/* Router: logits[t,e] = sum_k Wg[e,k] x[t,k] accumulated in fp64; each bf16 x bf16 product
 * is exact in fp64 and added with one rounding (fused multiply-add); top-k by
 * logit descending, ties to the lower expert index; gates renormalised
 * over the selected experts, g_i = exp(l_i - l_max) / sum_j exp(l_j - l_max), in fp64 and
 * written as fp32.  Wg [E][d] bf16, x [T][d] bf16, topk_idx [T][k], topk_gate [T][k],
 * logits [T][E] (may be NULL).  1 <= T <= 64, 1 <= k <= 8, k <= E <= 1024, d % 8 == 0. */
size_t moe_route_workspace_bytes(int64_t T, int32_t E);
tern_status moe_route_topk(const uint16_t *Wg, const uint16_t *x, int64_t T, int64_t d, int32_t E,
                           int32_t k, int32_t *topk_idx, float *topk_gate, double *logits,
                           void *workspace, size_t ws_bytes, void *stream);

/* moe_route_topk_static -- the same routing as moe_route_topk, for callers that cannot
 * allocate device memory (the pages have no counterpart; this is a library convenience).
 * A caller that only receives device pointers to its inputs and outputs -- a plugin whose
 * host framework owns every allocation, or a serving loop that forbids allocator calls after
 * start-up -- has no way to provide a workspace.  This call needs none: its scratch (arrival
 * counter, fp64 logits, fp64 gates; 135,424 bytes) is a fixed array inside the library,
 * held on every GPU that loads the library until the process exits.  Inputs and outputs are
 * the caller's, exactly as for moe_route_topk.
 *   Limits: 1 <= T <= 64 and T * E <= 16384 (e.g. 64 tokens x 256 experts); larger requests
 *   return TERN_EINVAL before anything is enqueued.
 *   Each call outside stream capture looks up the array's device address on the calling
 *   thread's current device (so a context rebuilt by cudaDeviceReset is handled); a call made
 *   while `stream` is capturing reuses the address of the last non-capturing call on that
 *   device, so make the first call on each device before any stream capture.
 *   All calls on a device share the one array: calls that overlap on the GPU (different
 *   streams, no ordering between them) race and give undefined results.  The call clears
 *   the part that must start at zero (the arrival counter) itself.
 *   It allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine. */
tern_status moe_route_topk_static(const uint16_t *Wg, const uint16_t *x, int64_t T, int64_t d, int32_t E,
                                  int32_t k, int32_t *topk_idx, float *topk_gate, double *logits,
                                  void *stream);

/* One MoE FFN layer for T tokens (decode):
 *   route (as moe_route_topk) -> group the (token, slot) pairs by expert so every selected
 *   expert's packed weights stream from memory once per call -> for each pair
 *   h = silu(s_g * (G x)) * (s_u * (U x)) -> y_e = s_d * (D h) -> y[t] = sum over the k
 *   slots in top-k order of gate * fp32(y_e) (each expert output rounded once to fp32, the
 *   precision in which the persistent kernel passes it between SMs), accumulated in fp64,
 *   written as bf16 (nearest even) and, if
 *   y_f32 != NULL, as fp32.
 *   act = TERN_ACT_BF16: x and h enter the dots on a 24-bit fixed-point grid (see tern_gemv).
 *   act = TERN_ACT_INT8: x is absmax-quantised per token and h per (token, slot); the dots
 *     are exact int32; g = ((float)acc_g * s_g) * s_x, u likewise, h = fp32 of the fp64
 *     SwiGLU, y_e = ((float)acc_d * s_d) * s_h.
 * From 32 tokens on (d and f multiples of 64), the grouped gate/up and down stages run on the
 * fifth-generation tensor cores (int8 MMAs on decoded weight tiles, accumulators in tensor
 * memory); their integer sums are the same as those of the other kernels, so a token's output
 * does not depend on the batch it is in.
 * x [T][d] bf16, y [T][d] bf16, y_f32 [T][d] or NULL.  1 <= T <= T_max <= 64. */
size_t moe_ffn_workspace_bytes(const tern_moe_layer *L, int64_t T_max, tern_act act);
tern_status moe_ffn_workspace_layout(const tern_moe_layer *L, int64_t T_max, tern_act act,
                                     tern_ffn_layout *out);
tern_status moe_ffn_decode(const tern_moe_layer *L, const uint16_t *x, int64_t T, tern_act act,
                           uint16_t *y, float *y_f32, void *workspace, size_t ws_bytes,
                           void *stream);

/* A stack of n_layers residual MoE FFN layers, applied in place to x [T][d] (bf16):
 *   n = bf16(x / sqrt(mean(x^2) + rms_eps))   (fp64, no learned gain)
 *   x = bf16(x + moe_ffn_decode(n))            (exact sum, one rounding)
 * All layers must share d, f, E, k.  1 <= n_layers <= 64.  The whole stack runs in ONE
 * cooperative launch (one CTA per SM, every in-kernel wait bounded) when
 *   T == 1: the batch-1 kernel (the CTAs exchange data through tagged words in the
 *           workspace); needs d == 2048, f % 64 == 0 with f / 64 a power of two, E <= 256,
 *           k <= 8, 16-byte aligned scale arrays;
 *   2 <= T <= 16: the small-batch kernel (grid-wide barriers between the stages of a layer;
 *           every selected expert's rows are read once per layer and applied to all of its
 *           tokens); needs d == 2048, f in {128, 256, 512}, E <= 256, k <= 8;
 * otherwise it runs layer by layer, kernel per stage.  Every path gives each token the same
 * bits, whatever else is in its batch.  A timed-out in-kernel wait sets the device status
 * word to TERN_ETIMEOUT (read it with tern_stream_status); x is then unspecified, and the
 * workspace can be used again as it is. */
size_t moe_stack_workspace_bytes(const tern_moe_layer *L0, int64_t T_max, tern_act act);
tern_status moe_stack_decode(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, int64_t T,
                             float rms_eps, tern_act act, void *workspace, size_t ws_bytes,
                             void *stream);

/* Approximate output head ("A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on
 * a $599 Mac Mini", "The Architecture: Designed for the Hardware": cluster the vocabulary,
 * score 4-bit cluster centroids, project only the tokens of the best clusters).
 * The unembedding W [V][d] (bf16, V = n_clusters * cluster_size) is stored cluster-major:
 * cluster c holds tokens c*cluster_size .. (c+1)*cluster_size - 1.
 *
 * flash_head_centroids (preparation, once per W): centroid c = exact mean of its cluster's
 * rows; stored as symmetric int4 codes C4 [n_clusters][d/2] (values in [-7, 7], element 2j in
 * the low nibble of byte j, two's complement) and one fp64 scale c_scale[c] = absmax / 7
 * (codes = clamp(rint(centroid / scale)), ties to even; a zero centroid has scale 0).
 *
 * flash_head, one token x [d] (bf16):
 *   scores[c] = c_scale[c] * sum_k code_ck x_k           (fp64, exact sum) [n_clusters];
 *   sel_clusters = the top_c clusters by score, larger first, ties to the lower index [top_c];
 *   cand_ids / cand_logits = the tokens of the selected clusters in selection order, then row
 *     order, and sum_k W_vk x_k (fp64, exact products)   [top_c * cluster_size];
 *   best_id[0] = the candidate with the largest logit, ties to the lower token id.
 * top_c = n_clusters gives the full head.  64 <= d <= 8192, d % 64 == 0,
 * 1 <= n_clusters <= 8192, 1 <= cluster_size <= 1024, 1 <= top_c <= n_clusters.  W 16-byte
 * aligned.  All outputs are caller-owned device arrays; nothing else is allocated. */
tern_status flash_head_centroids(const uint16_t *W, int64_t d, int32_t n_clusters, int32_t cluster_size,
                                 uint8_t *C4, double *c_scale, void *stream);
tern_status flash_head(const uint8_t *C4, const double *c_scale, const uint16_t *W, const uint16_t *x,
                       int64_t d, int32_t n_clusters, int32_t cluster_size, int32_t top_c,
                       double *scores, int32_t *sel_clusters, int32_t *cand_ids, double *cand_logits,
                       int32_t *best_id, void *stream);

/* Where, inside a moe_stack_decode workspace, a one-launch call with T tokens leaves its
 * per-layer record, for inspection and parity checks (byte offsets; pass T_max = T, and a
 * workspace of at least moe_stack_workspace_bytes(L0, T, act) bytes):
 *   hist    uint16 [n_layers+1][T][d]  bf16 x entering each layer, and the final x;
 *   idx     int32  [n_layers][T][k]    experts chosen at each layer (descending logit);
 *   gates64 double [n_layers][T][k]    their renormalised gates;
 *   y32     float  [n_layers][T][d]    each layer's FFN output y before its bf16 cast (the
 *                                      value the residual adds), for parity checks;
 *   h32     float  [n_layers][T][k][f] each layer's SwiGLU output h of every slot (the down
 *                                      projection's input, before its limbs or int8 codes);
 *   (T == 1 only:)
 *   trace   uint64 [2][n_layers][P][24]: %globaltimer (ns), then clock64 (SM cycles), stamped
 *           by each of the P CTAs (one per SM, P = moe_stack_persistent_ctas(), P <= 256) at
 *           phase boundaries, written only when
 *           the environment variable TERNMOE_TRACE is "1" at the time of the call: 0 layer
 *           start, 1 x received, 2 router logits published, 3 activation limbs built (with
 *           TERNMOE_PREDICT=1: predicted next-layer logits published), 4 all logits received, 5 top-k done and row copies issued, 6 first
 *           gate/up rows landed, 7 gate/up dots done, 8 h published, 9 slot's h received,
 *           10 h limbs built, 11 down rows landed, 12 down dots done and published, 13 the
 *           slots' outputs of this CTA's rows received, 14 x' published; inside the phases
 *           (CTA thread 0): 15 r known, 16 n known, 17 own router partials written, 18 top-k
 *           known (before the copies are issued); 19..23 unused.
 * With TERNMOE_PREDICT=1 in the environment the persistent kernel also prefetches the experts
 * it predicts for the next layer into L2 (a hint that changes no value; off by default). */
typedef struct {
    int64_t hist, idx, gates64, y32, h32, trace, total;
} tern_stack_layout;
tern_status moe_stack_workspace_layout(const tern_moe_layer *L0, int64_t T_max, tern_act act,
                                       tern_stack_layout *out);

/* CTAs of the persistent T == 1 kernel for these layers on the current device (k groups of
 * G CTAs, at most one per SM), or 0 when a T == 1 call would run layer by layer instead. */
int32_t moe_stack_persistent_ctas(const tern_moe_layer *L0, int32_t n_layers, tern_act act);

/* Number of kernel launches one moe_stack_decode call with these arguments makes on the
 * current device (1 on the one-launch paths), or -1 if the arguments are invalid. */
int32_t moe_stack_kernel_launches(const tern_moe_layer *L0, int32_t n_layers, int64_t T, tern_act act);

/* Waits for `stream`, then returns and clears the device status word of the current device
 * (TERN_OK, or TERN_ETIMEOUT if an in-kernel bounded wait gave up since the last read), or
 * TERN_ECUDA if the wait itself failed. */
tern_status tern_stream_status(void *stream);

/* Test hook for the persistent stack kernel's own bounded waits: the same launch as
 * moe_stack_decode at T = 1, except that at layer `stall_layer` CTA 0 waits for a slot's h
 * with a tag no CTA ever writes, and every in-kernel wait gives up after limit_ns (1 us ..
 * 1 s) instead of one second.  CTA 0 gives up first; the others then miss its outputs and give
 * up too; each lets its own bulk copies land before it leaves.  The kernel returns by itself:
 * tern_stream_status then reports TERN_ETIMEOUT, and the next moe_stack_decode call on the
 * same workspace runs normally (its tags carry a new launch epoch).  x is left unspecified.
 * Returns TERN_EUNSUPPORTED when the arguments would not take the persistent path. */
tern_status tern_test_stack_stall(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, float rms_eps,
                                  tern_act act, int32_t stall_layer, int64_t limit_ns, void *workspace,
                                  size_t ws_bytes, void *stream);

/* Test hook for the small-batch stack kernel's own bounded waits (2 <= T <= 16): the same
 * launch as moe_stack_decode with T tokens, except that at layer `stall_layer` CTA 0 waits at
 * the grid barrier after the gate/up stage without arriving there, and every in-kernel wait
 * gives up after limit_ns (1 us .. 1 s).  Every CTA then gives up at that barrier and leaves;
 * the last one out resets the barrier counters, so the next moe_stack_decode call on the same
 * workspace runs normally.  tern_stream_status reports TERN_ETIMEOUT; x is left unspecified.
 * Returns TERN_EUNSUPPORTED when the arguments would not take the small-batch path. */
tern_status tern_test_stack_batch_stall(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, int64_t T,
                                        float rms_eps, tern_act act, int32_t stall_layer, int64_t limit_ns,
                                        void *workspace, size_t ws_bytes, void *stream);

/* Test hook for the bounded waits: launches one block that waits on a flag nobody sets,
 * for at most `spin_limit` polls, then sets TERN_ETIMEOUT in the device status word and
 * returns.  `flag` is a device int the caller owns (must stay 0). */
tern_status tern_test_bounded_wait(int32_t *flag, int64_t spin_limit, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* TERNMOE_H */
