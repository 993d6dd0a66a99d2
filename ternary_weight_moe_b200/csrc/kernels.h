// kernels.h -- host-side launchers of the sm_100a kernels (internal to libternmoe).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ternmoe.h"

namespace tern {

// ---- limits shared by the host checks and the kernels' fixed-size shared arrays
constexpr int64_t kMaxT = 64;      // tokens per call
constexpr int32_t kMaxE = 1024;    // experts per layer
constexpr int32_t kMaxKsel = 8;    // experts selected per token
constexpr int32_t kMaxLayers = 64; // layers per stack call

// ---- fixed scratch of the allocation-free routing call (moe_route_topk_static)
constexpr int64_t kStaticRouteMaxT = 64;      // tokens
constexpr int64_t kStaticRouteMaxTE = 16384;  // tokens x experts, e.g. 64 x 256
constexpr size_t kStaticCtrlBytes = 256;
constexpr size_t kStaticLogitsBytes = (size_t)kStaticRouteMaxTE * 8;             // fp64 logits
constexpr size_t kStaticGatesBytes = (size_t)kStaticRouteMaxT * kMaxKsel * 8;    // fp64 gates
constexpr size_t kStaticRouteBytes = kStaticCtrlBytes + kStaticLogitsBytes + kStaticGatesBytes;  // 135,424 B
static_assert(kStaticRouteMaxT <= kMaxT, "the static route serves at most the tokens the kernels handle");
static_assert(kStaticRouteBytes == 135424, "documented size of the fixed routing scratch");

// ---- format
cudaError_t launch_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, unsigned long long *bad,
                        cudaStream_t s);
cudaError_t launch_unpack(const uint8_t *p, int64_t M, int64_t K, int8_t *w, unsigned long long *bad,
                          cudaStream_t s);
cudaError_t launch_quant_absmax(const uint16_t *x, int64_t T, int64_t n, int8_t *q, float *sc,
                                cudaStream_t s);

// ---- ternary GEMV
cudaError_t launch_gemv(const uint8_t *Wp, const float *rs, int64_t M, int64_t K, tern_act act,
                        const void *x, const float *xs, int64_t T, int32_t *acc, float *y, cudaStream_t s);

// ---- MoE layer, general T (kernel-per-stage path)
struct FfnWs {           // device pointers carved from the caller's workspace
    unsigned int *ctrl;  // [0] route arrival counter
    double *logits;      // [T][E]
    int32_t *idx;        // [T][k]
    double *g64;         // [T][k]
    float *g32;          // [T][k]
    int32_t *n_unique;   // [1]
    int32_t *uexp;       // [E]
    int32_t *uoff;       // [E+1]
    int32_t *ent;        // [T*k]
    uint32_t *xw;        // [T][NL][d/4] activation limb words
    float *xsc;          // [T] int8 scale, or shift (as int bits) on the bf16 path
    float *h;            // [T*k][f]
    uint32_t *hw;        // [T*k][NL][f/4]
    float *hsc;          // [T*k]
    int32_t *acc_g, *acc_u, *acc_d;  // int8 path traces
    double *ye;          // [T*k][d]
};

// grouped gate/up (phase 0) and down (phase 1) on tcgen05 tensor cores (moe_tc.cu), for the
// >= 32-token path; d and f multiples of 128
bool tc_grouped_supported(int d, int f);
template <int NL>
cudaError_t launch_grouped_tc(const tern_moe_layer *L, int T, const FfnWs &w, cudaStream_t s, int phase);

cudaError_t launch_route(const uint16_t *Wg, const uint16_t *x, int T, int d, int E, int k, double *logits,
                         int32_t *idx, float *g32, double *g64, unsigned int *counter, bool dispatch,
                         int32_t *n_unique, int32_t *uexp, int32_t *uoff, int32_t *ent, cudaStream_t s);

cudaError_t launch_ffn_stages(const tern_moe_layer *L, const uint16_t *x, int T, tern_act act, const FfnWs &w,
                              uint16_t *y, float *y_f32, const uint16_t *residual, uint16_t *x_out,
                              cudaStream_t s);

cudaError_t launch_rmsnorm(const uint16_t *x, int T, int d, double eps, uint16_t *n, cudaStream_t s);

// ---- persistent whole-stack decode, T == 1
struct StackLayerDev {
    const uint8_t *gate, *up, *down;
    const float *sg, *su, *sd;
    const uint16_t *router;
};
size_t stack_persistent_ws_bytes(const tern_moe_layer *L0);
bool stack_persistent_supported(const tern_moe_layer *L0, int n_layers, tern_act act);
int stack_persistent_ctas(const tern_moe_layer *L0, int n_layers, tern_act act);
void stack_persistent_offsets(const tern_moe_layer *L0, int64_t *hist, int64_t *idx_hist, int64_t *gate_hist,
                              int64_t *y_hist, int64_t *h_hist, int64_t *ttrace);
// stall_layer: -1, or a layer at which CTA 0 waits for data nobody sends (timeout test);
// limit_ns: bound on every in-kernel wait
tern_status launch_stack_persistent(const tern_moe_layer *layers, int n_layers, uint16_t *x, float eps,
                                    tern_act act, void *ws, size_t ws_bytes, int *status, int stall_layer,
                                    long long limit_ns, cudaStream_t s);

// ---- one-launch small-batch stack (stack_batch.cu): 2 <= T <= 16 tokens
constexpr int64_t kBatchMaxT = 16;
size_t stack_batch_ws_bytes(const tern_moe_layer *L0, int64_t T);
bool stack_batch_supported(const tern_moe_layer *L0, int n_layers, int64_t T, tern_act act);
void stack_batch_offsets(const tern_moe_layer *L0, int64_t T, int64_t *hist, int64_t *idx, int64_t *gates,
                         int64_t *y32, int64_t *h32, int64_t *trace);
// stall_layer: -1, or a layer at which CTA 0 does not arrive at the barrier after phase C (the
// timeout test); limit_ns: bound on every in-kernel wait
tern_status launch_stack_batch(const tern_moe_layer *layers, int n_layers, uint16_t *x, int64_t T, float eps,
                               tern_act act, void *ws, size_t ws_bytes, int *status, long long limit_ns,
                               cudaStream_t s, int stall_layer = -1);

// ---- bounded-wait test hook
cudaError_t launch_test_wait(int32_t *flag, long long limit, int *status, cudaStream_t s);

// address of the device status word on the current device
int *status_word();

}  // namespace tern
