// api.cu -- the extern "C" entry points of libternmoe.so: argument checks, workspace
// carving and dispatch to the sm_100a kernels.  See include/ternmoe.h for the contract.
#include <cuda_runtime.h>

#include <algorithm>
#include <stdint.h>

#include "../../include/ternmoe.h"
#include "kernels.h"

namespace tern {
__device__ int g_status = 0;
__device__ unsigned long long g_code_errors = 0;

int *status_word() {
    int *p = nullptr;
    if (cudaGetSymbolAddress((void **)&p, g_status) != cudaSuccess) return nullptr;
    return p;
}
}  // namespace tern

using namespace tern;

namespace {

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }
inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline int64_t up256(int64_t v) { return (v + 255) & ~int64_t(255); }
constexpr long long kStackWaitLimitNs = 1000000000ll;  // every wait of the persistent kernel: 1 s

// K <= 2048 must give a power-of-two lane count (K/64 in {1,2,4,...,32})
bool lanes_ok(int64_t K) {
    if (K <= 0 || K % 64 != 0) return false;
    if (K > 2048) return K % 2048 == 0 && K <= 16384;
    const int64_t g = K / 64;
    return g >= 1 && (g & (g - 1)) == 0;
}

tern_status check_layer(const tern_moe_layer *L) {
    if (!L) return TERN_EINVAL;
    if (!L->gate || !L->up || !L->down || !L->gate_scale || !L->up_scale || !L->down_scale || !L->router)
        return TERN_EINVAL;
    if (L->d <= 0 || L->f <= 0 || L->d % 64 || L->f % 64 || L->d > 2048 || L->f > 2048) return TERN_EINVAL;
    if (!lanes_ok(L->d) || !lanes_ok(L->f)) return TERN_EINVAL;
    if (L->E < 1 || L->E > kMaxE || L->k < 1 || L->k > kMaxKsel || L->k > L->E) return TERN_EINVAL;
    if (!aligned(L->gate, 16) || !aligned(L->up, 16) || !aligned(L->down, 16) || !aligned(L->router, 16) ||
        !aligned(L->gate_scale, 4) || !aligned(L->up_scale, 4) || !aligned(L->down_scale, 4))
        return TERN_EALIGN;
    return TERN_OK;
}

struct Layout {
    int64_t ctrl, logits, idx, g64, g32, n_unique, uexp, uoff, ent, xw, xsc, h, hw, hsc, acc_g, acc_u, acc_d, ye;
    int64_t total;
};

Layout make_layout(int64_t d, int64_t f, int32_t E, int32_t k, int64_t T, tern_act act) {
    const int64_t NL = act == TERN_ACT_INT8 ? 1 : 3;
    Layout o{};
    int64_t p = 0;
    auto take = [&](int64_t bytes) {
        const int64_t r = p;
        p = up256(p + bytes);
        return r;
    };
    o.ctrl = take(256);
    o.logits = take(T * E * 8);
    o.idx = take(T * k * 4);
    o.g64 = take(T * k * 8);
    o.g32 = take(T * k * 4);
    o.n_unique = take(16);
    o.uexp = take((int64_t)E * 4);
    o.uoff = take(((int64_t)E + 1) * 4);
    o.ent = take(T * k * 4);
    o.xw = take(T * NL * d);          // NL limb bytes per element
    o.xsc = take(T * 4);
    o.h = take(T * k * f * 4);
    o.hw = take(T * k * NL * f);
    o.hsc = take(T * k * 4);
    o.acc_g = take(act == TERN_ACT_INT8 ? T * k * f * 4 : 0);
    o.acc_u = take(act == TERN_ACT_INT8 ? T * k * f * 4 : 0);
    o.acc_d = take(act == TERN_ACT_INT8 ? T * k * d * 4 : 0);
    o.ye = take(T * k * d * 8);
    o.total = p;
    return o;
}

FfnWs carve(void *ws, const Layout &o, tern_act act) {
    char *b = static_cast<char *>(ws);
    FfnWs w{};
    w.ctrl = reinterpret_cast<unsigned int *>(b + o.ctrl);
    w.logits = reinterpret_cast<double *>(b + o.logits);
    w.idx = reinterpret_cast<int32_t *>(b + o.idx);
    w.g64 = reinterpret_cast<double *>(b + o.g64);
    w.g32 = reinterpret_cast<float *>(b + o.g32);
    w.n_unique = reinterpret_cast<int32_t *>(b + o.n_unique);
    w.uexp = reinterpret_cast<int32_t *>(b + o.uexp);
    w.uoff = reinterpret_cast<int32_t *>(b + o.uoff);
    w.ent = reinterpret_cast<int32_t *>(b + o.ent);
    w.xw = reinterpret_cast<uint32_t *>(b + o.xw);
    w.xsc = reinterpret_cast<float *>(b + o.xsc);
    w.h = reinterpret_cast<float *>(b + o.h);
    w.hw = reinterpret_cast<uint32_t *>(b + o.hw);
    w.hsc = reinterpret_cast<float *>(b + o.hsc);
    w.acc_g = act == TERN_ACT_INT8 ? reinterpret_cast<int32_t *>(b + o.acc_g) : nullptr;
    w.acc_u = act == TERN_ACT_INT8 ? reinterpret_cast<int32_t *>(b + o.acc_u) : nullptr;
    w.acc_d = act == TERN_ACT_INT8 ? reinterpret_cast<int32_t *>(b + o.acc_d) : nullptr;
    w.ye = reinterpret_cast<double *>(b + o.ye);
    return w;
}

tern_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TERN_OK : TERN_ECUDA; }

}  // namespace

extern "C" {

const char *tern_status_str(tern_status s) {
    switch (s) {
        case TERN_OK: return "TERN_OK";
        case TERN_EINVAL: return "TERN_EINVAL: invalid argument";
        case TERN_EALIGN: return "TERN_EALIGN: misaligned pointer";
        case TERN_ECODE: return "TERN_ECODE: invalid ternary value or code";
        case TERN_ECUDA: return "TERN_ECUDA: CUDA error";
        case TERN_ETIMEOUT: return "TERN_ETIMEOUT: bounded in-kernel wait gave up";
        case TERN_EWORKSPACE: return "TERN_EWORKSPACE: workspace missing or too small";
        case TERN_EUNSUPPORTED: return "TERN_EUNSUPPORTED: not implemented for these arguments";
    }
    return "unknown tern_status";
}

int32_t tern_abi_version(void) { return TERNMOE_ABI_VERSION; }

static tern_status pack_common(bool pack, const void *src, int64_t M, int64_t K, void *dst, void *stream) {
    if (!src || !dst || M <= 0 || K <= 0 || K % 4) return TERN_EINVAL;
    unsigned long long *bad = nullptr;
    if (cudaGetSymbolAddress((void **)&bad, g_code_errors) != cudaSuccess) return TERN_ECUDA;
    if (cudaMemsetAsync(bad, 0, sizeof(unsigned long long), S(stream)) != cudaSuccess) return TERN_ECUDA;
    cudaError_t e = pack ? launch_pack(static_cast<const int8_t *>(src), M, K, static_cast<uint8_t *>(dst), bad, S(stream))
                         : launch_unpack(static_cast<const uint8_t *>(src), M, K, static_cast<int8_t *>(dst), bad,
                                         S(stream));
    if (e != cudaSuccess) return TERN_ECUDA;
    unsigned long long h = 0;
    if (cudaMemcpyAsync(&h, bad, sizeof(h), cudaMemcpyDeviceToHost, S(stream)) != cudaSuccess) return TERN_ECUDA;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return TERN_ECUDA;
    return h ? TERN_ECODE : TERN_OK;
}

tern_status tern_pack(const int8_t *w, int64_t M, int64_t K, uint8_t *packed, void *stream) {
    return pack_common(true, w, M, K, packed, stream);
}

tern_status tern_unpack(const uint8_t *packed, int64_t M, int64_t K, int8_t *w, void *stream) {
    return pack_common(false, packed, M, K, w, stream);
}

tern_status tern_gemv(const uint8_t *Wp, const float *row_scale, int64_t M, int64_t K, tern_act act, const void *x,
                      const float *x_scale, int64_t T, int32_t *acc, float *y, void *stream) {
    if (!Wp || !row_scale || !x || !y || M <= 0 || M > (1ll << 30) || T < 1 || T > kMaxT) return TERN_EINVAL;
    if (!lanes_ok(K)) return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    if (act == TERN_ACT_BF16 && (acc || x_scale)) return TERN_EINVAL;
    if (!aligned(Wp, 16) || !aligned(x, 16) || !aligned(row_scale, 4) || !aligned(y, 4) ||
        (acc && !aligned(acc, 4)) || (x_scale && !aligned(x_scale, 4)))
        return TERN_EALIGN;
    return cuda_status(launch_gemv(Wp, row_scale, M, K, act, x, x_scale, T, acc, y, S(stream)));
}

tern_status tern_quant_absmax(const uint16_t *x, int64_t T, int64_t n, int8_t *q, float *s, void *stream) {
    if (!x || !q || !s || T < 1 || n < 1 || T > (1 << 30)) return TERN_EINVAL;
    if (!aligned(x, 2) || !aligned(s, 4)) return TERN_EALIGN;
    return cuda_status(launch_quant_absmax(x, T, n, q, s, S(stream)));
}

size_t moe_route_workspace_bytes(int64_t T, int32_t E) {
    if (T < 1 || E < 1) return 0;
    return (size_t)(256 + up256(T * E * 8) + up256(T * kMaxKsel * 8));
}

tern_status moe_route_topk(const uint16_t *Wg, const uint16_t *x, int64_t T, int64_t d, int32_t E, int32_t k,
                           int32_t *topk_idx, float *topk_gate, double *logits, void *workspace, size_t ws_bytes,
                           void *stream) {
    if (!Wg || !x || !topk_idx || !topk_gate || T < 1 || T > kMaxT || d < 8 || d % 8 || E < 1 || E > kMaxE ||
        k < 1 || k > kMaxKsel || k > E)
        return TERN_EINVAL;
    if (!aligned(Wg, 16) || !aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_gate, 4) ||
        (logits && !aligned(logits, 8)))
        return TERN_EALIGN;
    if (!workspace || ws_bytes < moe_route_workspace_bytes(T, E)) return TERN_EWORKSPACE;
    if (!aligned(workspace, 256)) return TERN_EALIGN;
    char *b = static_cast<char *>(workspace);
    unsigned int *ctrl = reinterpret_cast<unsigned int *>(b);
    double *lg = logits ? logits : reinterpret_cast<double *>(b + 256);
    double *g64 = reinterpret_cast<double *>(b + 256 + up256(T * E * 8));
    return cuda_status(launch_route(Wg, x, (int)T, (int)d, E, k, lg, topk_idx, topk_gate, g64, ctrl, false, nullptr,
                                    nullptr, nullptr, nullptr, S(stream)));
}

size_t moe_ffn_workspace_bytes(const tern_moe_layer *L, int64_t T_max, tern_act act) {
    if (check_layer(L) != TERN_OK || T_max < 1 || T_max > kMaxT) return 0;
    return (size_t)make_layout(L->d, L->f, L->E, L->k, T_max, act).total;
}

tern_status moe_ffn_workspace_layout(const tern_moe_layer *L, int64_t T_max, tern_act act, tern_ffn_layout *out) {
    tern_status st = check_layer(L);
    if (st != TERN_OK) return st;
    if (!out || T_max < 1 || T_max > kMaxT) return TERN_EINVAL;
    const Layout o = make_layout(L->d, L->f, L->E, L->k, T_max, act);
    const bool i8 = act == TERN_ACT_INT8;
    out->logits = o.logits;
    out->idx = o.idx;
    out->gates64 = o.g64;
    out->gates32 = o.g32;
    out->h = o.h;
    out->qx = i8 ? o.xw : -1;
    out->sx = i8 ? o.xsc : -1;
    out->qh = i8 ? o.hw : -1;
    out->sh = i8 ? o.hsc : -1;
    out->acc_g = i8 ? o.acc_g : -1;
    out->acc_u = i8 ? o.acc_u : -1;
    out->acc_d = i8 ? o.acc_d : -1;
    out->ye = o.ye;
    out->n_unique = o.n_unique;
    out->total = o.total;
    return TERN_OK;
}

tern_status moe_ffn_decode(const tern_moe_layer *L, const uint16_t *x, int64_t T, tern_act act, uint16_t *y,
                           float *y_f32, void *workspace, size_t ws_bytes, void *stream) {
    tern_status st = check_layer(L);
    if (st != TERN_OK) return st;
    if (!x || !y || T < 1 || T > kMaxT) return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    if (!aligned(x, 16) || !aligned(y, 2) || (y_f32 && !aligned(y_f32, 4))) return TERN_EALIGN;
    const Layout o = make_layout(L->d, L->f, L->E, L->k, T, act);
    if (!workspace || ws_bytes < (size_t)o.total) return TERN_EWORKSPACE;
    if (!aligned(workspace, 256)) return TERN_EALIGN;
    const FfnWs w = carve(workspace, o, act);
    return cuda_status(launch_ffn_stages(L, x, (int)T, act, w, y, y_f32, nullptr, nullptr, S(stream)));
}

// One-launch regions after the stage path's workspace and the layer input copy: the batch-1
// persistent kernel's region, then (T_max >= 2) the small-batch kernel's, sized for
// min(T_max, 16) tokens.  The two never overlap, so neither kernel sees the other's words.
static int64_t batch_region_bytes(const tern_moe_layer *L0, int64_t T_max) {
    return T_max >= 2 ? up256((int64_t)stack_batch_ws_bytes(L0, std::min<int64_t>(T_max, kBatchMaxT))) : 0;
}

size_t moe_stack_workspace_bytes(const tern_moe_layer *L0, int64_t T_max, tern_act act) {
    if (check_layer(L0) != TERN_OK || T_max < 1 || T_max > kMaxT) return 0;
    const Layout o = make_layout(L0->d, L0->f, L0->E, L0->k, T_max, act);
    int64_t tot = o.total + up256(T_max * L0->d * 2);
    const int64_t pers = (int64_t)stack_persistent_ws_bytes(L0);
    return (size_t)(tot + up256(pers) + batch_region_bytes(L0, T_max));
}

tern_status moe_stack_decode(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, int64_t T, float rms_eps,
                             tern_act act, void *workspace, size_t ws_bytes, void *stream) {
    if (!layers || n_layers < 1 || n_layers > kMaxLayers || !x || T < 1 || T > kMaxT) return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    if (!(rms_eps >= 0.0f)) return TERN_EINVAL;
    for (int i = 0; i < n_layers; i++) {
        tern_status st = check_layer(&layers[i]);
        if (st != TERN_OK) return st;
        if (layers[i].d != layers[0].d || layers[i].f != layers[0].f || layers[i].E != layers[0].E ||
            layers[i].k != layers[0].k)
            return TERN_EINVAL;
    }
    if (!aligned(x, 16)) return TERN_EALIGN;
    const size_t need = moe_stack_workspace_bytes(&layers[0], T, act);
    if (!workspace || ws_bytes < need) return TERN_EWORKSPACE;
    if (!aligned(workspace, 256)) return TERN_EALIGN;
    const Layout o = make_layout(layers[0].d, layers[0].f, layers[0].E, layers[0].k, T, act);
    char *b = static_cast<char *>(workspace);
    if (T == 1) {
        tern_status st = launch_stack_persistent(layers, n_layers, x, rms_eps, act,
                                                 b + o.total + up256(T * layers[0].d * 2),
                                                 (size_t)up256((int64_t)stack_persistent_ws_bytes(&layers[0])),
                                                 status_word(), -1, kStackWaitLimitNs, S(stream));
        if (st != TERN_EUNSUPPORTED) return st;
    }
    if (T >= 2 && T <= kBatchMaxT) {
        const int64_t at = o.total + up256(T * layers[0].d * 2) + up256((int64_t)stack_persistent_ws_bytes(&layers[0]));
        tern_status st = launch_stack_batch(layers, n_layers, x, T, rms_eps, act, b + at,
                                            (size_t)batch_region_bytes(&layers[0], T), status_word(),
                                            kStackWaitLimitNs, S(stream));
        if (st != TERN_EUNSUPPORTED) return st;
    }
    const FfnWs w = carve(workspace, o, act);
    uint16_t *n = reinterpret_cast<uint16_t *>(b + o.total);
    for (int l = 0; l < n_layers; l++) {
        cudaError_t e = launch_rmsnorm(x, (int)T, (int)layers[l].d, (double)rms_eps, n, S(stream));
        if (e != cudaSuccess) return TERN_ECUDA;
        e = launch_ffn_stages(&layers[l], n, (int)T, act, w, nullptr, nullptr, x, x, S(stream));
        if (e != cudaSuccess) return TERN_ECUDA;
    }
    return TERN_OK;
}

tern_status moe_stack_workspace_layout(const tern_moe_layer *L0, int64_t T_max, tern_act act, tern_stack_layout *out) {
    tern_status st = check_layer(L0);
    if (st != TERN_OK) return st;
    if (!out || T_max < 1 || T_max > kMaxT) return TERN_EINVAL;
    const Layout o = make_layout(L0->d, L0->f, L0->E, L0->k, T_max, act);
    const int64_t base = o.total + up256(T_max * L0->d * 2);
    int64_t hist, idx, g, y32, h32, tr;
    stack_persistent_offsets(L0, &hist, &idx, &g, &y32, &h32, &tr);
    out->trace = base + tr;
    if (T_max >= 2) {
        // the small-batch kernel's record (a call with T = T_max tokens writes it)
        const int64_t bb = base + up256((int64_t)stack_persistent_ws_bytes(L0));
        stack_batch_offsets(L0, std::min<int64_t>(T_max, kBatchMaxT), &hist, &idx, &g, &y32, &h32, &tr);
        out->trace = bb + tr;
        hist += bb - base;
        idx += bb - base;
        g += bb - base;
        y32 += bb - base;
        h32 += bb - base;
    }
    out->hist = base + hist;
    out->idx = base + idx;
    out->gates64 = base + g;
    out->y32 = base + y32;
    out->h32 = base + h32;
    out->total = (int64_t)moe_stack_workspace_bytes(L0, T_max, act);
    return TERN_OK;
}

int32_t moe_stack_kernel_launches(const tern_moe_layer *L0, int32_t n_layers, int64_t T, tern_act act) {
    if (check_layer(L0) != TERN_OK || n_layers < 1 || n_layers > kMaxLayers || T < 1 || T > kMaxT) return -1;
    if (T == 1 && stack_persistent_supported(L0, n_layers, act)) return 1;
    if (T >= 2 && T <= kBatchMaxT && stack_batch_supported(L0, n_layers, T, act)) return 1;
    return 8 * n_layers;  // rmsnorm, logits, select, prep, gate/up, prep, down, combine
}

int32_t moe_stack_persistent_ctas(const tern_moe_layer *L0, int32_t n_layers, tern_act act) {
    if (check_layer(L0) != TERN_OK || n_layers < 1 || n_layers > kMaxLayers) return 0;
    return stack_persistent_ctas(L0, n_layers, act);
}

tern_status tern_stream_status(void *stream) {
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return TERN_ECUDA;
    int h = 0;
    if (cudaMemcpyFromSymbol(&h, g_status, sizeof(int)) != cudaSuccess) return TERN_ECUDA;
    const int z = 0;
    if (cudaMemcpyToSymbol(g_status, &z, sizeof(int)) != cudaSuccess) return TERN_ECUDA;
    return (tern_status)h;
}

tern_status tern_test_stack_stall(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, float rms_eps,
                                  tern_act act, int32_t stall_layer, int64_t limit_ns, void *workspace,
                                  size_t ws_bytes, void *stream) {
    if (!layers || n_layers < 1 || n_layers > kMaxLayers || !x || stall_layer < 0 || stall_layer >= n_layers ||
        limit_ns < 1000 || limit_ns > kStackWaitLimitNs)
        return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    for (int i = 0; i < n_layers; i++) {
        tern_status st = check_layer(&layers[i]);
        if (st != TERN_OK) return st;
        if (layers[i].d != layers[0].d || layers[i].f != layers[0].f || layers[i].E != layers[0].E ||
            layers[i].k != layers[0].k)
            return TERN_EINVAL;
    }
    if (!aligned(x, 16)) return TERN_EALIGN;
    const size_t need = moe_stack_workspace_bytes(&layers[0], 1, act);
    if (!workspace || ws_bytes < need) return TERN_EWORKSPACE;
    if (!aligned(workspace, 256)) return TERN_EALIGN;
    const Layout o = make_layout(layers[0].d, layers[0].f, layers[0].E, layers[0].k, 1, act);
    char *b = static_cast<char *>(workspace);
    int *st = status_word();
    if (!st) return TERN_ECUDA;
    return launch_stack_persistent(layers, n_layers, x, rms_eps, act, b + o.total + up256(layers[0].d * 2),
                                   (size_t)up256((int64_t)stack_persistent_ws_bytes(&layers[0])), st, stall_layer,
                                   (long long)limit_ns, S(stream));
}

tern_status tern_test_stack_batch_stall(const tern_moe_layer *layers, int32_t n_layers, uint16_t *x, int64_t T,
                                        float rms_eps, tern_act act, int32_t stall_layer, int64_t limit_ns,
                                        void *workspace, size_t ws_bytes, void *stream) {
    if (!layers || n_layers < 1 || n_layers > kMaxLayers || !x || T < 2 || T > kBatchMaxT || stall_layer < 0 ||
        stall_layer >= n_layers || limit_ns < 1000 || limit_ns > kStackWaitLimitNs)
        return TERN_EINVAL;
    if (act != TERN_ACT_INT8 && act != TERN_ACT_BF16) return TERN_EINVAL;
    for (int i = 0; i < n_layers; i++) {
        tern_status st = check_layer(&layers[i]);
        if (st != TERN_OK) return st;
        if (layers[i].d != layers[0].d || layers[i].f != layers[0].f || layers[i].E != layers[0].E ||
            layers[i].k != layers[0].k)
            return TERN_EINVAL;
    }
    if (!aligned(x, 16)) return TERN_EALIGN;
    const size_t need = moe_stack_workspace_bytes(&layers[0], T, act);
    if (!workspace || ws_bytes < need) return TERN_EWORKSPACE;
    if (!aligned(workspace, 256)) return TERN_EALIGN;
    const Layout o = make_layout(layers[0].d, layers[0].f, layers[0].E, layers[0].k, T, act);
    char *b = static_cast<char *>(workspace);
    int *st = status_word();
    if (!st) return TERN_ECUDA;
    const int64_t at = o.total + up256(T * layers[0].d * 2) + up256((int64_t)stack_persistent_ws_bytes(&layers[0]));
    return launch_stack_batch(layers, n_layers, x, T, rms_eps, act, b + at, (size_t)batch_region_bytes(&layers[0], T), st,
                              (long long)limit_ns, S(stream), stall_layer);
}

tern_status tern_test_bounded_wait(int32_t *flag, int64_t spin_limit, void *stream) {
    if (!flag || spin_limit < 1) return TERN_EINVAL;
    if (!aligned(flag, 4)) return TERN_EALIGN;
    int *st = status_word();
    if (!st) return TERN_ECUDA;
    return cuda_status(launch_test_wait(flag, (long long)spin_limit, st, S(stream)));
}

}  // extern "C"
