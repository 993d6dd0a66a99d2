// route_static.cu -- moe_route_topk_static: the router / top-k call without a caller
// workspace, for callers that cannot allocate device memory.
//
// Some callers only ever receive device pointers to their inputs and outputs and have no
// way to obtain scratch memory: a plugin whose host framework owns every allocation, or a
// serving loop that forbids allocator calls once it has started.  This entry point lets
// them route tokens anyway: the scratch the router needs (an arrival counter, the fp64
// logits and the fp64 gates) lives in a fixed array compiled into the library, sized for at
// most kStaticRouteMaxT tokens and kStaticRouteMaxTE token-expert logits.  Every GPU that
// loads the library holds that array until the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/ternmoe.h"
#include "kernels.h"

namespace {

using tern::kMaxE;
using tern::kMaxKsel;
using tern::kStaticCtrlBytes;
using tern::kStaticLogitsBytes;
using tern::kStaticRouteBytes;
using tern::kStaticRouteMaxT;
using tern::kStaticRouteMaxTE;

// The scratch itself.  In host code this name is only a stand-in for the symbol, never a
// device address: the address comes from cudaGetSymbolAddress on the device that runs.
static __device__ __align__(256) unsigned char g_route_scratch[kStaticRouteBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
unsigned char *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch on the current device.  Outside stream capture it is looked
// up again on every call, so a context torn down and rebuilt (cudaDeviceReset) cannot leave a
// stale address behind; while `stream` is capturing, the address cached by the last
// non-capturing call on this device is used (a lookup may not be legal then), so the first
// call on a device must come before any capture.
tern_status scratch_on_current_device(cudaStream_t stream, unsigned char **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TERN_ECUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return TERN_ECUDA;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        unsigned char *p = nullptr;
        if (cudaGetSymbolAddress((void **)&p, g_route_scratch) != cudaSuccess || p == nullptr) return TERN_ECUDA;
        g_scratch_ptr[dev] = p;
    } else if (g_scratch_ptr[dev] == nullptr) {
        return TERN_ECUDA;  // never set up on this device outside a capture
    }
    *out = g_scratch_ptr[dev];
    return TERN_OK;
}

inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

extern "C" tern_status moe_route_topk_static(const uint16_t *Wg, const uint16_t *x, int64_t T, int64_t d, int32_t E,
                                             int32_t k, int32_t *topk_idx, float *topk_gate, double *logits,
                                             void *stream) {
    if (!Wg || !x || !topk_idx || !topk_gate || T < 1 || d < 8 || d % 8 || E < 1 || E > kMaxE || k < 1 ||
        k > kMaxKsel || k > E)
        return TERN_EINVAL;
    if (T > kStaticRouteMaxT || T * (int64_t)E > kStaticRouteMaxTE) return TERN_EINVAL;  // beyond the fixed scratch
    if (!aligned(Wg, 16) || !aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_gate, 4) ||
        (logits && !aligned(logits, 8)))
        return TERN_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    unsigned char *base = nullptr;
    const tern_status st = scratch_on_current_device(s, &base);
    if (st != TERN_OK) return st;
    unsigned int *ctrl = reinterpret_cast<unsigned int *>(base);
    double *lg = logits ? logits : reinterpret_cast<double *>(base + kStaticCtrlBytes);
    double *g64 = reinterpret_cast<double *>(base + kStaticCtrlBytes + kStaticLogitsBytes);
    // the arrival counter must start at zero; the array keeps whatever the last call left
    if (cudaMemsetAsync(ctrl, 0, sizeof(unsigned int), s) != cudaSuccess) return TERN_ECUDA;
    const cudaError_t e = tern::launch_route(Wg, x, (int)T, (int)d, E, k, lg, topk_idx, topk_gate, g64, ctrl, false,
                                             nullptr, nullptr, nullptr, nullptr, s);
    return e == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
