"""Python binding of libternmoe.so (ternary-weight MoE FFN decode on B200, sm_100a).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  torch supplies device memory and the current stream; arrays are passed as
raw device pointers.  There is no CPU fallback: if the shared library is missing or no
CUDA device is present the calls raise.

The functions keep the C names of include/ternmoe.h.  Each takes torch tensors, checks
dtype/device/contiguity, calls the entry point and raises TernError on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libternmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "ternmoe.h")

TERN_ACT_BF16 = 0
TERN_ACT_INT8 = 1
STATUS = ["TERN_OK", "TERN_EINVAL", "TERN_EALIGN", "TERN_ECODE", "TERN_ECUDA", "TERN_ETIMEOUT",
          "TERN_EWORKSPACE", "TERN_EUNSUPPORTED"]


class TernError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        name = STATUS[code] if 0 <= code < len(STATUS) else str(code)
        super().__init__(f"{where}: {name}")


class MoELayerC(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("gate_scale", ctypes.c_void_p), ("up_scale", ctypes.c_void_p),
                ("down_scale", ctypes.c_void_p), ("router", ctypes.c_void_p),
                ("d", ctypes.c_int64), ("f", ctypes.c_int64), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32)]


_LAYOUT_FIELDS = ("logits", "idx", "gates64", "gates32", "h", "qx", "sx", "qh", "sh", "acc_g",
                  "acc_u", "acc_d", "ye", "n_unique", "total")


class FfnLayoutC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in _LAYOUT_FIELDS]


class StackLayoutC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("hist", "idx", "gates64", "y32", "h32", "trace", "total")]


_lib = None


def header_functions():
    """Names of the functions declared in include/ternmoe.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(tern_\w+|tern5_\w+|moe_\w+|flash_head\w*)\s*\(", txt)))


def lib():
    """Load libternmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run ternary_weight_moe_b200/build.py (no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        i64, i32, vp, st, sz = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sig = {
            "tern_status_str": (ctypes.c_char_p, [st]),
            "tern_abi_version": (i32, []),
            "tern_pack": (st, [vp, i64, i64, vp, vp]),
            "tern_unpack": (st, [vp, i64, i64, vp, vp]),
            "tern_gemv": (st, [vp, vp, i64, i64, st, vp, vp, i64, vp, vp, vp]),
            "tern_quant_absmax": (st, [vp, i64, i64, vp, vp, vp]),
            "flash_head_centroids": (st, [vp, i64, i32, i32, vp, vp, vp]),
            "flash_head": (st, [vp, vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
            "tern5_row_bytes": (i64, [i64]),
            "tern5_pack": (st, [vp, i64, i64, vp, vp]),
            "tern5_unpack": (st, [vp, i64, i64, vp, vp]),
            "tern5_gemv": (st, [vp, vp, i64, i64, st, vp, vp, i64, vp, vp, vp]),
            "moe_route_workspace_bytes": (sz, [i64, i32]),
            "moe_route_topk": (st, [vp, vp, i64, i64, i32, i32, vp, vp, vp, vp, sz, vp]),
            "moe_route_topk_static": (st, [vp, vp, i64, i64, i32, i32, vp, vp, vp, vp]),
            "moe_ffn_workspace_bytes": (sz, [ctypes.POINTER(MoELayerC), i64, st]),
            "moe_ffn_workspace_layout": (st, [ctypes.POINTER(MoELayerC), i64, st, ctypes.POINTER(FfnLayoutC)]),
            "moe_ffn_decode": (st, [ctypes.POINTER(MoELayerC), vp, i64, st, vp, vp, vp, sz, vp]),
            "moe_stack_workspace_bytes": (sz, [ctypes.POINTER(MoELayerC), i64, st]),
            "moe_stack_decode": (st, [ctypes.POINTER(MoELayerC), i32, vp, i64, ctypes.c_float, st, vp, sz, vp]),
            "moe_stack_workspace_layout": (st, [ctypes.POINTER(MoELayerC), i64, st, ctypes.POINTER(StackLayoutC)]),
            "moe_stack_kernel_launches": (i32, [ctypes.POINTER(MoELayerC), i32, i64, st]),
            "tern_stream_status": (st, [vp]),
            "tern_test_bounded_wait": (st, [vp, i64, vp]),
            "moe_stack_persistent_ctas": (i32, [ctypes.POINTER(MoELayerC), i32, st]),
            "tern_test_stack_stall": (st, [ctypes.POINTER(MoELayerC), i32, vp, ctypes.c_float, st, i32, i64, vp, sz,
                                           vp]),
            "tern_test_stack_batch_stall": (st, [ctypes.POINTER(MoELayerC), i32, vp, i64, ctypes.c_float, st, i32,
                                                 i64, vp, sz, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, where: str):
    if code != 0:
        raise TernError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _bits16(t, name):
    """bf16 tensors travel as their 16-bit patterns."""
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return _dev(t, torch.int16, name)


def status_str(code: int) -> str:
    return lib().tern_status_str(code).decode()


def abi_version() -> int:
    return lib().tern_abi_version()


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled device workspace (torch allocations are 512-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------- format

def tern_pack(w: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _dev(w, torch.int8, "w")
    M, K = w.shape
    if out is None:
        out = torch.empty((M, K // 4), dtype=torch.uint8, device=w.device)
    _dev(out, torch.uint8, "packed")
    _check(lib().tern_pack(_ptr(w), M, K, _ptr(out), _stream(stream)), "tern_pack")
    return out


def tern_unpack(packed: torch.Tensor, K: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _dev(packed, torch.uint8, "packed")
    M = packed.shape[0]
    if out is None:
        out = torch.empty((M, K), dtype=torch.int8, device=packed.device)
    _dev(out, torch.int8, "w")
    _check(lib().tern_unpack(_ptr(packed), M, K, _ptr(out), _stream(stream)), "tern_unpack")
    return out


# ------------------------------------------------------------------------------ GEMV

def tern_gemv(Wp, row_scale, x, act=TERN_ACT_BF16, x_scale=None, acc=None, y=None, K=None, stream=None):
    """y [T,M] (and acc [T,M] int32 on the int8 path) for x [T,K] (bf16 or int8)."""
    _dev(Wp, torch.uint8, "Wp")
    _dev(row_scale, torch.float32, "row_scale")
    M = Wp.shape[0]
    K = Wp.shape[1] * 4 if K is None else K
    if x.dim() == 1:
        x = x.view(1, -1)
    T = x.shape[0]
    if act == TERN_ACT_INT8:
        _dev(x, torch.int8, "x")
        if x_scale is not None:
            _dev(x_scale, torch.float32, "x_scale")
    else:
        x = _bits16(x, "x")
    if y is None:
        y = torch.empty((T, M), dtype=torch.float32, device=Wp.device)
    _dev(y, torch.float32, "y")
    if acc is not None:
        _dev(acc, torch.int32, "acc")
    _check(lib().tern_gemv(_ptr(Wp), _ptr(row_scale), M, K, act, _ptr(x), _ptr(x_scale), T, _ptr(acc),
                           _ptr(y), _stream(stream)), "tern_gemv")
    return y


def tern5_row_bytes(K: int) -> int:
    return int(lib().tern5_row_bytes(int(K)))


def tern5_pack(w: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Five weights per byte (base 3): [M, K] int8 -> [M, tern5_row_bytes(K)] uint8."""
    _dev(w, torch.int8, "w")
    M, K = w.shape
    if out is None:
        out = torch.empty((M, tern5_row_bytes(K)), dtype=torch.uint8, device=w.device)
    _dev(out, torch.uint8, "packed")
    _check(lib().tern5_pack(_ptr(w), M, K, _ptr(out), _stream(stream)), "tern5_pack")
    return out


def tern5_unpack(p: torch.Tensor, K: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _dev(p, torch.uint8, "packed")
    M = p.shape[0]
    if out is None:
        out = torch.empty((M, K), dtype=torch.int8, device=p.device)
    _dev(out, torch.int8, "w")
    _check(lib().tern5_unpack(_ptr(p), M, K, _ptr(out), _stream(stream)), "tern5_unpack")
    return out


def tern5_gemv(W5, row_scale, x, K, act=TERN_ACT_BF16, x_scale=None, acc=None, y=None, stream=None):
    """tern_gemv on base-3 packed rows; K is the number of weights per row."""
    _dev(W5, torch.uint8, "W5")
    _dev(row_scale, torch.float32, "row_scale")
    M = W5.shape[0]
    if x.dim() == 1:
        x = x.view(1, -1)
    T = x.shape[0]
    if act == TERN_ACT_INT8:
        _dev(x, torch.int8, "x")
        if x_scale is not None:
            _dev(x_scale, torch.float32, "x_scale")
    else:
        x = _bits16(x, "x")
    if y is None:
        y = torch.empty((T, M), dtype=torch.float32, device=W5.device)
    _dev(y, torch.float32, "y")
    if acc is not None:
        _dev(acc, torch.int32, "acc")
    _check(lib().tern5_gemv(_ptr(W5), _ptr(row_scale), M, K, act, _ptr(x), _ptr(x_scale), T, _ptr(acc), _ptr(y),
                            _stream(stream)), "tern5_gemv")
    return y


def flash_head_centroids(W, cluster_size: int, stream=None):
    """4-bit cluster centroids of a cluster-major bf16 unembedding W [V, d]: (C4, c_scale)."""
    W = _bits16(W, "W")
    V, d = W.shape
    nc = V // cluster_size
    C4 = torch.empty((nc, d // 2), dtype=torch.uint8, device=W.device)
    sc = torch.empty(nc, dtype=torch.float64, device=W.device)
    _check(lib().flash_head_centroids(_ptr(W), d, nc, cluster_size, _ptr(C4), _ptr(sc), _stream(stream)),
           "flash_head_centroids")
    return C4, sc


def flash_head(C4, c_scale, W, x, cluster_size: int, top_c: int, out=None, stream=None) -> dict:
    """One token through the approximate head; returns the device arrays of every output."""
    W = _bits16(W, "W")
    x = _bits16(x.view(-1), "x")
    V, d = W.shape
    nc = C4.shape[0]
    dev = W.device
    if out is None:
        out = {"scores": torch.empty(nc, dtype=torch.float64, device=dev),
               "sel": torch.empty(top_c, dtype=torch.int32, device=dev),
               "ids": torch.empty(top_c * cluster_size, dtype=torch.int32, device=dev),
               "logits": torch.empty(top_c * cluster_size, dtype=torch.float64, device=dev),
               "best": torch.empty(1, dtype=torch.int32, device=dev)}
    _check(lib().flash_head(_ptr(C4), _ptr(c_scale), _ptr(W), _ptr(x), d, nc, cluster_size, top_c,
                            _ptr(out["scores"]), _ptr(out["sel"]), _ptr(out["ids"]), _ptr(out["logits"]),
                            _ptr(out["best"]), _stream(stream)), "flash_head")
    return out


def tern_quant_absmax(x, q=None, s=None, stream=None):
    x = _bits16(x.view(-1, x.shape[-1]) if x.dim() > 1 else x.view(1, -1), "x")
    T, n = x.shape
    q = torch.empty((T, n), dtype=torch.int8, device=x.device) if q is None else q
    s = torch.empty(T, dtype=torch.float32, device=x.device) if s is None else s
    _check(lib().tern_quant_absmax(_ptr(x), T, n, _ptr(q), _ptr(s), _stream(stream)), "tern_quant_absmax")
    return q, s


# ---------------------------------------------------------------------------- router

def moe_route_workspace_bytes(T: int, E: int) -> int:
    return int(lib().moe_route_workspace_bytes(T, E))


def _route_args(Wg, x, k, logits, idx, gates):
    """Shape checks of the routing calls (before anything touches the device): Wg [E][d],
    x [T][d] (or [d]), logits [T][E], idx and gates [T][k]; then dtype/device checks."""
    if Wg.dim() != 2:
        raise ValueError(f"Wg must be [E, d], got {tuple(Wg.shape)}")
    E, d = Wg.shape
    x = x.view(1, -1) if x.dim() == 1 else x
    if x.dim() != 2 or x.shape[1] != d:
        raise ValueError(f"x must be [T, {d}], got {tuple(x.shape)}")
    T = x.shape[0]
    for name, t, shp in (("logits", logits, (T, E)), ("idx", idx, (T, k)), ("gates", gates, (T, k))):
        if t is not None and tuple(t.shape) != shp:
            raise ValueError(f"{name} must be {list(shp)}, got {tuple(t.shape)}")
    Wg = _bits16(Wg, "Wg")
    x = _bits16(x, "x")
    dev = Wg.device
    idx = torch.empty((T, k), dtype=torch.int32, device=dev) if idx is None else _dev(idx, torch.int32, "idx")
    gates = torch.empty((T, k), dtype=torch.float32, device=dev) if gates is None else _dev(gates, torch.float32,
                                                                                              "gates")
    if logits is not None:
        _dev(logits, torch.float64, "logits")
    return Wg, x, E, d, T, dev, idx, gates


def moe_route_topk(Wg, x, k=8, ws=None, logits=None, idx=None, gates=None, stream=None):
    Wg, x, E, d, T, dev, idx, gates = _route_args(Wg, x, k, logits, idx, gates)
    need = moe_route_workspace_bytes(T, E)
    ws = workspace(need, dev) if ws is None else ws
    _check(lib().moe_route_topk(_ptr(Wg), _ptr(x), T, d, E, k, _ptr(idx), _ptr(gates), _ptr(logits), _ptr(ws),
                                ws.numel(), _stream(stream)), "moe_route_topk")
    return idx, gates


def moe_route_topk_static(Wg, x, k=8, logits=None, idx=None, gates=None, stream=None):
    """Routing without a workspace (scratch is a fixed array inside the library; T <= 64,
    T * E <= 16384).  For callers that cannot allocate device memory."""
    Wg, x, E, d, T, dev, idx, gates = _route_args(Wg, x, k, logits, idx, gates)
    _check(lib().moe_route_topk_static(_ptr(Wg), _ptr(x), T, d, E, k, _ptr(idx), _ptr(gates), _ptr(logits),
                                       _stream(stream)), "moe_route_topk_static")
    return idx, gates


# ------------------------------------------------------------------------- MoE layer

class MoELayer:
    """Device tensors of one MoE FFN layer and the C struct that points at them."""

    def __init__(self, gate, up, down, gate_scale, up_scale, down_scale, router, k=8):
        self.gate = _dev(gate, torch.uint8, "gate")
        self.up = _dev(up, torch.uint8, "up")
        self.down = _dev(down, torch.uint8, "down")
        self.gate_scale = _dev(gate_scale, torch.float32, "gate_scale")
        self.up_scale = _dev(up_scale, torch.float32, "up_scale")
        self.down_scale = _dev(down_scale, torch.float32, "down_scale")
        self.router = _bits16(router, "router")
        self.E, self.f = gate_scale.shape
        self.d = down_scale.shape[1]
        self.k = k
        self.c = MoELayerC(gate.data_ptr(), up.data_ptr(), down.data_ptr(), gate_scale.data_ptr(),
                           up_scale.data_ptr(), down_scale.data_ptr(), self.router.data_ptr(),
                           self.d, self.f, self.E, k)


def moe_ffn_workspace_bytes(layer: MoELayer, T_max: int, act=TERN_ACT_BF16) -> int:
    return int(lib().moe_ffn_workspace_bytes(ctypes.byref(layer.c), T_max, act))


def moe_ffn_workspace_layout(layer: MoELayer, T_max: int, act=TERN_ACT_BF16) -> dict:
    out = FfnLayoutC()
    _check(lib().moe_ffn_workspace_layout(ctypes.byref(layer.c), T_max, act, ctypes.byref(out)),
           "moe_ffn_workspace_layout")
    return {n: int(getattr(out, n)) for n in _LAYOUT_FIELDS}


def moe_ffn_decode(layer: MoELayer, x, act=TERN_ACT_BF16, ws=None, y=None, y_f32=None, stream=None):
    """y [T,d] bf16 (and optionally y_f32) for x [T,d] bf16."""
    x = x.view(1, -1) if x.dim() == 1 else x
    xb = _bits16(x, "x")
    T = xb.shape[0]
    dev = xb.device
    y = torch.empty((T, layer.d), dtype=torch.bfloat16, device=dev) if y is None else y
    yb = _bits16(y, "y")
    if y_f32 is not None:
        _dev(y_f32, torch.float32, "y_f32")
    ws = workspace(moe_ffn_workspace_bytes(layer, T, act), dev) if ws is None else ws
    _check(lib().moe_ffn_decode(ctypes.byref(layer.c), _ptr(xb), T, act, _ptr(yb), _ptr(y_f32), _ptr(ws),
                                ws.numel(), _stream(stream)), "moe_ffn_decode")
    return y


def moe_stack_workspace_bytes(layer0: MoELayer, T_max: int, act=TERN_ACT_BF16) -> int:
    return int(lib().moe_stack_workspace_bytes(ctypes.byref(layer0.c), T_max, act))


class Stack:
    """A list of MoE layers packed into the C array moe_stack_decode takes."""

    def __init__(self, layers: list[MoELayer]):
        self.layers = layers
        arr = (MoELayerC * len(layers))()
        for i, L in enumerate(layers):
            arr[i] = L.c
        self.c = arr


def moe_stack_decode(stack: Stack, x, eps=1e-6, act=TERN_ACT_BF16, ws=None, stream=None):
    """In place: x [T,d] bf16 <- the residual stack applied to x."""
    xb = _bits16(x.view(1, -1) if x.dim() == 1 else x, "x")
    T = xb.shape[0]
    if ws is None:
        ws = workspace(moe_stack_workspace_bytes(stack.layers[0], T, act), xb.device)
    _check(lib().moe_stack_decode(stack.c, len(stack.layers), _ptr(xb), T, float(eps), act, _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_stack_decode")
    return x


def moe_stack_workspace_layout(layer0: MoELayer, T_max: int = 1, act=TERN_ACT_BF16) -> dict:
    out = StackLayoutC()
    _check(lib().moe_stack_workspace_layout(ctypes.byref(layer0.c), T_max, act, ctypes.byref(out)),
           "moe_stack_workspace_layout")
    return {n: int(getattr(out, n)) for n in ("hist", "idx", "gates64", "y32", "h32", "trace", "total")}


def moe_stack_persistent_ctas(layer0: MoELayer, n_layers: int, act=TERN_ACT_BF16) -> int:
    return int(lib().moe_stack_persistent_ctas(ctypes.byref(layer0.c), n_layers, act))


def moe_stack_kernel_launches(layer0: MoELayer, n_layers: int, T: int, act=TERN_ACT_BF16) -> int:
    return int(lib().moe_stack_kernel_launches(ctypes.byref(layer0.c), n_layers, T, act))


def tern_stream_status(stream=None) -> int:
    return int(lib().tern_stream_status(_stream(stream)))


def tern_test_stack_stall(stack: Stack, x, stall_layer: int, limit_ns: int, eps=1e-6, act=TERN_ACT_BF16, ws=None,
                          stream=None):
    """The T = 1 stack launch with one exchange that never completes (CTA 0, layer
    stall_layer) and every in-kernel wait bounded by limit_ns; the kernel must give up by
    itself and leave TERN_ETIMEOUT in the device status word."""
    xb = _bits16(x.view(1, -1) if x.dim() == 1 else x, "x")
    if ws is None:
        ws = workspace(moe_stack_workspace_bytes(stack.layers[0], 1, act), xb.device)
    _check(lib().tern_test_stack_stall(stack.c, len(stack.layers), _ptr(xb), float(eps), act, int(stall_layer),
                                       int(limit_ns), _ptr(ws), ws.numel(), _stream(stream)), "tern_test_stack_stall")
    return ws


def tern_test_stack_batch_stall(stack: Stack, x, stall_layer: int, limit_ns: int, eps=1e-6, act=TERN_ACT_BF16,
                                ws=None, stream=None):
    """The small-batch stack launch (x [T, d], 2 <= T <= 16) with CTA 0 not arriving at the grid
    barrier after the gate/up stage of layer stall_layer, and every in-kernel wait bounded by
    limit_ns; the kernel must give up by itself and leave TERN_ETIMEOUT in the status word."""
    xb = _bits16(x, "x")
    T = xb.shape[0]
    if ws is None:
        ws = workspace(moe_stack_workspace_bytes(stack.layers[0], T, act), xb.device)
    _check(lib().tern_test_stack_batch_stall(stack.c, len(stack.layers), _ptr(xb), T, float(eps), act,
                                             int(stall_layer), int(limit_ns), _ptr(ws), ws.numel(), _stream(stream)),
           "tern_test_stack_batch_stall")
    return ws


def tern_test_bounded_wait(flag: torch.Tensor, spin_limit: int, stream=None):
    _dev(flag, torch.int32, "flag")
    _check(lib().tern_test_bounded_wait(_ptr(flag), int(spin_limit), _stream(stream)), "tern_test_bounded_wait")
