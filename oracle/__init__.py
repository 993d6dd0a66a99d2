"""CPU oracle for ternary-weight MoE FFN decode (ctypes wrapper around ternmoe_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its Python binding) never imports this package, and this package
never imports the product.  Inputs come from `synth`, outputs are compared
against the CUDA library by the tests.

Every function takes and returns numpy arrays.  See ternmoe_oracle.c for the
definitions and the passages of the pages each one follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ternmoe_oracle.c")
_LIB = os.path.join(_HERE, "libternmoe_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libternmoe_oracle_omp.so")
_lock = threading.Lock()
_lib = None
_lib_omp = None

ACT_BF16 = 0
ACT_INT8 = 1


def build(force: bool = False, omp: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction).  omp=True builds the
    same source with -fopenmp (rows split across cores, identical results; timing only)."""
    out = _LIB_OMP if omp else _LIB
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", *(["-fopenmp"] if omp else []), "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, out)
    return out


class _Layer(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("gate_scale", ctypes.c_void_p), ("up_scale", ctypes.c_void_p),
                ("down_scale", ctypes.c_void_p), ("router", ctypes.c_void_p),
                ("d", ctypes.c_int64), ("f", ctypes.c_int64), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32)]


class _Trace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("idx", "gates", "logits", "h", "acc_g", "acc_u", "qx", "sx", "qh", "sh",
                 "acc_d", "ye")]


def lib():
    """The single-threaded oracle (the one every test uses)."""
    global _lib
    with _lock:
        if _lib is None:
            # a test may point the wrapper at a deliberately broken copy of the oracle
            _lib = _load(os.environ.get("TERNMOE_ORACLE_LIB") or build())
    return _lib


def lib_omp():
    """The same oracle built with OpenMP (for the benchmark's all-cores CPU timing)."""
    global _lib_omp
    with _lock:
        if _lib_omp is None:
            _lib_omp = _load(build(omp=True))
    return _lib_omp


def _load(path):
    L = ctypes.CDLL(path)
    i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
    L.or_pack.restype = i64
    L.or_pack.argtypes = [vp, i64, i64, vp]
    L.or_unpack.restype = i64
    L.or_unpack.argtypes = [vp, i64, i64, vp]
    L.or_tern5_row_bytes.restype = i64
    L.or_tern5_row_bytes.argtypes = [i64]
    L.or_pack5.restype = i64
    L.or_pack5.argtypes = [vp, i64, i64, vp]
    L.or_unpack5.restype = i64
    L.or_unpack5.argtypes = [vp, i64, i64, vp]
    L.or_gemv_i8.restype = ctypes.c_int
    L.or_gemv_i8.argtypes = [vp, vp, i64, i64, i64, vp, vp, vp, vp]
    L.or_gemv_bf16.restype = i64
    L.or_gemv_bf16.argtypes = [vp, vp, i64, i64, i64, vp, vp]
    L.or_quant_absmax.restype = None
    L.or_quant_absmax.argtypes = [vp, i64, vp, vp]
    L.or_rmsnorm.restype = i64
    L.or_rmsnorm.argtypes = [vp, i64, dbl, vp]
    L.or_route.restype = i64
    L.or_route.argtypes = [vp, vp, i64, i64, i32, i32, vp, vp, vp]
    L.or_moe_ffn.restype = i64
    L.or_moe_ffn.argtypes = [ctypes.POINTER(_Layer), vp, i64, ctypes.c_int, vp, vp,
                             ctypes.POINTER(_Trace), vp, vp, vp]
    L.or_stack_layer.restype = i64
    L.or_stack_layer.argtypes = [ctypes.POINTER(_Layer), vp, i64, dbl, ctypes.c_int, vp,
                                 vp, vp, vp, ctypes.POINTER(_Trace)]
    L.or_f64_to_bf16.restype = ctypes.c_uint16
    L.or_f64_to_bf16.argtypes = [dbl]
    L.or_bf16_to_f64.restype = dbl
    L.or_bf16_to_f64.argtypes = [ctypes.c_uint16]
    return L


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def pack(w):
    w = _c(w, np.int8)
    M, K = w.shape
    assert K % 4 == 0
    out = np.empty((M, K // 4), dtype=np.uint8)
    bad = lib().or_pack(_p(w), M, K, _p(out))
    return out, int(bad)


def unpack(p, K):
    p = _c(p, np.uint8)
    M = p.shape[0]
    w = np.empty((M, K), dtype=np.int8)
    bad = lib().or_unpack(_p(p), M, K, _p(w))
    return w, int(bad)


def tern5_row_bytes(K):
    """Bytes per row of the base-3 format (five weights per byte, rows padded to 16 bytes)."""
    return int(lib().or_tern5_row_bytes(int(K)))


def pack5(w):
    w = _c(w, np.int8)
    M, K = w.shape
    out = np.empty((M, tern5_row_bytes(K)), dtype=np.uint8)
    bad = lib().or_pack5(_p(w), M, K, _p(out))
    return out, int(bad)


def unpack5(p, K):
    p = _c(p, np.uint8)
    M = p.shape[0]
    w = np.empty((M, K), dtype=np.int8)
    bad = lib().or_unpack5(_p(p), M, K, _p(w))
    return w, int(bad)


def gemv5_i8(W5, s, q, x_scale=None):
    """The int8 GEMV of base-3 packed weights: the weights it decodes to, through gemv_i8."""
    q = np.atleast_2d(q)
    w, _ = unpack5(W5, q.shape[1])
    return gemv_i8(pack(w)[0], s, q, x_scale)


def gemv5_bf16(W5, s, x):
    x = np.atleast_2d(x)
    w, _ = unpack5(W5, x.shape[1])
    return gemv_bf16(pack(w)[0], s, x)


def gemv_i8(Wp, s, q, x_scale=None):
    """acc [T,M] int32 and y [T,M] fp32 for int8 activations q [T,K]."""
    Wp = _c(Wp, np.uint8)
    s = _c(s, np.float32)
    q = _c(np.atleast_2d(q), np.int8)
    T, K = q.shape
    M = Wp.shape[0]
    xs = None if x_scale is None else _c(np.atleast_1d(x_scale), np.float32)
    acc = np.empty((T, M), dtype=np.int32)
    y = np.empty((T, M), dtype=np.float32)
    rc = lib().or_gemv_i8(_p(Wp), _p(s), M, K, T, _p(q), _p(xs), _p(acc), _p(y))
    if rc != 0:
        raise OverflowError("int32 accumulator overflow")
    return acc, y


def gemv_bf16(Wp, s, x):
    """y [T,M] fp64 = s * exact ternary dot, for bf16 bits x [T,K]; also the inexact count."""
    Wp = _c(Wp, np.uint8)
    s = _c(s, np.float32)
    x = _c(np.atleast_2d(x), np.uint16)
    T, K = x.shape
    M = Wp.shape[0]
    y = np.empty((T, M), dtype=np.float64)
    bad = lib().or_gemv_bf16(_p(Wp), _p(s), M, K, T, _p(x), _p(y))
    return y, int(bad)


def quant_absmax(x):
    x = _c(x, np.float32)
    q = np.empty(x.shape, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    lib().or_quant_absmax(_p(x), x.size, _p(q), _p(s))
    return q, float(s[0])


def rmsnorm(x, eps=1e-6):
    x = _c(np.atleast_2d(x), np.uint16)
    n = np.empty_like(x)
    bad = 0
    for t in range(x.shape[0]):
        bad += lib().or_rmsnorm(_p(x[t]), x.shape[1], float(eps), _p(n[t]))
    return n, int(bad)


def route(Wg, x, k=8):
    Wg = _c(Wg, np.uint16)
    x = _c(np.atleast_2d(x), np.uint16)
    E, d = Wg.shape
    T = x.shape[0]
    logits = np.empty((T, E), dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    gates = np.empty((T, k), dtype=np.float64)
    bad = lib().or_route(_p(Wg), _p(x), T, d, E, k, _p(logits), _p(idx), _p(gates))
    return logits, idx, gates, int(bad)


def f64_to_bf16(v: float) -> int:
    return int(lib().or_f64_to_bf16(float(v)))


def bf16_to_f64(b: int) -> float:
    return float(lib().or_bf16_to_f64(int(b)))


class Layer:
    """Host copy of one MoE FFN layer (packed weights, scales, router)."""

    def __init__(self, gate_p, up_p, down_p, sg, su, sd, router, k=8):
        self.gate = _c(gate_p, np.uint8)     # [E,f,d/4]
        self.up = _c(up_p, np.uint8)         # [E,f,d/4]
        self.down = _c(down_p, np.uint8)     # [E,d,f/4]
        self.sg = _c(sg, np.float32)         # [E,f]
        self.su = _c(su, np.float32)
        self.sd = _c(sd, np.float32)         # [E,d]
        self.router = _c(router, np.uint16)  # [E,d]
        self.E, self.f = self.sg.shape
        self.d = self.sd.shape[1]
        self.k = k

    def _struct(self):
        return _Layer(_p(self.gate).value, _p(self.up).value, _p(self.down).value,
                      _p(self.sg).value, _p(self.su).value, _p(self.sd).value,
                      _p(self.router).value, self.d, self.f, self.E, self.k)


def moe_ffn(layer: Layer, x, act=ACT_BF16, qh_in=None, sh_in=None, h_in=None):
    """One MoE FFN layer; returns a dict of outputs and intermediates."""
    x = _c(np.atleast_2d(x), np.uint16)
    T = x.shape[0]
    d, f, E, k = layer.d, layer.f, layer.E, layer.k
    out = {
        "y_bf16": np.empty((T, d), np.uint16), "y64": np.empty((T, d), np.float64),
        "idx": np.empty((T, k), np.int32), "gates": np.empty((T, k), np.float64),
        "logits": np.empty((T, E), np.float64), "h": np.empty((T, k, f), np.float32),
        "acc_g": np.zeros((T, k, f), np.int32), "acc_u": np.zeros((T, k, f), np.int32),
        "qx": np.zeros((T, d), np.int8), "sx": np.zeros(T, np.float32),
        "qh": np.zeros((T, k, f), np.int8), "sh": np.zeros((T, k), np.float32),
        "acc_d": np.zeros((T, k, d), np.int32), "ye": np.empty((T, k, d), np.float64),
    }
    tr = _Trace(*[_p(out[n]).value for n in ("idx", "gates", "logits", "h", "acc_g", "acc_u",
                                              "qx", "sx", "qh", "sh", "acc_d", "ye")])
    L = layer._struct()
    qh_in = None if qh_in is None else _c(qh_in, np.int8)
    sh_in = None if sh_in is None else _c(sh_in, np.float32)
    h_in = None if h_in is None else _c(h_in, np.float32)
    bad = lib().or_moe_ffn(ctypes.byref(L), _p(x), T, act, _p(out["y_bf16"]), _p(out["y64"]),
                           ctypes.byref(tr), _p(qh_in), _p(sh_in), _p(h_in))
    out["inexact"] = int(bad)
    return out


def stack_layer(layer: Layer, x, eps=1e-6, act=ACT_BF16, omp=False):
    """One residual layer: returns x_out, n, y (bf16 bits), y64 and the FFN trace.
    omp=True runs the OpenMP build (same results, rows split across cores)."""
    x = _c(np.atleast_2d(x), np.uint16)
    T = x.shape[0]
    d, f, E, k = layer.d, layer.f, layer.E, layer.k
    x_out = np.empty_like(x)
    n = np.empty_like(x)
    y = np.empty_like(x)
    y64 = np.empty((T, d), np.float64)
    tr_arrays = {"idx": np.empty((T, k), np.int32), "gates": np.empty((T, k), np.float64),
                 "logits": np.empty((T, E), np.float64)}
    tr = _Trace(*[(_p(tr_arrays[nm]).value if nm in tr_arrays else None) for nm in
                  ("idx", "gates", "logits", "h", "acc_g", "acc_u", "qx", "sx", "qh", "sh",
                   "acc_d", "ye")])
    L = layer._struct()
    bad = (lib_omp() if omp else lib()).or_stack_layer(ctypes.byref(L), _p(x), T, float(eps), act, _p(x_out), _p(n),
                               _p(y), _p(y64), ctypes.byref(tr))
    return {"x_out": x_out, "n": n, "y": y, "y64": y64, "inexact": int(bad), **tr_arrays}


def pack_layer_codes(gc, uc, dc):
    """Pack int8 code tensors [E,f,d], [E,f,d], [E,d,f] with the oracle's packer."""
    E, f, d = gc.shape
    gp, b1 = pack(gc.reshape(E * f, d))
    up, b2 = pack(uc.reshape(E * f, d))
    dp, b3 = pack(dc.reshape(E * d, f))
    assert b1 == b2 == b3 == 0
    return gp.reshape(E, f, d // 4), up.reshape(E, f, d // 4), dp.reshape(E, d, f // 4)
