"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no packing, no dot products, no routing).  Every value is
a pure function of (seed, element index), so any slice of any tensor can be
regenerated on its own -- the CPU oracle regenerates only the experts a token
selected, the GPU side generates whole 24-layer stacks on the device.

Generator: the SplitMix64 output function (Steele, Lea & Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014; constants as in
Vigna's public-domain splitmix64.c) applied to a counter:

    draw(seed, i) = mix64(seed + (i + 1) * 0x9E3779B97F4A7C15   mod 2^64)
    mix64(z):  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
               z ^= z >> 27; z *= 0x94D049BB133111EB;  z ^= z >> 31

Value recipes (all integer decisions are made on the top 53 bits
v = draw >> 11, so host and device agree bit for bit):
  * ternary codes with P(0)=p0, P(+1)=P(-1)=(1-p0)/2: 0 if v < t0,
    +1 if v < t1, else -1, with t0 = floor(p0 2^53), t1 = t0 + floor((1-p0)/2 2^53);
  * uniform int8 in [lo, hi]: lo + v mod (hi-lo+1);
  * U(a,b) fp32: a + (b-a) * v 2^-53 in fp64, rounded to fp32;
  * N(0, sigma) bf16: Box-Muller on the draws (2i, 2i+1) in fp64, times sigma,
    rounded to nearest-even bf16.
The bf16/fp32 values are produced on the host only and copied to the device;
the ternary codes additionally have a device implementation (integer ops only)
because a 24-layer stack holds 19.3e9 of them.
"""
from __future__ import annotations

from fractions import Fraction

import math

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
C1 = 0xBF58476D1CE4E5B9
C2 = 0x94D049BB133111EB
M64 = (1 << 64) - 1

# tensor kinds used to derive per-tensor seeds
KIND_GATE, KIND_UP, KIND_DOWN = 1, 2, 3
KIND_GATE_SCALE, KIND_UP_SCALE, KIND_DOWN_SCALE = 4, 5, 6
KIND_ROUTER, KIND_X, KIND_W, KIND_S, KIND_XQ = 7, 8, 9, 10, 11

BASE_SEED = 0x7E47A000  # + workload id


def mix64_int(z: int) -> int:
    z &= M64
    z ^= z >> 30
    z = (z * C1) & M64
    z ^= z >> 27
    z = (z * C2) & M64
    z ^= z >> 31
    return z


def derive(seed: int, *keys: int) -> int:
    """Sub-seed for a tensor: fold each key through one counter draw."""
    s = seed & M64
    for k in keys:
        s = mix64_int(s + (int(k) + 1) * GAMMA)
    return s


def u64(seed: int, offset: int, n: int) -> np.ndarray:
    """draw(seed, offset .. offset+n-1) as uint64."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(seed & M64) + i * np.uint64(GAMMA)
        z ^= z >> np.uint64(30)
        z *= np.uint64(C1)
        z ^= z >> np.uint64(27)
        z *= np.uint64(C2)
        z ^= z >> np.uint64(31)
    return z


def top53(seed: int, offset: int, n: int) -> np.ndarray:
    return (u64(seed, offset, n) >> np.uint64(11)).astype(np.int64)


def _thresholds(p0) -> tuple[int, int]:
    p0 = Fraction(p0)
    t0 = (p0 * (1 << 53)).__floor__()
    t1 = t0 + (((1 - p0) / 2) * (1 << 53)).__floor__()
    return int(t0), int(t1)


def ternary_codes(seed: int, offset: int, n: int, p0) -> np.ndarray:
    """int8 values in {-1,0,+1}; p0 is a Fraction-compatible probability of 0."""
    t0, t1 = _thresholds(p0)
    v = top53(seed, offset, n)
    out = np.full(n, -1, dtype=np.int8)
    out[v < t1] = 1
    out[v < t0] = 0
    return out


def int8_uniform(seed: int, offset: int, n: int, lo: int = -127, hi: int = 127) -> np.ndarray:
    v = top53(seed, offset, n)
    return (lo + v % (hi - lo + 1)).astype(np.int8)


def uniform01(seed: int, offset: int, n: int) -> np.ndarray:
    return top53(seed, offset, n).astype(np.float64) * (2.0 ** -53)


def uniform_f32(seed: int, offset: int, n: int, a: float, b: float) -> np.ndarray:
    return (a + (b - a) * uniform01(seed, offset, n)).astype(np.float32)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 to the nearest bf16 (ties to even), returned as uint16 bits.

    Finite inputs only (the generators never produce inf/nan)."""
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    sign = (b >> np.uint64(63)).astype(np.uint64)
    a = np.abs(np.asarray(x, dtype=np.float64))
    # scale into the bf16 grid: bf16 has 8 significant bits; for a normal value
    # with exponent e the grid step is 2^(e-7); below 2^-126 the step is 2^-133.
    e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    # guard against log2 rounding at binade edges
    e = np.where(np.ldexp(1.0, e) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, e + 1) <= a, e + 1, e)
    e = np.maximum(e, -126)
    step_exp = e - 7
    q = np.rint(np.ldexp(a, -step_exp))  # exact scaling, then ties-to-even
    r = np.ldexp(q, step_exp)
    r32 = r.astype(np.float32)  # exact: r has <= 9 significant bits
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(a > 0, bits, np.uint16(0)).astype(np.uint16)
    return (bits | (sign.astype(np.uint16) << np.uint16(15))).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, offset: int, n: int, sigma: float) -> np.ndarray:
    """N(0, sigma^2) rounded to bf16 (uint16 bits); element i uses draws 2i, 2i+1."""
    u1 = uniform01(seed, 2 * offset, 2 * n)
    u2 = u1[1::2]
    u1 = u1[0::2]
    z = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)
    return f64_to_bf16_bits(sigma * z)


# ---------------------------------------------------------------------------
# device variant of the ternary code generator (torch int64 ops, plumbing only)
# ---------------------------------------------------------------------------

def _signed(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def ternary_codes_torch(seed: int, offset: int, n: int, p0, device, chunk: int = 1 << 26):
    """Same values as ternary_codes(), computed with torch int64 ops on `device`.

    Wrapping int64 multiplies and masked arithmetic shifts reproduce the
    uint64 recipe exactly.  Returns an int8 tensor of length n."""
    import torch

    t0, t1 = _thresholds(p0)
    out = torch.empty(n, dtype=torch.int8, device=device)
    g = _signed(GAMMA)
    c1 = _signed(C1)
    c2 = _signed(C2)
    s = _signed(seed & M64)

    def lsr(z, k):
        return (z >> k) & ((1 << (64 - k)) - 1)

    for start in range(0, n, chunk):
        m = min(chunk, n - start)
        i = torch.arange(offset + start + 1, offset + start + m + 1, dtype=torch.int64, device=device)
        z = i * g + s
        z = z ^ lsr(z, 30)
        z = z * c1
        z = z ^ lsr(z, 27)
        z = z * c2
        z = z ^ lsr(z, 31)
        v = lsr(z, 11)
        o = torch.full((m,), -1, dtype=torch.int8, device=device)
        o[v < t1] = 1
        o[v < t0] = 0
        out[start:start + m] = o
    return out


def normal_bf16_torch(seed: int, offset: int, n: int, sigma: float, device, chunk: int = 1 << 25):
    """N(0, sigma^2) as bf16 bits (int16 tensor of length n) on `device`: the draws of
    normal_bf16() (same SplitMix64 stream, same Box-Muller pairing) with the transcendental
    functions evaluated by torch on the device, rounded fp64 -> fp32 -> bf16 (nearest, ties to
    even each time).  The values follow the same distribution as normal_bf16() but need not
    match it bit for bit: tests hand the device values themselves to the oracle."""
    import torch

    out = torch.empty(n, dtype=torch.int16, device=device)
    g = _signed(GAMMA)
    c1 = _signed(C1)
    c2 = _signed(C2)
    s = _signed(seed & M64)

    def lsr(z, k):
        return (z >> k) & ((1 << (64 - k)) - 1)

    def draws(first, m):
        i = torch.arange(first + 1, first + m + 1, dtype=torch.int64, device=device)
        z = i * g + s
        z = z ^ lsr(z, 30)
        z = z * c1
        z = z ^ lsr(z, 27)
        z = z * c2
        z = z ^ lsr(z, 31)
        return lsr(z, 11).to(torch.float64) * (2.0 ** -53)

    for start in range(0, n, chunk):
        m = min(chunk, n - start)
        u = draws(2 * (offset + start), 2 * m)
        u1, u2 = u[0::2], u[1::2]
        z = torch.sqrt(-2.0 * torch.log1p(-u1)) * torch.cos(2.0 * math.pi * u2) * sigma
        out[start:start + m] = z.to(torch.float32).to(torch.bfloat16).view(torch.int16)
    return out


def head_shape():
    """The approximate head's workload: a 151,936-token vocabulary in 4,748 clusters of 32
    tokens, hidden size 2,048, the top 512 clusters kept."""
    return {"V": 151936, "d": 2048, "n_clusters": 4748, "cluster_size": 32, "top_c": 512}


# ---------------------------------------------------------------------------
# workload recipes (shapes, distributions and seeds of the five workloads)
# ---------------------------------------------------------------------------

P0_UNIFORM = Fraction(1, 3)     # codes i.i.d. uniform over {-1,0,+1}
P0_SPARSE = Fraction(2, 5)      # P(0)=0.4, P(+1)=P(-1)=0.3

GEMV_SWEEP = [(512, 2048), (2048, 512), (4096, 2048), (2048, 8192), (16384, 2048)]


def gemv_int8_case(M=256, K=512, wid=1):
    """Single ternary GEMV with int8 activations (the 256x512 workload)."""
    base = BASE_SEED + wid
    w = ternary_codes(derive(base, KIND_W), 0, M * K, P0_UNIFORM).reshape(M, K)
    s = uniform_f32(derive(base, KIND_S), 0, M, 0.5, 1.5)
    x = int8_uniform(derive(base, KIND_XQ), 0, K)
    return w, s, x


def gemv_bf16_case(M, K, wid=2, T=1):
    """Ternary GEMV with bf16 activations N(0,1) (the shape sweep)."""
    base = derive(BASE_SEED + wid, M, K)
    w = ternary_codes(derive(base, KIND_W), 0, M * K, P0_SPARSE).reshape(M, K)
    s = uniform_f32(derive(base, KIND_S), 0, M, 0.01, 0.05)
    x = normal_bf16(derive(base, KIND_X), 0, T * K, 1.0).reshape(T, K)
    return w, s, x


class MoEShape:
    def __init__(self, d=2048, f=512, E=256, k=8):
        self.d, self.f, self.E, self.k = d, f, E, k


def layer_seed(wid: int, layer: int) -> int:
    return derive(BASE_SEED + wid, 1000 + layer)


def expert_codes(wid: int, layer: int, shape: MoEShape, e: int):
    """Host codes of one expert: gate [f,d], up [f,d], down [d,f] (int8)."""
    ls = layer_seed(wid, layer)
    d, f = shape.d, shape.f
    g = ternary_codes(derive(ls, KIND_GATE), e * f * d, f * d, P0_SPARSE).reshape(f, d)
    u = ternary_codes(derive(ls, KIND_UP), e * f * d, f * d, P0_SPARSE).reshape(f, d)
    dn = ternary_codes(derive(ls, KIND_DOWN), e * d * f, d * f, P0_SPARSE).reshape(d, f)
    return g, u, dn


def layer_scales(wid: int, layer: int, shape: MoEShape):
    """fp32 per-row scales U(0.01,0.05): gate [E,f], up [E,f], down [E,d]."""
    ls = layer_seed(wid, layer)
    E, d, f = shape.E, shape.d, shape.f
    sg = uniform_f32(derive(ls, KIND_GATE_SCALE), 0, E * f, 0.01, 0.05).reshape(E, f)
    su = uniform_f32(derive(ls, KIND_UP_SCALE), 0, E * f, 0.01, 0.05).reshape(E, f)
    sd = uniform_f32(derive(ls, KIND_DOWN_SCALE), 0, E * d, 0.01, 0.05).reshape(E, d)
    return sg, su, sd


def layer_router(wid: int, layer: int, shape: MoEShape):
    """bf16 router W_g [E,d] ~ N(0, 0.02^2) as uint16 bits."""
    ls = layer_seed(wid, layer)
    return normal_bf16(derive(ls, KIND_ROUTER), 0, shape.E * shape.d, 0.02).reshape(shape.E, shape.d)


def layer_all_codes(wid: int, layer: int, shape: MoEShape):
    """Host codes of every expert of a layer (only for small E)."""
    ls = layer_seed(wid, layer)
    E, d, f = shape.E, shape.d, shape.f
    g = ternary_codes(derive(ls, KIND_GATE), 0, E * f * d, P0_SPARSE).reshape(E, f, d)
    u = ternary_codes(derive(ls, KIND_UP), 0, E * f * d, P0_SPARSE).reshape(E, f, d)
    dn = ternary_codes(derive(ls, KIND_DOWN), 0, E * d * f, P0_SPARSE).reshape(E, d, f)
    return g, u, dn


def layer_codes_torch(wid: int, layer: int, shape: MoEShape, device):
    """Device codes of every expert of a layer (int8 tensors [E,f,d],[E,f,d],[E,d,f])."""
    ls = layer_seed(wid, layer)
    E, d, f = shape.E, shape.d, shape.f
    g = ternary_codes_torch(derive(ls, KIND_GATE), 0, E * f * d, P0_SPARSE, device).view(E, f, d)
    u = ternary_codes_torch(derive(ls, KIND_UP), 0, E * f * d, P0_SPARSE, device).view(E, f, d)
    dn = ternary_codes_torch(derive(ls, KIND_DOWN), 0, E * d * f, P0_SPARSE, device).view(E, d, f)
    return g, u, dn


def tokens_bf16(wid: int, step: int, T: int, d: int):
    """Decode-step inputs x [T,d] ~ N(0,1) as bf16 bits."""
    return normal_bf16(derive(BASE_SEED + wid, KIND_X, step), 0, T * d, 1.0).reshape(T, d)
