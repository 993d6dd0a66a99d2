"""Pins for the CPU oracle: values it must reproduce that come from somewhere other
than the oracle itself -- figures the pages print, hand-derived bytes, closed forms,
exact rational arithmetic, brute force on tiny inputs and library routines on
special cases.  Runs on CPU only."""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(vals):
    return synth.f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


def _bf16f(bits):
    return synth.bf16_bits_to_f64(bits)


# ----------------------------------------------------------------- format

def test_pack_golden_bytes():
    rows = []
    with open(os.path.join(GOLD, "format_bytes.txt")) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            *w, b = line.split()
            rows.append(([int(v) for v in w], int(b, 16)))
    w = np.array([r[0] for r in rows], dtype=np.int8)
    p, bad = oracle.pack(w)
    assert bad == 0
    assert [int(v) for v in p[:, 0]] == [r[1] for r in rows]


def test_pack_roundtrip_all_81_quads():
    quads = np.array(list(itertools.product([-1, 0, 1], repeat=4)), dtype=np.int8)
    p, bad = oracle.pack(quads)
    assert bad == 0
    assert len(set(p[:, 0].tolist())) == 81
    # code 11 never produced
    for b in p[:, 0]:
        for j in range(4):
            assert (int(b) >> (2 * j)) & 3 != 3
    w, bad = oracle.unpack(p, 4)
    assert bad == 0
    assert (w == quads).all()


def test_pack_rejects_out_of_range_and_unpack_reports_code11():
    w = np.array([[0, 2, 1, -2]], dtype=np.int8)
    _, bad = oracle.pack(w)
    assert bad == 2
    w2, bad2 = oracle.unpack(np.array([[0xFF, 0x03]], dtype=np.uint8), 8)
    assert bad2 == 5
    assert (w2 == 0).all()


def test_packed_size_is_quarter():
    w = synth.ternary_codes(7, 0, 512 * 2048, synth.P0_SPARSE).reshape(512, 2048)
    p, _ = oracle.pack(w)
    assert p.nbytes == 512 * 2048 // 4 == 262144


# ---------------------------------------------------- ternary dot products

@pytest.mark.parametrize("K", [4, 8])
def test_dot_bruteforce_every_ternary_row(K):
    """All 3^K ternary rows against random int8 x: the oracle equals an integer
    matmul of the dense matrix and the pages' identity sum(+1) - sum(-1)."""
    rows = np.array(list(itertools.product([-1, 0, 1], repeat=K)), dtype=np.int8)
    x = synth.int8_uniform(123, 0, K)
    p, _ = oracle.pack(rows)
    acc, _ = oracle.gemv_i8(p, np.ones(len(rows), np.float32), x)
    dense = rows.astype(np.int64) @ x.astype(np.int64)
    ident = np.array([x[r == 1].astype(np.int64).sum() - x[r == -1].astype(np.int64).sum() for r in rows])
    assert (acc[0] == dense).all()
    assert (acc[0] == ident).all()


def test_dot_special_cases_int8():
    M, K = 4, 64
    x = synth.int8_uniform(5, 0, K)
    s = np.array([1.0, 0.5, 2.0, 0.75], np.float32)
    # all +1 -> s * sum(x); all 0 -> 0
    w = np.zeros((M, K), np.int8)
    w[0] = 1
    w[2] = -1
    p, _ = oracle.pack(w)
    acc, y = oracle.gemv_i8(p, s, x)
    sx = int(x.astype(np.int64).sum())
    assert acc[0, 0] == sx and acc[0, 1] == 0 and acc[0, 2] == -sx and acc[0, 3] == 0
    assert y[0, 0] == np.float32(sx) * s[0]
    # x = e_k picks column k
    wr = synth.ternary_codes(9, 0, M * K, synth.P0_UNIFORM).reshape(M, K)
    pr, _ = oracle.pack(wr)
    for kk in (0, 17, 63):
        e = np.zeros(K, np.int8)
        e[kk] = 1
        acc, _ = oracle.gemv_i8(pr, s, e)
        assert (acc[0] == wr[:, kk]).all()
    # w -> -w negates
    pn, _ = oracle.pack(-wr)
    a1, _ = oracle.gemv_i8(pr, s, x)
    a2, _ = oracle.gemv_i8(pn, s, x)
    assert (a1 == -a2).all()


def test_gemv_int8_256x512_matches_integer_matmul():
    w, s, x = synth.gemv_int8_case()
    p, _ = oracle.pack(w)
    acc, y = oracle.gemv_i8(p, s, x)
    ref = w.astype(np.int64) @ x.astype(np.int64)
    assert (acc[0] == ref).all()
    assert np.abs(ref).max() <= 65024
    assert (y[0] == ref.astype(np.float32) * s).all()  # one fp32 rounding
    # with an activation scale: ((fp32)acc * s) * s_x, left to right
    acc2, y2 = oracle.gemv_i8(p, s, x, x_scale=np.float32(0.37))
    assert (y2[0] == (ref.astype(np.float32) * s) * np.float32(0.37)).all()


def test_gemv_bf16_exact_against_fractions():
    M, K = 6, 128
    w = synth.ternary_codes(11, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = synth.uniform_f32(12, 0, M, 0.01, 0.05)
    x = synth.normal_bf16(13, 0, K, 1.0)
    p, _ = oracle.pack(w)
    y, bad = oracle.gemv_bf16(p, s, x)
    assert bad == 0
    xf = [Fraction(v) for v in _bf16f(x)]
    for m in range(M):
        exact = sum((Fraction(int(w[m, k])) * xf[k] for k in range(K)), Fraction(0))
        assert y[0, m] == float(exact) * float(s[m])


@pytest.mark.parametrize("M,K", synth.GEMV_SWEEP[:3])
def test_gemv_bf16_sweep_equals_float64_matmul(M, K):
    """Every partial sum is exact, so any summation order -- here a BLAS
    matmul of the dense matrix -- gives the oracle's value bit for bit."""
    w, s, x = synth.gemv_bf16_case(M, K)
    p, _ = oracle.pack(w)
    y, bad = oracle.gemv_bf16(p, s, x)
    assert bad == 0
    ref = (w.astype(np.float64) @ _bf16f(x[0])) * s.astype(np.float64)
    assert np.array_equal(y[0], ref)


# ------------------------------------------------------------ quantisation

def test_quant_absmax_hand_values():
    q, s = oracle.quant_absmax(np.array([1.0, -2.0, 0.5, 0.0], np.float32))
    # inv = 127/2 = 63.5: 63.5 -> 64 (tie to even), -127, 31.75 -> 32, 0
    assert q.tolist() == [64, -127, 32, 0]
    assert s == float(np.float32(2.0) / np.float32(127.0))
    # ties to even at inv = 1
    q, s = oracle.quant_absmax(np.array([127.0, 0.5, 1.5, -2.5, 126.5], np.float32))
    assert q.tolist() == [127, 0, 2, -2, 126]
    assert s == 1.0
    q, s = oracle.quant_absmax(np.zeros(8, np.float32))
    assert (q == 0).all() and s == 0.0


def test_quant_absmax_matches_numpy_fp32():
    x = _bf16f(synth.normal_bf16(21, 0, 2048, 1.0)).astype(np.float32)
    q, s = oracle.quant_absmax(x)
    amax = np.abs(x).max()
    inv = np.float32(127.0) / amax
    ref = np.clip(np.rint(x * inv), -127, 127).astype(np.int8)
    assert (q == ref).all()
    assert s == float(amax / np.float32(127.0))


# ----------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_forms():
    d = 64
    # constant vector, eps = 0: exactly +-1
    n, bad = oracle.rmsnorm(_bf16(np.full(d, 3.25)), eps=0.0)
    assert bad == 0 and (n[0] == 0x3F80).all()
    n, _ = oracle.rmsnorm(_bf16(np.full(d, -0.375)), eps=0.0)
    assert (n[0] == 0xBF80).all()
    # one-hot a*e_0 with d = 4: n_0 = sqrt(4) = 2 exactly
    n, _ = oracle.rmsnorm(_bf16([5.0, 0, 0, 0]), eps=0.0)
    assert _bf16f(n[0]).tolist() == [2.0, 0.0, 0.0, 0.0]
    # zero vector with eps > 0 -> zeros
    n, _ = oracle.rmsnorm(_bf16(np.zeros(d)), eps=1e-6)
    assert (n[0] == 0).all()
    # eps inside the root: constant c with mean c^2 + eps a perfect square
    n, _ = oracle.rmsnorm(_bf16(np.full(d, 1.0)), eps=3.0)       # 1 / sqrt(1 + 3) = 0.5
    assert (n[0] == 0x3F00).all()
    n, _ = oracle.rmsnorm(_bf16(np.full(d, -2.0)), eps=12.0)     # -2 / sqrt(4 + 12) = -0.5
    assert (n[0] == 0xBF00).all()
    # scale invariance under x -> 2x (eps = 0) is exact
    x = synth.normal_bf16(31, 0, 2048, 1.0)
    n1, _ = oracle.rmsnorm(x, eps=0.0)
    n2, _ = oracle.rmsnorm(_bf16(2.0 * _bf16f(x)), eps=0.0)
    assert (n1 == n2).all()


def test_rmsnorm_matches_fraction_bound():
    x = synth.normal_bf16(32, 0, 2048, 1.0)
    eps = 1e-6
    n, bad = oracle.rmsnorm(x, eps)
    assert bad == 0
    xf = _bf16f(x)
    ss = sum(Fraction(v) * Fraction(v) for v in xf)
    r = math.sqrt(float(ss / 2048) + eps)
    # each output is the nearest bf16 of x/r: within half a bf16 ulp of the real quotient
    for k in range(0, 2048, 97):
        q = xf[k] / r
        got = _bf16f(n[0, k:k + 1])[0]
        ulp = 2.0 ** (math.floor(math.log2(abs(q))) - 7) if q != 0 else 0
        assert abs(got - q) <= 0.5 * ulp + 1e-300


# ------------------------------------------------------------------ router

def test_route_zero_router_ties_to_lower_index():
    Wg = np.zeros((256, 2048), np.uint16)
    x = synth.normal_bf16(41, 0, 2048, 1.0)
    logits, idx, gates, bad = oracle.route(Wg, x, 8)
    assert (logits == 0).all()
    assert idx[0].tolist() == list(range(8))
    assert (gates[0] == 0.125).all()


def test_route_one_hot_rows_closed_form():
    E, d, k = 16, 16, 4
    Wg = np.zeros((E, d), np.float64)
    for e in range(E):
        Wg[e, e] = 1.0
    x = np.arange(d, dtype=np.float64)  # logit_e = e
    logits, idx, gates, _ = oracle.route(_bf16(Wg), _bf16(x), k)
    assert logits[0].tolist() == [float(e) for e in range(E)]
    assert idx[0].tolist() == [15, 14, 13, 12]
    z = sum(math.exp(-i) for i in range(k))
    for i in range(k):
        assert abs(gates[0, i] - math.exp(-i) / z) <= 1e-16
    # duplicated best rows: ties resolved toward the lower index
    Wg2 = Wg.copy()
    Wg2[3] = Wg2[15]
    Wg2[5] = Wg2[15]
    _, idx2, g2, _ = oracle.route(_bf16(Wg2), _bf16(x), k)
    assert idx2[0].tolist() == [3, 5, 15, 14]
    assert g2[0, 0] == g2[0, 1] == g2[0, 2]


def test_route_bruteforce_exact_topk():
    E, d, k, T = 16, 64, 4, 5
    Wg = synth.normal_bf16(51, 0, E * d, 0.02).reshape(E, d)
    x = synth.normal_bf16(52, 0, T * d, 1.0).reshape(T, d)
    logits, idx, gates, bad = oracle.route(Wg, x, k)
    assert bad == 0
    Wf = [[Fraction(v) for v in row] for row in _bf16f(Wg)]
    for t in range(T):
        xf = [Fraction(v) for v in _bf16f(x[t])]
        ex = [sum((a * b for a, b in zip(Wf[e], xf)), Fraction(0)) for e in range(E)]
        assert [float(v) for v in ex] == logits[t].tolist()
        order = sorted(range(E), key=lambda e: (-ex[e], e))[:k]
        assert idx[t].tolist() == order
        # renormalised gates = softmax over all experts restricted to the top-k
        from scipy.special import softmax

        p = softmax(logits[t])
        ref = p[order] / p[order].sum()
        assert np.allclose(gates[t], ref, rtol=1e-14, atol=0)


def test_route_invariants_full_size():
    Wg = synth.layer_router(3, 0, synth.MoEShape())
    x = synth.tokens_bf16(3, 0, 4, 2048)
    logits, idx, gates, bad = oracle.route(Wg, x, 8)
    assert bad == 0
    for t in range(4):
        sel = idx[t]
        assert len(set(sel.tolist())) == 8 and sel.min() >= 0 and sel.max() < 256
        l = logits[t]
        assert all(l[sel[i]] >= l[sel[i + 1]] for i in range(7))
        rest = np.setdiff1d(np.arange(256), sel)
        assert l[sel].min() >= l[rest].max()
        assert abs(gates[t].sum() - 1.0) <= 1e-15


# ------------------------------------------------------------- MoE FFN layer

def _small_layer(E=8, d=128, f=64, k=4, seed=61, zero_up=False):
    g = synth.ternary_codes(seed, 0, E * f * d, synth.P0_SPARSE).reshape(E, f, d)
    u = synth.ternary_codes(seed + 1, 0, E * f * d, synth.P0_SPARSE).reshape(E, f, d)
    if zero_up:
        u = np.zeros_like(u)
    dn = synth.ternary_codes(seed + 2, 0, E * d * f, synth.P0_SPARSE).reshape(E, d, f)
    sg = synth.uniform_f32(seed + 3, 0, E * f, 0.01, 0.05).reshape(E, f)
    su = synth.uniform_f32(seed + 4, 0, E * f, 0.01, 0.05).reshape(E, f)
    sd = synth.uniform_f32(seed + 5, 0, E * d, 0.01, 0.05).reshape(E, d)
    Wg = synth.normal_bf16(seed + 6, 0, E * d, 0.02).reshape(E, d)
    gp, up, dp = oracle.pack_layer_codes(g, u, dn)
    L = oracle.Layer(gp, up, dp, sg, su, sd, Wg, k=k)
    return L, (g, u, dn, sg, su, sd, Wg)


def test_moe_ffn_matches_dense_numpy_composition():
    L, (g, u, dn, sg, su, sd, Wg) = _small_layer()
    x = synth.normal_bf16(70, 0, 3 * L.d, 1.0).reshape(3, L.d)
    out = oracle.moe_ffn(L, x, oracle.ACT_BF16)
    assert out["inexact"] == 0
    for t in range(3):
        xf = _bf16f(x[t])
        y = np.zeros(L.d)
        for i, e in enumerate(out["idx"][t]):
            gv = (g[e].astype(np.float64) @ xf) * sg[e].astype(np.float64)
            uv = (u[e].astype(np.float64) @ xf) * su[e].astype(np.float64)
            h = (gv / (1.0 + np.exp(-gv)) * uv).astype(np.float32)
            assert np.allclose(out["h"][t, i], h, rtol=2e-7, atol=0)
            ye = (dn[e].astype(np.float64) @ h.astype(np.float64)) * sd[e].astype(np.float64)
            y += out["gates"][t, i] * ye
        assert np.allclose(out["y64"][t], y, rtol=1e-6, atol=1e-9)


def test_moe_ffn_single_expert_and_zero_up():
    L, _ = _small_layer(k=1)
    x = synth.normal_bf16(71, 0, L.d, 1.0)
    out = oracle.moe_ffn(L, x)
    assert out["gates"][0, 0] == 1.0
    assert np.array_equal(out["y64"][0], out["ye"][0, 0])
    L0, _ = _small_layer(zero_up=True)
    out0 = oracle.moe_ffn(L0, x)
    assert (out0["h"] == 0).all() and (out0["y64"] == 0).all()


def test_swiglu_at_one():
    """G row = e_0, U row = e_0, x = e_0, scales 1: h = silu(1) * 1."""
    E, d, f = 1, 64, 64
    g = np.zeros((E, f, d), np.int8)
    g[0, 0, 0] = 1
    u = g.copy()
    dn = np.zeros((E, d, f), np.int8)
    dn[0, 5, 0] = 1
    gp, up, dp = oracle.pack_layer_codes(g, u, dn)
    one = np.ones((E, f), np.float32)
    L = oracle.Layer(gp, up, dp, one, one, np.ones((E, d), np.float32), np.zeros((E, d), np.uint16), k=1)
    x = np.zeros(d)
    x[0] = 1.0
    out = oracle.moe_ffn(L, _bf16(x))
    silu1 = 1.0 / (1.0 + math.exp(-1.0))  # 0.7310585786300049
    assert out["h"][0, 0, 0] == np.float32(silu1)
    assert out["y64"][0, 5] == float(np.float32(silu1))
    assert np.count_nonzero(out["y64"]) == 1


def test_moe_ffn_int8_accumulators_match_integer_matmul():
    L, (g, u, dn, sg, su, sd, Wg) = _small_layer()
    x = synth.normal_bf16(72, 0, 2 * L.d, 1.0).reshape(2, L.d)
    out = oracle.moe_ffn(L, x, oracle.ACT_INT8)
    for t in range(2):
        x32 = _bf16f(x[t]).astype(np.float32)
        amax = np.abs(x32).max()
        qx = np.clip(np.rint(x32 * (np.float32(127.0) / amax)), -127, 127).astype(np.int64)
        assert (out["qx"][t] == qx).all()
        for i, e in enumerate(out["idx"][t]):
            assert (out["acc_g"][t, i] == g[e].astype(np.int64) @ qx).all()
            assert (out["acc_u"][t, i] == u[e].astype(np.int64) @ qx).all()
            assert (out["acc_d"][t, i] == dn[e].astype(np.int64) @ out["qh"][t, i].astype(np.int64)).all()
            # fp32 epilogue: g = ((fp32)acc_g * s_g) * s_x, u likewise, h = fp32(silu(g) * u)
            sx = np.float32(out["sx"][t])
            gv = (out["acc_g"][t, i].astype(np.float32) * sg[e]) * sx
            uv = (out["acc_u"][t, i].astype(np.float32) * su[e]) * sx
            gd, ud = gv.astype(np.float64), uv.astype(np.float64)
            h = (gd / (1.0 + np.exp(-gd)) * ud).astype(np.float32)
            assert np.allclose(out["h"][t, i], h, rtol=2e-7, atol=0)
            ye = (out["acc_d"][t, i].astype(np.float32) * sd[e]) * np.float32(out["sh"][t, i])
            assert np.array_equal(out["ye"][t, i], ye.astype(np.float64))


def test_moe_ffn_teacher_forced_down_uses_given_qh():
    L, (g, u, dn, *_ ) = _small_layer()
    x = synth.normal_bf16(73, 0, L.d, 1.0)
    out = oracle.moe_ffn(L, x, oracle.ACT_INT8)
    qh = out["qh"].copy()
    qh[0, 0, 0] = np.int8(qh[0, 0, 0] ^ 1)
    out2 = oracle.moe_ffn(L, x, oracle.ACT_INT8, qh_in=qh, sh_in=out["sh"])
    e = out["idx"][0, 0]
    assert (out2["acc_d"][0, 0] == dn[e].astype(np.int64) @ qh[0, 0].astype(np.int64)).all()


def test_stack_layer_zero_ffn_is_identity_and_residual_rounding():
    L, _ = _small_layer(zero_up=True)
    x = synth.normal_bf16(74, 0, L.d, 1.0)
    r = oracle.stack_layer(L, x, eps=1e-6)
    assert (r["x_out"] == x).all()
    L2, _ = _small_layer(seed=91)
    r2 = oracle.stack_layer(L2, x, eps=1e-6)
    n, _ = oracle.rmsnorm(x, 1e-6)
    assert (r2["n"] == n).all()
    ref = synth.f64_to_bf16_bits(_bf16f(x) + _bf16f(r2["y"][0]))
    assert (r2["x_out"][0] == ref).all()


# ------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_ties_and_library():
    assert oracle.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80         # tie -> even (down)
    assert oracle.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82     # tie -> even (up)
    assert oracle.f64_to_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -30)) == 0xBF81
    import torch

    v = (synth.uniform01(81, 0, 4096) - 0.5) * 1e3
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle.f64_to_bf16(float(a)) for a in v32], np.uint16)
    assert (got == ref).all()


# ------------------------------------------------ bytes-per-token arithmetic

def test_page_bytes_per_token_arithmetic():
    with open(os.path.join(GOLD, "page_figures.json")) as fh:
        P = {k: v["value"] for k, v in json.load(fh).items() if not k.startswith("_")}
    ms = P["bytes_per_token"] / P["peak_bandwidth_Bps"] * 1e3
    assert round(ms, 2) == P["ms_per_token_at_peak"]
    ceiling = 1e3 / ms
    assert round(ceiling) == P["tok_s_ceiling"]
    assert round(P["tok_s_measured"] / ceiling, 2) == P["fraction_of_peak"]
    assert round(P["params_total"] * P["bits_per_ternary_weight"] / 8 / 1e9, 2) == P["ideal_bytes_20B"] / 1e9
    assert P["params_total"] * 2 == P["bf16_bytes_20B"]
    # four per byte is 2 bits: 5.0 GB, not the page's 3.9 GB (the page states both)
    assert P["params_total"] / P["weights_per_byte"] == 5.0e9 != P["raw_ternary_bytes_20B_page"]


def test_synthetic_model_byte_count():
    """The per-token byte model of the synthetic 24-layer model, counted from the
    arrays the oracle's packer produces for one expert."""
    shape = synth.MoEShape()
    g, u, dn = synth.expert_codes(3, 0, shape, 0)
    gp, up, dp = oracle.pack_layer_codes(g[None], u[None], dn[None])
    packed = gp.nbytes + up.nbytes + dp.nbytes
    scales = 4 * (shape.f + shape.f + shape.d)
    router = 2 * shape.E * shape.d
    assert packed == 786432 and scales == 12288 and router == 1048576
    per_layer_token = 8 * (packed + scales) + router
    assert per_layer_token == 7438336
    assert 24 * per_layer_token == 178520064
    assert 24 * (256 * (packed + scales) + router) == 4932501504


# ------------------------------------------------ base-3 packing (five weights per byte)

def test_pack5_is_a_bijection_on_all_243_quintuples():
    """Every ternary 5-tuple packs to its own byte below 243, and unpacks back."""
    tuples = np.array(list(itertools.product((-1, 0, 1), repeat=5)), dtype=np.int8)  # [243, 5]
    p, bad = oracle.pack5(tuples)
    assert bad == 0 and p.shape == (243, 16)
    assert (p[:, 1:] == 0).all()                     # row padding to 16 bytes
    assert len(set(p[:, 0].tolist())) == 243 and p[:, 0].max() <= 242
    w, bad = oracle.unpack5(p, 5)
    assert bad == 0 and (w == tuples).all()


def test_pack5_place_values():
    """Little-endian base 3 along K with the 2-bit format's digits (0, +1 -> 1, -1 -> 2)."""
    rows = np.array([[1, 0, 0, 0, 0], [0, 0, 0, 0, -1], [1, 1, 1, 1, 1], [-1] * 5, [0] * 5,
                     [0, -1, 1, 0, 0]], dtype=np.int8)
    p, _ = oracle.pack5(rows)
    assert p[:, 0].tolist() == [1, 162, 121, 242, 0, 2 * 3 + 1 * 9]


def test_pack5_tail_density_and_bad_bytes():
    # K = 7: the second byte holds two weights, its other three digits are zero
    w = np.array([[1, -1, 0, 1, -1, -1, 1]], dtype=np.int8)
    p, _ = oracle.pack5(w)
    assert p[0, 1] == 2 + 3 * 1 and (p[0, 2:] == 0).all()
    assert (oracle.unpack5(p, 7)[0] == w).all()
    # bytes per row: ceil(K/5) rounded up to 16; 2048 weights take 416 bytes instead of 512
    assert [oracle.tern5_row_bytes(k) for k in (1, 5, 80, 81, 2048, 16384)] == [16, 16, 16, 32, 416, 3280]
    assert oracle.tern5_row_bytes(2048) / 512 == 0.8125
    # a byte that no 5-tuple produces is reported and read as five zeros
    q = np.zeros((1, 16), np.uint8)
    q[0, 0] = 250
    wq, bad = oracle.unpack5(q, 5)
    assert bad == 1 and (wq == 0).all()
    # values that are not ternary are counted
    assert oracle.pack5(np.array([[2, 0, 0, 0, 0]], np.int8))[1] == 1


def test_gemv5_equals_two_bit_gemv():
    """The base-3 GEMV computes the same dot products as the 2-bit one on the same weights."""
    w = synth.ternary_codes(41, 0, 33 * 128, synth.P0_UNIFORM).reshape(33, 128)
    s = synth.uniform_f32(42, 0, 33, 0.5, 1.5)
    q = synth.int8_uniform(43, 0, 3 * 128).reshape(3, 128)
    a5, y5 = oracle.gemv5_i8(oracle.pack5(w)[0], s, q)
    a2, y2 = oracle.gemv_i8(oracle.pack(w)[0], s, q)
    assert (a5 == a2).all() and (y5 == y2).all()
    assert (a2 == q.astype(np.int64) @ w.T.astype(np.int64)).all()


def test_openmp_build_returns_identical_results():
    """The all-cores build (same source, -fopenmp) only splits independent rows across
    threads: a full-size layer gives the same bits as the single-threaded build."""
    from gpu_cases import HostLayer

    shape = synth.MoEShape()
    H = HostLayer(5, 0, shape)
    x = synth.tokens_bf16(5, 77, 1, shape.d)
    n, _ = oracle.rmsnorm(x, 1e-6)
    _, idx, _, _ = H.route(n)
    H.fill(idx)
    for act in (oracle.ACT_BF16, oracle.ACT_INT8):
        a = oracle.stack_layer(H.oracle_layer(), x, act=act)
        b = oracle.stack_layer(H.oracle_layer(), x, act=act, omp=True)
        assert (a["x_out"] == b["x_out"]).all() and (a["y64"] == b["y64"]).all()
        assert (a["idx"] == b["idx"]).all() and (a["gates"] == b["gates"]).all()
        assert a["inexact"] == b["inexact"] == 0
