"""GPU parity of the format, the GEMV and the router against the CPU oracle, called
through the C-ABI.  Integer work is compared bit for bit; floating point within the
stated tolerance (rel-L2 <= 1e-5 and max-abs <= 1e-4 * ||x||_2 against fp64)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_moe_b200 as tm
from gpu_cases import dev_u16, host_u16

pytestmark = pytest.mark.gpu


def _rel_l2(got, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(np.asarray(got, np.float64) - ref) / max(np.linalg.norm(ref), 1e-300))


# ------------------------------------------------------------------------ format

def test_device_codes_equal_host_codes(cuda_dev):
    a = synth.ternary_codes(0x51, 777, 300001, synth.P0_SPARSE)
    b = synth.ternary_codes_torch(0x51, 777, 300001, synth.P0_SPARSE, cuda_dev).cpu().numpy()
    assert (a == b).all()


@pytest.mark.parametrize("M,K", [(1, 4), (3, 12), (256, 512), (517, 2048), (64, 8192)])
def test_pack_unpack_bit_exact(cuda_dev, M, K):
    w = synth.ternary_codes(M * 7 + K, 0, M * K, synth.P0_UNIFORM).reshape(M, K)
    ref, bad = oracle.pack(w)
    got = tm.tern_pack(torch.from_numpy(w).to(cuda_dev)).cpu().numpy()
    assert bad == 0 and (got == ref).all()
    back = tm.tern_unpack(torch.from_numpy(ref).to(cuda_dev), K).cpu().numpy()
    assert (back == w).all()


def test_pack_reports_bad_codes(cuda_dev):
    w = torch.tensor([[0, 1, 2, -1]], dtype=torch.int8, device=cuda_dev)
    with pytest.raises(tm.TernError) as ei:
        tm.tern_pack(w)
    assert ei.value.code == 3
    p = torch.tensor([[0xFF]], dtype=torch.uint8, device=cuda_dev)
    with pytest.raises(tm.TernError):
        tm.tern_unpack(p, 4)


# -------------------------------------------------------------------------- GEMV

def test_gemv_int8_256x512_bit_exact(cuda_dev):
    w, s, x = synth.gemv_int8_case()
    Wp, _ = oracle.pack(w)
    acc_ref, y_ref = oracle.gemv_i8(Wp, s, x)
    acc = torch.empty((1, 256), dtype=torch.int32, device=cuda_dev)
    y = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev),
                     torch.from_numpy(x).to(cuda_dev), act=tm.TERN_ACT_INT8, acc=acc)
    assert (acc.cpu().numpy() == acc_ref).all()
    assert (y.cpu().numpy() == y_ref).all()


@pytest.mark.parametrize("M,K,T", [(256, 512, 3), (77, 64, 2), (130, 128, 1), (33, 8192, 2), (1000, 2048, 5),
                                   (5003, 8192, 2), (77, 6144, 2), (301, 14336, 1)])
def test_gemv_int8_shapes_bit_exact(cuda_dev, M, K, T):
    w = synth.ternary_codes(M + K, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = synth.uniform_f32(M + 1, 0, M, 0.01, 0.05)
    q = synth.int8_uniform(K + 2, 0, T * K).reshape(T, K)
    xs = synth.uniform_f32(K + 3, 0, T, 0.001, 0.01)
    Wp, _ = oracle.pack(w)
    acc_ref, y_ref = oracle.gemv_i8(Wp, s, q, x_scale=xs)
    acc = torch.empty((T, M), dtype=torch.int32, device=cuda_dev)
    y = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev),
                     torch.from_numpy(q).to(cuda_dev), act=tm.TERN_ACT_INT8,
                     x_scale=torch.from_numpy(xs).to(cuda_dev), acc=acc)
    assert (acc.cpu().numpy() == acc_ref).all()
    assert (y.cpu().numpy() == y_ref).all()


@pytest.mark.parametrize("M,K", synth.GEMV_SWEEP)
def test_gemv_bf16_sweep_tolerance(cuda_dev, M, K):
    w, s, x = synth.gemv_bf16_case(M, K)
    Wp, _ = oracle.pack(w)
    y_ref, bad = oracle.gemv_bf16(Wp, s, x)
    assert bad == 0
    y = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev), dev_u16(x, cuda_dev))
    y = y.cpu().numpy().astype(np.float64)
    xn = np.linalg.norm(synth.bf16_bits_to_f64(x))
    assert _rel_l2(y, y_ref) <= 1e-5
    assert np.abs(y - y_ref).max() <= 1e-4 * xn


@pytest.mark.parametrize("M,K,T", [(100, 64, 3), (333, 1024, 2), (64, 16384, 1), (4099, 16384, 1), (50, 10240, 2)])
def test_gemv_bf16_ragged_tolerance(cuda_dev, M, K, T):
    w = synth.ternary_codes(M * 3 + K, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = synth.uniform_f32(M + 5, 0, M, 0.01, 0.05)
    x = synth.normal_bf16(K + 6, 0, T * K, 1.0).reshape(T, K)
    Wp, _ = oracle.pack(w)
    y_ref, _ = oracle.gemv_bf16(Wp, s, x)
    y = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev), dev_u16(x, cuda_dev))
    assert _rel_l2(y.cpu().numpy(), y_ref) <= 1e-5


@pytest.mark.parametrize("M,K", [(77, 64), (130, 128), (1000, 256), (333, 1024), (517, 2048), (16384, 2048),
                                 (300, 8192), (64, 16384), (40000, 2048)])
def test_gemv_lean_and_ring_kernels_agree_bit_exact(cuda_dev, M, K):
    """One token takes the lean kernel (no decode table, rows loaded straight into registers)
    when the call is small; two tokens always take the ring kernel.  Both form the same exact
    integer sums and the same epilogue, so the token's outputs (and int32 sums) must be
    identical bit for bit; the largest case here is too big for the lean kernel and checks
    the switch.  Also against the oracle (int8: bit-exact)."""
    w = synth.ternary_codes(M * 5 + K, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = synth.uniform_f32(M + 7, 0, M, 0.01, 0.05)
    Wp, _ = oracle.pack(w)
    Wd, sd = torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev)
    xb = synth.normal_bf16(K + 8, 0, K, 1.0).reshape(1, K)
    y1 = tm.tern_gemv(Wd, sd, dev_u16(xb, cuda_dev))
    y2 = tm.tern_gemv(Wd, sd, dev_u16(np.concatenate([xb, xb]), cuda_dev))
    assert torch.equal(y1[0], y2[0]) and torch.equal(y2[0], y2[1])
    q = synth.int8_uniform(K + 9, 0, K).reshape(1, K)
    xs = np.array([0.004], np.float32)
    acc1 = torch.empty((1, M), dtype=torch.int32, device=cuda_dev)
    acc2 = torch.empty((2, M), dtype=torch.int32, device=cuda_dev)
    z1 = tm.tern_gemv(Wd, sd, torch.from_numpy(q).to(cuda_dev), act=tm.TERN_ACT_INT8,
                      x_scale=torch.from_numpy(xs).to(cuda_dev), acc=acc1)
    z2 = tm.tern_gemv(Wd, sd, torch.from_numpy(np.concatenate([q, q])).to(cuda_dev), act=tm.TERN_ACT_INT8,
                      x_scale=torch.from_numpy(np.concatenate([xs, xs])).to(cuda_dev), acc=acc2)
    assert torch.equal(acc1[0], acc2[0]) and torch.equal(z1[0], z2[0])
    acc_ref, y_ref = oracle.gemv_i8(Wp, s, q, x_scale=xs)
    assert (acc1.cpu().numpy() == acc_ref).all()
    assert (z1.cpu().numpy() == y_ref).all()
    if M * K <= 4 << 20:
        y_ref, _ = oracle.gemv_bf16(Wp, s, xb)
        assert _rel_l2(y1.cpu().numpy(), y_ref) <= 1e-5


def test_gemv_bf16_zero_and_tiny_inputs(cuda_dev):
    M, K = 64, 512
    w = synth.ternary_codes(99, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = np.ones(M, np.float32)
    Wp, _ = oracle.pack(w)
    x0 = np.zeros((1, K), np.uint16)
    y0 = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev), dev_u16(x0, cuda_dev))
    assert (y0.cpu().numpy() == 0).all()
    # a vector spanning many binades: elements far below the absmax round onto the grid
    xv = synth.bf16_bits_to_f64(synth.normal_bf16(98, 0, K, 1.0)) * np.exp2(np.arange(K) % 40 - 20)
    xb = synth.f64_to_bf16_bits(xv)[None]
    y_ref, _ = oracle.gemv_bf16(Wp, s, xb)
    y = tm.tern_gemv(torch.from_numpy(Wp).to(cuda_dev), torch.from_numpy(s).to(cuda_dev), dev_u16(xb, cuda_dev))
    assert _rel_l2(y.cpu().numpy(), y_ref) <= 1e-5


def test_quant_absmax_bit_exact(cuda_dev):
    x = synth.normal_bf16(97, 0, 4 * 2048, 1.0).reshape(4, 2048)
    x[2] = 0
    q, s = tm.tern_quant_absmax(dev_u16(x, cuda_dev))
    for t in range(4):
        qr, sr = oracle.quant_absmax(synth.bf16_bits_to_f64(x[t]).astype(np.float32))
        assert (q[t].cpu().numpy() == qr).all()
        assert float(s[t]) == sr


# ------------------------------------------------------------------------ router

@pytest.mark.parametrize("T", [1, 4, 64])
def test_route_full_size_bit_exact(cuda_dev, T):
    shape = synth.MoEShape()
    Wg = synth.layer_router(3, 0, shape)
    x = synth.tokens_bf16(3, 10 + T, T, shape.d)
    lg_ref, idx_ref, g_ref, bad = oracle.route(Wg, x, 8)
    assert bad == 0
    logits = torch.empty((T, 256), dtype=torch.float64, device=cuda_dev)
    idx, g = tm.moe_route_topk(dev_u16(Wg, cuda_dev), dev_u16(x, cuda_dev), 8, logits=logits)
    assert (logits.cpu().numpy() == lg_ref).all()       # exact sums: order-independent
    assert (idx.cpu().numpy() == idx_ref).all()
    assert np.abs(g.cpu().numpy() - g_ref).max() <= 1e-7
    assert np.abs(g.cpu().numpy().astype(np.float64).sum(1) - 1.0).max() <= 1e-6


def test_route_ties_and_small_E(cuda_dev):
    Wg = np.zeros((256, 2048), np.uint16)
    x = synth.tokens_bf16(3, 1, 2, 2048)
    idx, g = tm.moe_route_topk(dev_u16(Wg, cuda_dev), dev_u16(x, cuda_dev), 8)
    assert (idx.cpu().numpy() == np.arange(8)).all()
    assert (g.cpu().numpy() == 0.125).all()
    E, d, k = 16, 64, 4
    Wg = synth.normal_bf16(51, 0, E * d, 0.02).reshape(E, d)
    x = synth.normal_bf16(52, 0, 5 * d, 1.0).reshape(5, d)
    _, idx_ref, g_ref, _ = oracle.route(Wg, x, k)
    idx, g = tm.moe_route_topk(dev_u16(Wg, cuda_dev), dev_u16(x, cuda_dev), k)
    assert (idx.cpu().numpy() == idx_ref).all()
    assert np.abs(g.cpu().numpy() - g_ref).max() <= 1e-7


def test_route_large_E(cuda_dev):
    E, d, k = 1000, 256, 8
    Wg = synth.normal_bf16(53, 0, E * d, 0.02).reshape(E, d)
    x = synth.normal_bf16(54, 0, 3 * d, 1.0).reshape(3, d)
    _, idx_ref, g_ref, _ = oracle.route(Wg, x, k)
    idx, g = tm.moe_route_topk(dev_u16(Wg, cuda_dev), dev_u16(x, cuda_dev), k)
    assert (idx.cpu().numpy() == idx_ref).all()


def test_bounded_wait_times_out_cleanly(cuda_dev):
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    assert tm.tern_stream_status() == 0
    tm.tern_test_bounded_wait(flag, 1000)
    assert tm.tern_stream_status() == 5   # TERN_ETIMEOUT, context still usable
    assert tm.tern_stream_status() == 0   # read clears it
    y = torch.ones(4, device=cuda_dev) * 2
    assert float(y.sum()) == 8.0
