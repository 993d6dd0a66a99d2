"""Base-3 packed format (five ternary weights per byte) on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_moe_b200 as tm
from gpu_cases import dev_u16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(1, 5), (3, 7), (256, 512), (33, 2048), (5, 16384), (77, 1000)])
def test_pack5_unpack5_bit_exact(cuda_dev, M, K):
    w = synth.ternary_codes(M * 11 + K, 0, M * K, synth.P0_UNIFORM).reshape(M, K)
    ref, bad = oracle.pack5(w)
    assert bad == 0
    got = tm.tern5_pack(torch.from_numpy(w).to(cuda_dev))
    assert torch.equal(got.cpu(), torch.from_numpy(ref))
    back = tm.tern5_unpack(got, K)
    assert torch.equal(back.cpu(), torch.from_numpy(w))


def test_pack5_and_unpack5_report_bad_values(cuda_dev):
    w = torch.zeros((2, 10), dtype=torch.int8, device=cuda_dev)
    w[1, 3] = 2
    with pytest.raises(tm.TernError):
        tm.tern5_pack(w)
    p = torch.zeros((1, 16), dtype=torch.uint8, device=cuda_dev)
    p[0, 1] = 250
    with pytest.raises(tm.TernError):
        tm.tern5_unpack(p, 10)


@pytest.mark.parametrize("M,K,T", [(256, 512, 3), (77, 2048, 2), (130, 1000, 1), (33, 16384, 2), (1000, 2048, 5),
                                   (5003, 8192, 1)])
def test_gemv5_int8_bit_exact(cuda_dev, M, K, T):
    w = synth.ternary_codes(M + 3 * K, 0, M * K, synth.P0_SPARSE).reshape(M, K)
    s = synth.uniform_f32(M + 7, 0, M, 0.01, 0.05)
    q = synth.int8_uniform(K + 9, 0, T * K).reshape(T, K)
    xs = synth.uniform_f32(K + 11, 0, T, 0.001, 0.01)
    W5, _ = oracle.pack5(w)
    acc_ref, y_ref = oracle.gemv5_i8(W5, s, q, x_scale=xs)
    acc = torch.empty((T, M), dtype=torch.int32, device=cuda_dev)
    y = tm.tern5_gemv(torch.from_numpy(W5).to(cuda_dev), torch.from_numpy(s).to(cuda_dev),
                      torch.from_numpy(q).to(cuda_dev), K, act=tm.TERN_ACT_INT8,
                      x_scale=torch.from_numpy(xs).to(cuda_dev), acc=acc)
    assert (acc.cpu().numpy() == acc_ref).all()
    assert (y.cpu().numpy() == y_ref).all()


@pytest.mark.parametrize("M,K", list(synth.GEMV_SWEEP) + [(100, 1000)])
def test_gemv5_bf16_tolerance_and_same_as_two_bit(cuda_dev, M, K):
    w, s, x = synth.gemv_bf16_case(M, K)
    W5, _ = oracle.pack5(w)
    y_ref, bad = oracle.gemv5_bf16(W5, s, x)
    assert bad == 0
    sd = torch.from_numpy(s).to(cuda_dev)
    y5 = tm.tern5_gemv(torch.from_numpy(W5).to(cuda_dev), sd, dev_u16(x, cuda_dev), K)
    yg = y5.cpu().numpy().astype(np.float64)
    xn = np.linalg.norm(synth.bf16_bits_to_f64(x))
    assert np.linalg.norm(yg - y_ref) <= 1e-5 * np.linalg.norm(y_ref)
    assert np.abs(yg - y_ref).max() <= 1e-4 * xn
    if K % 64 == 0:
        # the same integer sums as the four-codes-per-byte GEMV, hence the same fp32 outputs
        y2 = tm.tern_gemv(torch.from_numpy(oracle.pack(w)[0]).to(cuda_dev), sd, dev_u16(x, cuda_dev))
        assert torch.equal(y5, y2)
