"""The seeded input generators: reference values of SplitMix64, host/torch agreement
and the stated value distributions."""
import numpy as np
import torch

import synth


def test_splitmix64_reference_values():
    # first outputs of Vigna's splitmix64.c seeded with 0 (x += gamma; then mix)
    ref = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert synth.u64(0, 0, 3).tolist() == ref
    assert [synth.mix64_int((i + 1) * synth.GAMMA) for i in range(3)] == ref


def test_torch_codes_equal_numpy_codes():
    for p0 in (synth.P0_SPARSE, synth.P0_UNIFORM):
        a = synth.ternary_codes(0xABCDEF, 12345, 100000, p0)
        b = synth.ternary_codes_torch(0xABCDEF, 12345, 100000, p0, "cpu", chunk=30000).numpy()
        assert (a == b).all()


def test_code_distribution():
    c = synth.ternary_codes(5, 0, 1 << 20, synth.P0_SPARSE)
    frac = np.bincount(c.astype(np.int64) + 1, minlength=3) / c.size
    assert abs(frac[1] - 0.4) < 0.003 and abs(frac[0] - 0.3) < 0.003 and abs(frac[2] - 0.3) < 0.003


def test_slices_are_consistent():
    full = synth.ternary_codes(77, 0, 5000, synth.P0_SPARSE)
    part = synth.ternary_codes(77, 1234, 100, synth.P0_SPARSE)
    assert (full[1234:1334] == part).all()
    shape = synth.MoEShape(d=64, f=32, E=4)
    g, u, dn = synth.layer_all_codes(9, 2, shape)
    g2, u2, dn2 = synth.expert_codes(9, 2, shape, 3)
    assert (g[3] == g2).all() and (u[3] == u2).all() and (dn[3] == dn2).all()


def test_normal_bf16_and_rounding():
    x = synth.bf16_bits_to_f64(synth.normal_bf16(3, 0, 1 << 16, 1.0))
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02
    v = (synth.uniform01(4, 0, 10000) - 0.5) * 100
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert (synth.f64_to_bf16_bits(v32.astype(np.float64)) == ref).all()


def test_device_normal_generator_matches_host_on_cpu():
    """The torch variant draws the same SplitMix64 stream with the same Box-Muller pairing;
    evaluated on the CPU it reproduces the host generator bit for bit (the device may differ
    in the last ulp of its transcendental functions, so GPU tests hand its values on)."""
    import torch

    t = synth.normal_bf16_torch(77, 5, 4099, 0.02, "cpu", chunk=1000)
    h = synth.normal_bf16(77, 5, 4099, 0.02)
    assert (t.numpy().view(np.uint16) == h).all()
    assert t.dtype == torch.int16
