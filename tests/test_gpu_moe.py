"""GPU parity of the MoE FFN layer and the residual stack against the CPU oracle.

Full-size layers: d=2048, 256 experts of SwiGLU 512x2048 / 2048x512, top-8.  The oracle
gets host copies of exactly the experts it routes to (regenerated from the same seeds).
  * routing: indices bit-exact, gates within 1e-7;
  * int8 path: gate/up/down int32 accumulators bit-exact (down teacher-forced on the
    GPU's quantised h, whose rare 1-step differences are counted), quantised input exact;
  * bf16 path: y (fp32 before the bf16 cast) within rel-L2 1e-5 and max-abs
    1e-4 * ||x||_2 of the fp64 oracle; y in bf16 within one bf16 ulp.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_moe_b200 as tm
from gpu_cases import HostLayer, dev_u16, device_layer, host_u16, ws_view

pytestmark = pytest.mark.gpu

WID_LAYER = 3
WID_STACK = 5


@pytest.fixture(scope="module")
def layer_pair(cuda_dev):
    shape = synth.MoEShape()
    dl = device_layer(WID_LAYER, 0, shape, cuda_dev)
    hl = HostLayer(WID_LAYER, 0, shape)
    return shape, dl, hl


# nearest-even bf16 as the oracle rounds (the residual's two roundings)
_oracle_bf16 = np.vectorize(oracle.f64_to_bf16, otypes=[np.uint16])


def _bf16_ulp_close(a_bits, b_bits):
    a = synth.bf16_bits_to_f64(a_bits)
    b = synth.bf16_bits_to_f64(b_bits)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 1e-30))) - 7)
    return np.abs(a - b) <= ulp * 1.0001


def _x_out_close(got_bits, ref_bits, y64):
    """x_out = bf16(x + bf16(y)) from a y within its tolerance of the oracle's y64: where
    bf16(y) matches the oracle's the result is identical; where it rounds to the neighbouring
    bf16 (y within tolerance of a rounding boundary) the sum moves by that one ulp of bf16(y)
    before its own rounding.  So each element is within one ulp of x_out plus one ulp of
    bf16(y64).  (With x and y of opposite signs and nearly equal, one ulp of y is many ulps of
    the small x_out, so a plain one-ulp check of x_out would not hold.)"""
    a = synth.bf16_bits_to_f64(got_bits)
    b = synth.bf16_bits_to_f64(ref_bits)
    ulp = lambda v: np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1e-30))) - 7)
    yb = synth.bf16_bits_to_f64(_oracle_bf16(y64))
    return np.abs(a - b) <= (ulp(b) + ulp(yb)) * 1.0001


def _check_bf16_output(y_bits, y32, ref_y64, ref_bits):
    """The GPU's bf16 output is the nearest bf16 of its own fp32-accurate value (checked
    against the fp64 oracle by the tolerance tests), so it may differ from the oracle's
    rounding only where that value sits within the tolerance of a rounding boundary:
    each element is within one bf16 ulp of the GPU's fp32 value, and at most 0.5% of the
    elements differ from the oracle's bf16 at all (each by at most one ulp, or by less than
    the fp32 tolerance)."""
    g = synth.bf16_bits_to_f64(y_bits)
    y32 = np.asarray(y32, np.float64)
    ulp32 = np.exp2(np.floor(np.log2(np.maximum(np.abs(y32), 1e-30))) - 7)
    assert (np.abs(g - y32) <= 0.5 * ulp32 * 1.0001).all()
    diff = y_bits != ref_bits
    assert diff.mean() <= 5e-3
    tol = 1e-5 * np.abs(ref_y64).max()
    r = synth.bf16_bits_to_f64(ref_bits)
    ok = _bf16_ulp_close(y_bits, ref_bits) | (np.abs(g - r) <= tol)
    assert ok.all()


def _run_layer(layer_pair, T, act, step):
    shape, dl, hl = layer_pair
    dev = dl.gate.device
    x = synth.tokens_bf16(WID_LAYER, step, T, shape.d)
    _, idx_ref, _, _ = hl.route(x)
    hl.fill(idx_ref)
    ws = tm.workspace(tm.moe_ffn_workspace_bytes(dl, T, act), dev)
    y32 = torch.empty((T, shape.d), dtype=torch.float32, device=dev)
    y = tm.moe_ffn_decode(dl, dev_u16(x, dev), act=act, ws=ws, y_f32=y32)
    torch.cuda.synchronize()
    lay = tm.moe_ffn_workspace_layout(dl, T, act)
    return x, y, y32, ws, lay


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_moe_layer_bf16(layer_pair, T):
    shape, dl, hl = layer_pair
    x, y, y32, ws, lay = _run_layer(layer_pair, T, tm.TERN_ACT_BF16, step=100 + T)
    ref = oracle.moe_ffn(hl.oracle_layer(), x, oracle.ACT_BF16)
    k = shape.k
    idx = ws_view(ws, lay["idx"], torch.int32, T * k).view(T, k).cpu().numpy()
    g64 = ws_view(ws, lay["gates64"], torch.float64, T * k).view(T, k).cpu().numpy()
    assert (idx == ref["idx"]).all()
    assert np.abs(g64 - ref["gates"]).max() <= 1e-12
    # unique experts: every selected expert grouped exactly once
    nu = int(ws_view(ws, lay["n_unique"], torch.int32, 1).cpu()[0])
    assert nu == len(np.unique(ref["idx"]))
    h = ws_view(ws, lay["h"], torch.float32, T * k * shape.f).view(T, k, shape.f).cpu().numpy()
    assert np.abs(h - ref["h"]).max() <= 1e-5 * np.abs(ref["h"]).max()
    y64 = ref["y64"]
    yg = y32.cpu().numpy().astype(np.float64)
    for t in range(T):
        xn = np.linalg.norm(synth.bf16_bits_to_f64(x[t]))
        rel = np.linalg.norm(yg[t] - y64[t]) / np.linalg.norm(y64[t])
        assert rel <= 1e-5, (t, rel)
        assert np.abs(yg[t] - y64[t]).max() <= 1e-4 * xn
    _check_bf16_output(host_u16(y), yg, y64, ref["y_bf16"])


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_moe_layer_int8_accumulators_bit_exact(layer_pair, T):
    shape, dl, hl = layer_pair
    x, y, y32, ws, lay = _run_layer(layer_pair, T, tm.TERN_ACT_INT8, step=200 + T)
    ref = oracle.moe_ffn(hl.oracle_layer(), x, oracle.ACT_INT8)
    k, f, d = shape.k, shape.f, shape.d
    idx = ws_view(ws, lay["idx"], torch.int32, T * k).view(T, k).cpu().numpy()
    assert (idx == ref["idx"]).all()
    qx = ws_view(ws, lay["qx"], torch.int8, T * d).view(T, d).cpu().numpy()
    sx = ws_view(ws, lay["sx"], torch.float32, T).cpu().numpy()
    assert (qx == ref["qx"]).all() and (sx == ref["sx"]).all()
    acc_g = ws_view(ws, lay["acc_g"], torch.int32, T * k * f).view(T, k, f).cpu().numpy()
    acc_u = ws_view(ws, lay["acc_u"], torch.int32, T * k * f).view(T, k, f).cpu().numpy()
    assert (acc_g == ref["acc_g"]).all() and (acc_u == ref["acc_u"]).all()
    # down stage teacher-forced on the GPU's own quantised h
    qh = ws_view(ws, lay["qh"], torch.int8, T * k * f).view(T, k, f).cpu().numpy()
    sh = ws_view(ws, lay["sh"], torch.float32, T * k).view(T, k).cpu().numpy()
    assert (qh != ref["qh"]).mean() <= 1e-3 and np.abs(qh.astype(int) - ref["qh"]).max() <= 1
    ref_tf = oracle.moe_ffn(hl.oracle_layer(), x, oracle.ACT_INT8, qh_in=qh, sh_in=sh)
    acc_d = ws_view(ws, lay["acc_d"], torch.int32, T * k * d).view(T, k, d).cpu().numpy()
    assert (acc_d == ref_tf["acc_d"]).all()
    yg = y32.cpu().numpy().astype(np.float64)
    assert np.abs(yg - ref_tf["y64"]).max() <= 1e-6 * np.abs(ref_tf["y64"]).max()
    _check_bf16_output(host_u16(y), yg, ref_tf["y64"], ref_tf["y_bf16"])


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_moe_layer_batch_invariance(layer_pair, act):
    """Token t's output in a batch of 64 -- the grouped int8 tensor-core (mma) kernels, taken
    from 32 tokens on -- equals its batch-1 output from the dp4a kernels, bit for bit, in both
    the fp32 pre-cast value and the bf16 output."""
    shape, dl, hl = layer_pair
    dev = dl.gate.device
    x = synth.tokens_bf16(WID_LAYER, 300, 64, shape.d)
    yb32 = torch.empty((64, shape.d), dtype=torch.float32, device=dev)
    yb = tm.moe_ffn_decode(dl, dev_u16(x, dev), act=act, y_f32=yb32)
    for t in (0, 17, 31, 63):
        y132 = torch.empty((1, shape.d), dtype=torch.float32, device=dev)
        y1 = tm.moe_ffn_decode(dl, dev_u16(x[t:t + 1], dev), act=act, y_f32=y132)
        assert torch.equal(y1.view(torch.int16), yb[t:t + 1].view(torch.int16))
        assert torch.equal(y132, yb32[t:t + 1])


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_moe_layer_grouped_multi_pass(layer_pair, act):
    """An expert with more tokens than one tensor-core pass takes with bf16 activations (20):
    50 copies of one token send 50 tokens to each of its experts (passes of 20, 20 and 10; with
    int8 activations one pass of 50 takes all); every token's output still equals its batch-1
    output bit for bit."""
    shape, dl, hl = layer_pair
    dev = dl.gate.device
    x = synth.tokens_bf16(WID_LAYER, 310, 64, shape.d)
    x[:50] = x[0]
    yb32 = torch.empty((64, shape.d), dtype=torch.float32, device=dev)
    yb = tm.moe_ffn_decode(dl, dev_u16(x, dev), act=act, y_f32=yb32)
    for t in (0, 21, 49, 50, 63):
        y132 = torch.empty((1, shape.d), dtype=torch.float32, device=dev)
        y1 = tm.moe_ffn_decode(dl, dev_u16(x[t:t + 1], dev), act=act, y_f32=y132)
        assert torch.equal(y1.view(torch.int16), yb[t:t + 1].view(torch.int16))
        assert torch.equal(y132, yb32[t:t + 1])


def test_moe_layer_repeat_is_deterministic(layer_pair):
    shape, dl, hl = layer_pair
    dev = dl.gate.device
    x = dev_u16(synth.tokens_bf16(WID_LAYER, 301, 4, shape.d), dev)
    ws = tm.workspace(tm.moe_ffn_workspace_bytes(dl, 4), dev)
    a = tm.moe_ffn_decode(dl, x, ws=ws).clone()
    b = tm.moe_ffn_decode(dl, x, ws=ws).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ------------------------------------------------------------------ residual stack

@pytest.fixture(scope="module")
def stack3(cuda_dev):
    shape = synth.MoEShape()
    layers = [device_layer(WID_STACK, l, shape, cuda_dev) for l in range(3)]
    hosts = [HostLayer(WID_STACK, l, shape) for l in range(3)]
    return shape, layers, hosts


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_stack_teacher_forced_per_layer(stack3, act):
    shape, layers, hosts = stack3
    dev = layers[0].gate.device
    x = synth.tokens_bf16(WID_STACK, 7, 1, shape.d)
    xd = dev_u16(x, dev)
    # the full stack in one call (T = 1: the persistent kernel)
    full = xd.clone()
    tm.moe_stack_decode(tm.Stack(layers), full, eps=1e-6, act=act)
    # layer by layer on the GPU, each compared with the oracle on the GPU's own input
    cur = xd.clone()
    mismatched = 0
    for l, (L, H) in enumerate(zip(layers, hosts)):
        xin = host_u16(cur)
        n, _ = oracle.rmsnorm(xin, 1e-6)
        _, idx, _, _ = H.route(n)
        H.fill(idx)
        ref = oracle.stack_layer(H.oracle_layer(), xin, eps=1e-6, act=act)
        tm.moe_stack_decode(tm.Stack([L]), cur, eps=1e-6, act=act)
        got = host_u16(cur)
        close = _x_out_close(got, ref["x_out"], ref["y64"])
        assert close.all(), (l, np.argwhere(~close)[:5])
        mismatched += int((got != ref["x_out"]).sum())
    assert mismatched <= 3 * 2048 * 5e-3
    assert torch.equal(full.view(torch.int16), cur.view(torch.int16))


def test_stack_next_layer_prediction_changes_no_value(stack3, monkeypatch):
    """With TERNMOE_PREDICT=1 the batch-1 kernel built with the next-layer prediction side task
    runs (L2 prefetches of predicted experts' rows): a hint only, so every token's output is
    the same bits as without it."""
    shape, layers, hosts = stack3
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    x = synth.tokens_bf16(WID_STACK, 9, 3, shape.d)
    for act in (tm.TERN_ACT_BF16, tm.TERN_ACT_INT8):
        for t in range(3):
            monkeypatch.delenv("TERNMOE_PREDICT", raising=False)
            plain = dev_u16(x[t:t + 1], dev)
            tm.moe_stack_decode(st, plain, act=act)
            monkeypatch.setenv("TERNMOE_PREDICT", "1")
            pred = dev_u16(x[t:t + 1], dev)
            tm.moe_stack_decode(st, pred, act=act)
            monkeypatch.delenv("TERNMOE_PREDICT", raising=False)
            assert tm.tern_stream_status() == 0
            assert torch.equal(plain.view(torch.int16), pred.view(torch.int16)), (act, t)


def test_one_launch_paths_match_stage_path_bit_exact(stack3):
    """Three ways through the same stack do the same arithmetic in the same order, so every
    token gives identical bits on all of them, whatever else is in its batch:
      * T = 17 distinct tokens: the kernel-per-stage path (24 launches);
      * the first 16 and the first 4 of them: the one-launch small-batch kernel;
      * single tokens: the one-launch batch-1 kernel."""
    shape, layers, hosts = stack3
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    for act in (tm.TERN_ACT_BF16, tm.TERN_ACT_INT8):
        assert tm.moe_stack_kernel_launches(layers[0], 3, 1, act) == 1
        assert tm.moe_stack_kernel_launches(layers[0], 3, 2, act) == 1
        assert tm.moe_stack_kernel_launches(layers[0], 3, 16, act) == 1
        assert tm.moe_stack_kernel_launches(layers[0], 3, 17, act) == 24
        x = synth.tokens_bf16(WID_STACK, 8, 17, shape.d)
        stage = dev_u16(x, dev)
        tm.moe_stack_decode(st, stage, act=act)
        b16 = dev_u16(x[:16], dev)
        tm.moe_stack_decode(st, b16, act=act)
        b4 = dev_u16(x[:4], dev)
        tm.moe_stack_decode(st, b4, act=act)
        b2 = dev_u16(np.concatenate([x[5:6], x[5:6]]), dev)  # one token twice: one expert list of two
        tm.moe_stack_decode(st, b2, act=act)
        assert tm.tern_stream_status() == 0
        s16 = stage.view(torch.int16)
        assert torch.equal(b16.view(torch.int16), s16[:16])
        assert torch.equal(b4.view(torch.int16), s16[:4])
        assert torch.equal(b2.view(torch.int16)[0], s16[5]) and torch.equal(b2.view(torch.int16)[1], s16[5])
        for i in (0, 3, 16):
            one = dev_u16(x[i:i + 1], dev)
            tm.moe_stack_decode(st, one, act=act)
            assert torch.equal(one.view(torch.int16)[0], s16[i]), i


@pytest.fixture(scope="module")
def stack24(cuda_dev):
    shape = synth.MoEShape()
    layers = [device_layer(WID_STACK, l, shape, cuda_dev) for l in range(24)]
    return shape, layers


@pytest.mark.parametrize("act,steps", [(tm.TERN_ACT_BF16, (0, 1)), (tm.TERN_ACT_INT8, (2, 3))])
def test_stack24_persistent_teacher_forced(stack24, act, steps):
    """The 24-layer stack, one launch per token (the benchmark's configuration).  Every layer
    is checked against the oracle run on the kernel's own input to that layer:
      * experts bit-exact, gates within 1e-12;
      * h (the slot SwiGLU outputs, fp32) within 1e-5 of the largest;
      * y, the FFN output before its bf16 cast (fp32): bf16 path within rel-L2 1e-5 and
        max-abs 1e-4 * ||n||_2 of the oracle (n = the layer's normalised input); int8 path
        within 1e-6 of the largest |y| of the oracle teacher-forced on the kernel's own h
        (its int8 codes), so the int32 down sums are the same integers;
      * x_out = bf16(x + bf16(y)) within one bf16 ulp of itself plus one of bf16(y) (at most
        0.5% differ)."""
    shape, layers = stack24
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], 1, act), dev)
    lay = tm.moe_stack_workspace_layout(layers[0], 1, act)
    k, d, f = shape.k, shape.d, shape.f
    hosts = [HostLayer(WID_STACK, l, shape) for l in range(24)]
    for step in steps:
        x = synth.tokens_bf16(WID_STACK, 1000 + step, 1, d)
        xd = dev_u16(x, dev)
        tm.moe_stack_decode(st, xd, eps=1e-6, act=act, ws=ws)
        assert tm.tern_stream_status() == 0
        hist = host_u16(ws_view(ws, lay["hist"], torch.int16, 25 * d).view(25, d))
        idx = ws_view(ws, lay["idx"], torch.int32, 24 * k).view(24, k).cpu().numpy()
        g64 = ws_view(ws, lay["gates64"], torch.float64, 24 * k).view(24, k).cpu().numpy()
        y32 = ws_view(ws, lay["y32"], torch.float32, 24 * d).view(24, d).cpu().numpy().astype(np.float64)
        h32 = ws_view(ws, lay["h32"], torch.float32, 24 * k * f).view(24, k, f).cpu().numpy()
        assert (hist[0] == x[0]).all()
        assert (hist[24] == host_u16(xd)[0]).all()
        mism = 0
        for l in range(24):
            n, _ = oracle.rmsnorm(hist[l], 1e-6)
            _, idx_ref, _, _ = hosts[l].route(n)
            hosts[l].fill(idx_ref)
            L = hosts[l].oracle_layer()
            ref = oracle.moe_ffn(L, n, act)
            assert (idx[l] == ref["idx"][0]).all(), l
            assert np.abs(g64[l] - ref["gates"][0]).max() <= 1e-12
            hmax = np.abs(ref["h"][0]).max()
            assert np.abs(h32[l] - ref["h"][0]).max() <= 1e-5 * hmax, l
            if act == tm.TERN_ACT_BF16:
                y64 = ref["y64"][0]
                nn = np.linalg.norm(synth.bf16_bits_to_f64(n[0]))
                assert np.linalg.norm(y32[l] - y64) <= 1e-5 * np.linalg.norm(y64), l
                assert np.abs(y32[l] - y64).max() <= 1e-4 * nn, l
            else:
                qh = np.empty((1, k, f), np.int8)
                sh = np.empty((1, k), np.float32)
                for q in range(k):
                    qh[0, q], sh[0, q] = oracle.quant_absmax(h32[l, q])
                y64 = oracle.moe_ffn(L, n, act, qh_in=qh, sh_in=sh)["y64"][0]
                assert np.abs(y32[l] - y64).max() <= 1e-6 * np.abs(y64).max(), l
            x_out = _oracle_bf16(synth.bf16_bits_to_f64(hist[l]) + synth.bf16_bits_to_f64(_oracle_bf16(y64)))
            close = _x_out_close(hist[l + 1], x_out, y64)
            assert close.all(), (l, np.argwhere(~close)[:5])
            mism += int((hist[l + 1] != x_out).sum())
        assert mism <= 24 * d * 5e-3
        # and the whole chain stays finite and of sane size
        xf = synth.bf16_bits_to_f64(hist)
        assert np.isfinite(xf).all() and np.abs(xf).max() < 1e3


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_stack_kernel_waits_time_out_and_the_next_call_recovers(stack3, act):
    """The persistent kernel's own bounded waits: with one exchange made to never complete
    (CTA 0 waits at layer 1 for an h tag that no CTA writes) and a 200 us bound on every wait,
    the kernel gives up by itself -- CTA 0 first, the others when its outputs do not arrive --
    and the device status word reads TERN_ETIMEOUT.  The same workspace then decodes a token
    normally, bit for bit as on a fresh workspace.  Nothing faults or hangs: every wait ends
    on its own."""
    shape, layers, hosts = stack3
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], 1, act), dev)
    assert tm.tern_stream_status() == 0
    xs = dev_u16(synth.tokens_bf16(WID_STACK, 21, 1, shape.d), dev)
    tm.tern_test_stack_stall(st, xs, stall_layer=1, limit_ns=200_000, act=act, ws=ws)
    assert tm.tern_stream_status() == 5  # TERN_ETIMEOUT
    assert tm.tern_stream_status() == 0  # read and cleared
    x = synth.tokens_bf16(WID_STACK, 22, 1, shape.d)
    a = dev_u16(x, dev)
    tm.moe_stack_decode(st, a, act=act, ws=ws)
    b = dev_u16(x, dev)
    tm.moe_stack_decode(st, b, act=act)  # fresh workspace
    assert tm.tern_stream_status() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_stack24_small_batch_teacher_forced(stack24, act):
    """The 24-layer stack for T = 4 tokens in one launch (the small-batch kernel).  Its
    per-layer record is checked token by token against the oracle run on the kernel's own
    input to that layer, with the batch-1 test's tolerances: experts bit-exact, gates within
    1e-12, h within 1e-5 of the largest, y within rel-L2 1e-5 and max-abs 1e-4 * ||n||_2
    (bf16; int8: within 1e-6 of the largest, teacher-forced on the kernel's h), x_out within
    one bf16 ulp of itself plus one of bf16(y)."""
    shape, layers = stack24
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    T = 4
    assert tm.moe_stack_kernel_launches(layers[0], 24, T, act) == 1
    ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], T, act), dev)
    lay = tm.moe_stack_workspace_layout(layers[0], T, act)
    k, d, f = shape.k, shape.d, shape.f
    hosts = [HostLayer(WID_STACK, l, shape) for l in range(24)]
    x = synth.tokens_bf16(WID_STACK, 2000 + act, T, d)
    xd = dev_u16(x, dev)
    tm.moe_stack_decode(st, xd, eps=1e-6, act=act, ws=ws)
    assert tm.tern_stream_status() == 0
    hist = host_u16(ws_view(ws, lay["hist"], torch.int16, 25 * T * d).view(25, T, d))
    idx = ws_view(ws, lay["idx"], torch.int32, 24 * T * k).view(24, T, k).cpu().numpy()
    g64 = ws_view(ws, lay["gates64"], torch.float64, 24 * T * k).view(24, T, k).cpu().numpy()
    y32 = ws_view(ws, lay["y32"], torch.float32, 24 * T * d).view(24, T, d).cpu().numpy().astype(np.float64)
    h32 = ws_view(ws, lay["h32"], torch.float32, 24 * T * k * f).view(24, T, k, f).cpu().numpy()
    assert (hist[0] == x).all()
    assert (hist[24] == host_u16(xd)).all()
    mism = 0
    for l in range(24):
        n, _ = oracle.rmsnorm(hist[l], 1e-6)
        _, idx_ref, _, _ = hosts[l].route(n)
        hosts[l].fill(idx_ref)
        L = hosts[l].oracle_layer()
        ref = oracle.moe_ffn(L, n, act)
        assert (idx[l] == ref["idx"]).all(), l
        assert np.abs(g64[l] - ref["gates"]).max() <= 1e-12
        for t in range(T):
            hmax = np.abs(ref["h"][t]).max()
            assert np.abs(h32[l, t] - ref["h"][t]).max() <= 1e-5 * hmax, (l, t)
        if act == tm.TERN_ACT_BF16:
            y64 = ref["y64"]
            for t in range(T):
                nn = np.linalg.norm(synth.bf16_bits_to_f64(n[t]))
                assert np.linalg.norm(y32[l, t] - y64[t]) <= 1e-5 * np.linalg.norm(y64[t]), (l, t)
                assert np.abs(y32[l, t] - y64[t]).max() <= 1e-4 * nn, (l, t)
        else:
            qh = np.empty((T, k, f), np.int8)
            sh = np.empty((T, k), np.float32)
            for t in range(T):
                for q in range(k):
                    qh[t, q], sh[t, q] = oracle.quant_absmax(h32[l, t, q])
            y64 = oracle.moe_ffn(L, n, act, qh_in=qh, sh_in=sh)["y64"]
            for t in range(T):
                assert np.abs(y32[l, t] - y64[t]).max() <= 1e-6 * np.abs(y64[t]).max(), (l, t)
        x_out = _oracle_bf16(synth.bf16_bits_to_f64(hist[l]) + synth.bf16_bits_to_f64(_oracle_bf16(y64)))
        close = _x_out_close(hist[l + 1], x_out, y64)
        assert close.all(), (l, np.argwhere(~close)[:5])
        mism += int((hist[l + 1] != x_out).sum())
    assert mism <= 24 * T * d * 5e-3


@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_small_batch_kernel_waits_time_out_and_the_next_call_recovers(stack3, act):
    """The small-batch kernel's own bounded waits: CTA 0 does not arrive at the grid barrier
    after the gate/up stage of layer 1, and every wait is bounded by 200 us.  All CTAs give up at
    that barrier and leave by themselves; the status word reads TERN_ETIMEOUT; the last CTA out
    resets the barrier counters, so the same workspace then decodes 4 tokens bit for bit as a
    fresh one.  Nothing faults or hangs: every wait ends on its own."""
    shape, layers, hosts = stack3
    dev = layers[0].gate.device
    st = tm.Stack(layers)
    T = 4
    ws = tm.workspace(tm.moe_stack_workspace_bytes(layers[0], T, act), dev)
    assert tm.tern_stream_status() == 0
    xs = dev_u16(synth.tokens_bf16(WID_STACK, 31, T, shape.d), dev)
    tm.tern_test_stack_batch_stall(st, xs, stall_layer=1, limit_ns=200_000, act=act, ws=ws)
    assert tm.tern_stream_status() == 5  # TERN_ETIMEOUT
    assert tm.tern_stream_status() == 0  # read and cleared
    x = synth.tokens_bf16(WID_STACK, 32, T, shape.d)
    a = dev_u16(x, dev)
    tm.moe_stack_decode(st, a, act=act, ws=ws)
    b = dev_u16(x, dev)
    tm.moe_stack_decode(st, b, act=act)  # fresh workspace
    assert tm.tern_stream_status() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
