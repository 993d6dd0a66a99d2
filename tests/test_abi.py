"""The C-ABI library: it loads without a GPU, exports every function the header declares,
and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os

import pytest

import ternary_weight_moe_b200 as tm


def test_library_exports_every_header_function():
    names = tm.header_functions()
    assert len(names) >= 15
    L = tm.lib()
    for n in names:
        assert hasattr(L, n), n
    assert tm.abi_version() == 3


def test_status_strings():
    assert tm.status_str(0) == "TERN_OK"
    for c in range(1, 8):
        assert tm.status_str(c).startswith(tm.STATUS[c])


def _fake_layer(d=2048, f=512, E=256, k=8, misalign=0):
    base = 1 << 40
    return tm.MoELayerC(base + misalign, base + 4096, base + 8192, base + 12288, base + 16384, base + 20480,
                        base + 24576, d, f, E, k)


def test_workspace_queries_are_host_only():
    L = _fake_layer()
    n1 = tm.lib().moe_ffn_workspace_bytes(ctypes.byref(L), 1, tm.TERN_ACT_BF16)
    n64 = tm.lib().moe_ffn_workspace_bytes(ctypes.byref(L), 64, tm.TERN_ACT_BF16)
    assert 0 < n1 < n64
    assert tm.lib().moe_ffn_workspace_bytes(ctypes.byref(L), 65, tm.TERN_ACT_BF16) == 0
    assert tm.lib().moe_stack_workspace_bytes(ctypes.byref(L), 1, tm.TERN_ACT_INT8) > 0
    out = tm.FfnLayoutC()
    assert tm.lib().moe_ffn_workspace_layout(ctypes.byref(L), 4, tm.TERN_ACT_INT8, ctypes.byref(out)) == 0
    assert out.total == tm.lib().moe_ffn_workspace_bytes(ctypes.byref(L), 4, tm.TERN_ACT_INT8)
    assert out.acc_g >= 0 and out.qx >= 0
    assert tm.lib().moe_ffn_workspace_layout(ctypes.byref(L), 4, tm.TERN_ACT_BF16, ctypes.byref(out)) == 0
    assert out.acc_g == -1 and out.qx == -1
    assert tm.lib().moe_route_workspace_bytes(1, 256) > 256 * 8


@pytest.mark.parametrize("T", [1, 2, 4, 16])
@pytest.mark.parametrize("act", [tm.TERN_ACT_BF16, tm.TERN_ACT_INT8])
def test_stack_record_layout_holds_the_documented_shapes(T, act):
    """The per-layer record of a one-launch stack call: regions in header order, 16-byte
    aligned, each large enough for the shapes the header documents at the largest stack (64
    layers), and the layout's total equal to the workspace size query."""
    L = _fake_layer()
    d, f, k, nl = 2048, 512, 8, 64
    out = tm.StackLayoutC()
    assert tm.lib().moe_stack_workspace_layout(ctypes.byref(L), T, act, ctypes.byref(out)) == 0
    assert out.total == tm.lib().moe_stack_workspace_bytes(ctypes.byref(L), T, act)
    offs = [out.hist, out.idx, out.gates64, out.y32, out.h32, out.trace, out.total]
    assert all(o % 16 == 0 for o in offs) and offs == sorted(offs)
    assert out.idx - out.hist >= (nl + 1) * T * d * 2
    assert out.gates64 - out.idx >= nl * T * k * 4
    assert out.y32 - out.gates64 >= nl * T * k * 8
    assert out.h32 - out.y32 >= nl * T * d * 4
    assert out.trace - out.h32 >= nl * T * k * f * 4
    if T == 1:
        assert out.total - out.trace >= 2 * nl * 256 * 24 * 8


@pytest.mark.parametrize("bad", [dict(d=100), dict(f=0), dict(E=0), dict(k=9), dict(k=300, E=256), dict(E=2000),
                                 dict(d=4096)])
def test_layer_validation(bad):
    L = _fake_layer(**bad)
    assert tm.lib().moe_ffn_workspace_bytes(ctypes.byref(L), 1, tm.TERN_ACT_BF16) == 0


def test_argument_checks_before_any_launch():
    L = tm.lib()
    p = ctypes.c_void_p(1 << 40)
    # K not a multiple of 64
    assert L.tern_gemv(p, p, 16, 100, 0, p, None, 1, None, p, None) == 1
    # T out of range
    assert L.tern_gemv(p, p, 16, 512, 0, p, None, 0, None, p, None) == 1
    assert L.tern_gemv(p, p, 16, 512, 0, p, None, 65, None, p, None) == 1
    # bf16 path takes no accumulator output
    assert L.tern_gemv(p, p, 16, 512, 0, p, None, 1, p, p, None) == 1
    # misaligned packed weights
    q = ctypes.c_void_p((1 << 40) + 4)
    assert L.tern_gemv(q, p, 16, 512, 1, p, None, 1, None, p, None) == 2
    # K = 3072 is neither <= 2048 nor a multiple of 2048
    assert L.tern_gemv(p, p, 16, 3072, 1, p, None, 1, None, p, None) == 1
    # null workspace
    Lc = _fake_layer()
    assert L.moe_ffn_decode(ctypes.byref(Lc), p, 1, 0, p, None, None, 0, None) == 6
    # misaligned expert weights
    Lm = _fake_layer(misalign=8)
    assert L.moe_ffn_decode(ctypes.byref(Lm), p, 1, 0, p, None, p, 1 << 30, None) == 2
    # route: k > E
    assert L.moe_route_topk(p, p, 1, 2048, 4, 8, p, p, None, p, 1 << 20, None) == 1
    # pack: K not a multiple of 4
    assert L.tern_pack(p, 4, 6, p, None) == 1
    # stack: too many layers / negative eps
    arr = (tm.MoELayerC * 1)(Lc)
    assert L.moe_stack_decode(arr, 0, p, 1, 1e-6, 0, p, 1 << 30, None) == 1
    assert L.moe_stack_decode(arr, 1, p, 1, -1.0, 0, p, 1 << 30, None) == 1
    assert L.tern_test_bounded_wait(None, 10, None) == 1


def test_base3_format_host_checks():
    """The five-weights-per-byte calls: row size arithmetic and argument checks, no GPU."""
    L = tm.lib()
    assert [L.tern5_row_bytes(k) for k in (0, 1, 5, 80, 81, 2048, 16384)] == [0, 16, 16, 16, 32, 416, 3280]
    p = ctypes.c_void_p(1 << 40)
    assert L.tern5_gemv(p, p, 16, 0, 0, p, None, 1, None, p, None) == 1          # K < 1
    assert L.tern5_gemv(p, p, 16, 16385, 0, p, None, 1, None, p, None) == 1      # K too large
    assert L.tern5_gemv(p, p, 16, 2048, 0, p, None, 65, None, p, None) == 1      # T out of range
    assert L.tern5_gemv(p, p, 16, 2048, 0, p, None, 1, p, p, None) == 1          # bf16 with acc
    q = ctypes.c_void_p((1 << 40) + 8)
    assert L.tern5_gemv(q, p, 16, 2048, 1, p, None, 1, None, p, None) == 2       # misaligned rows
    assert L.tern5_pack(None, 4, 10, p, None) == 1
    assert L.tern5_unpack(p, 0, 10, p, None) == 1


def test_flash_head_host_checks():
    """Argument checks of the approximate head, before any launch (no GPU needed)."""
    L = tm.lib()
    p = ctypes.c_void_p(1 << 40)
    args = dict(d=2048, nc=4748, cs=32, top=512)

    def call(d=2048, nc=4748, cs=32, top=512, W=p):
        return L.flash_head(p, p, W, p, d, nc, cs, top, p, p, p, p, p, None)

    assert call(d=100) == 1               # d not a multiple of 64
    assert call(d=16384) == 1             # d too large for the staged activations
    assert call(nc=8193) == 1             # too many clusters for the one-CTA selection
    assert call(top=0) == 1 and call(top=4749) == 1
    assert call(cs=0) == 1
    assert call(W=ctypes.c_void_p((1 << 40) + 2)) == 2   # rows not 16-byte aligned
    assert L.flash_head(None, p, p, p, 2048, 4748, 32, 512, p, p, p, p, p, None) == 1
    assert L.flash_head_centroids(p, 2048, 0, 32, p, p, None) == 1
    assert L.flash_head_centroids(p, 2048, 4748, 32, p, ctypes.c_void_p((1 << 40) + 4), None) == 2
    assert args["nc"] * args["cs"] == 151936


def test_binding_signatures_match_the_header():
    """Every declared function has a binding whose argument count matches its declaration."""
    import re

    txt = open(tm.HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    L = tm.lib()
    names = tm.header_functions()
    assert {"flash_head", "flash_head_centroids", "tern5_gemv", "moe_stack_decode"} <= set(names)
    for name in names:
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", txt)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert getattr(L, name).argtypes is not None, name
        assert len(getattr(L, name).argtypes) == len(params), name


def test_static_route_limits_before_any_launch():
    """The allocation-free routing call refuses, on the host, every request its fixed
    scratch cannot hold or that is malformed: more than 64 tokens even with few experts,
    more than 16,384 token-expert logits, k > E, d not a multiple of 8."""
    L = tm.lib()
    p = ctypes.c_void_p(1 << 40)
    assert L.moe_route_topk_static(p, p, 65, 64, 8, 8, p, p, None, None) == 1      # T > 64, small E
    assert L.moe_route_topk_static(p, p, 64, 64, 512, 8, p, p, None, None) == 1     # T*E = 32768
    assert L.moe_route_topk_static(p, p, 4, 64, 4, 8, p, p, None, None) == 1        # k > E
    assert L.moe_route_topk_static(p, p, 4, 60, 256, 8, p, p, None, None) == 1      # d % 8 != 0
    assert L.moe_route_topk_static(p, p, 4, 64, 256, 9, p, p, None, None) == 1      # k > 8
    q = ctypes.c_void_p((1 << 40) + 4)
    assert L.moe_route_topk_static(q, p, 4, 64, 256, 8, p, p, None, None) == 2      # misaligned router


def test_route_binding_rejects_wrong_shapes():
    """The Python routing calls check x, logits, idx and gates against Wg's shape before
    they touch the device (so a short buffer is a ValueError, not an out-of-bounds write)."""
    import torch

    Wg = torch.zeros((256, 2048), dtype=torch.int16)
    for fn in (tm.moe_route_topk, tm.moe_route_topk_static):
        with pytest.raises(ValueError):
            fn(Wg, torch.zeros((2, 1024), dtype=torch.int16))                     # x width != d
        x = torch.zeros((2, 2048), dtype=torch.int16)
        with pytest.raises(ValueError):
            fn(Wg, x, 8, logits=torch.zeros((2, 128), dtype=torch.float64))        # logits [T][E]
        with pytest.raises(ValueError):
            fn(Wg, x, 8, idx=torch.zeros((2, 4), dtype=torch.int32))               # idx [T][k]
        with pytest.raises(ValueError):
            fn(Wg, x, 8, gates=torch.zeros((1, 8), dtype=torch.float32))           # gates [T][k]


def test_table_free_decode_matches_the_code_table(tmp_path):
    """The integer-logic decode of the fused kernels (csrc/decode.cuh), compiled for the host:
    every byte value, byte position and code position gives 64 * w with w the code's weight
    (11 reads as 0), and the position-major segment dot equals the plain sum."""
    import subprocess

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = str(tmp_path / "decode_check")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-o", exe, os.path.join(root, "tests", "decode_check.cpp")])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and "decode ok" in out.stdout, out.stdout + out.stderr
