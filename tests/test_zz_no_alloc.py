"""The workspace-free routing call (moe_route_topk_static), for callers that cannot
allocate device memory: it must give the same experts, gates and logits as the
workspace-based moe_route_topk, on two calls in a row (the second call finds the fixed
scratch holding the first call's leftovers).  Collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_moe_b200 as tm

pytestmark = pytest.mark.gpu


def _dev16(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)


def test_static_route_matches_the_oracle_and_the_workspace_route_twice(cuda_dev):
    """Against the CPU oracle (experts and logits bit-exact, gates within fp32 rounding) and
    against the workspace call, on two calls in a row."""
    shape = synth.MoEShape()
    Wg_h = synth.layer_router(3, 0, shape)
    Wg = _dev16(Wg_h, cuda_dev)
    for call, T in enumerate((4, 64)):
        x_h = synth.tokens_bf16(3, 500 + call, T, shape.d)
        x = _dev16(x_h, cuda_dev)
        lg_or, idx_or, g_or, bad = oracle.route(Wg_h, x_h, 8)
        assert bad == 0
        lg_ref = torch.empty((T, shape.E), dtype=torch.float64, device=cuda_dev)
        idx_ref, g_ref = tm.moe_route_topk(Wg, x, 8, logits=lg_ref)
        lg = torch.full((T, shape.E), float("nan"), dtype=torch.float64, device=cuda_dev)
        idx, g = tm.moe_route_topk_static(Wg, x, 8, logits=lg)
        torch.cuda.synchronize()
        assert (idx.cpu().numpy() == idx_or).all()
        assert (lg.cpu().numpy() == lg_or).all()
        assert np.abs(g.cpu().numpy().astype(np.float64) - g_or).max() <= 1e-7
        assert torch.equal(idx, idx_ref)
        assert torch.equal(lg, lg_ref)
        assert (g - g_ref).abs().max().item() <= 1e-7
        # without a logits output the fixed scratch holds them
        idx2, g2 = tm.moe_route_topk_static(Wg, x, 8)
        torch.cuda.synchronize()
        assert torch.equal(idx2, idx_ref) and (g2 - g_ref).abs().max().item() <= 1e-7


def test_static_route_rejects_oversize(cuda_dev):
    E, d = 512, 64
    Wg = torch.zeros((E, d), dtype=torch.int16, device=cuda_dev)
    x = torch.zeros((64, d), dtype=torch.int16, device=cuda_dev)   # 64 x 512 > 16384
    with pytest.raises(tm.TernError) as ei:
        tm.moe_route_topk_static(Wg, x, 8)
    assert ei.value.code == 1
