"""Shared builders for the GPU parity tests: the same seeded workload on the device
(packed by the CUDA library) and on the host (packed by the oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
import ternary_weight_moe_b200 as tm


def dev_u16(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def device_layer(wid: int, layer: int, shape: synth.MoEShape, dev) -> tm.MoELayer:
    """Whole layer generated and packed on the device."""
    E, d, f = shape.E, shape.d, shape.f
    gc, uc, dc = synth.layer_codes_torch(wid, layer, shape, dev)
    gate = tm.tern_pack(gc.view(E * f, d)).view(E, f, d // 4)
    up = tm.tern_pack(uc.view(E * f, d)).view(E, f, d // 4)
    down = tm.tern_pack(dc.view(E * d, f)).view(E, d, f // 4)
    del gc, uc, dc
    sg, su, sd = synth.layer_scales(wid, layer, shape)
    router = synth.layer_router(wid, layer, shape)
    return tm.MoELayer(gate, up, down, torch.from_numpy(sg).to(dev), torch.from_numpy(su).to(dev),
                       torch.from_numpy(sd).to(dev), dev_u16(router, dev), k=shape.k)


class HostLayer:
    """Host copy for the oracle in which only the requested experts are filled."""

    def __init__(self, wid: int, layer: int, shape: synth.MoEShape):
        self.wid, self.layer, self.shape = wid, layer, shape
        E, d, f = shape.E, shape.d, shape.f
        self.gate = np.zeros((E, f, d // 4), np.uint8)
        self.up = np.zeros((E, f, d // 4), np.uint8)
        self.down = np.zeros((E, d, f // 4), np.uint8)
        self.sg, self.su, self.sd = synth.layer_scales(wid, layer, shape)
        self.router = synth.layer_router(wid, layer, shape)
        self.filled = set()

    def fill(self, experts):
        for e in sorted(set(int(v) for v in np.ravel(experts)) - self.filled):
            g, u, dn = synth.expert_codes(self.wid, self.layer, self.shape, e)
            gp, up, dp = oracle.pack_layer_codes(g[None], u[None], dn[None])
            self.gate[e], self.up[e], self.down[e] = gp[0], up[0], dp[0]
            self.filled.add(e)

    def oracle_layer(self) -> oracle.Layer:
        return oracle.Layer(self.gate, self.up, self.down, self.sg, self.su, self.sd, self.router, k=self.shape.k)

    def route(self, x):
        return oracle.route(self.router, x, self.shape.k)


def ws_view(ws: torch.Tensor, off: int, dtype, count: int) -> torch.Tensor:
    esz = torch.empty(0, dtype=dtype).element_size()
    return ws[off:off + count * esz].view(dtype)
