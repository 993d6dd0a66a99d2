"""The approximate output head on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import synth
import ternary_weight_moe_b200 as tm
from oracle import flashhead as fh

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _run(W_bits_dev, x_bits, cs, top_c):
    dev = W_bits_dev.device
    C4, sc = tm.flash_head_centroids(W_bits_dev, cs)
    xd = torch.from_numpy(x_bits.view(np.int16)).to(dev)
    out = tm.flash_head(C4, sc, W_bits_dev, xd, cs, top_c)
    torch.cuda.synchronize()
    return C4, sc, {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("top_c", [1, 7, 64])
def test_flash_head_small_bit_exact(cuda_dev, top_c):
    V, d, cs = 64 * 32, 256, 32
    W = synth.normal_bf16(21, 0, V * d, 0.02).reshape(V, d)
    x = synth.normal_bf16(22, 0, d, 1.0)
    Wd = torch.from_numpy(W.view(np.int16)).to(cuda_dev)
    C4, sc, out = _run(Wd, x, cs, top_c)
    q, s = fh.quant4(fh.centroids(W, cs))
    assert (C4.cpu().numpy() == fh.pack4(q)).all() and (sc.cpu().numpy() == s).all()
    ref = fh.flash_head(W, fh.pack4(q), s, x, cs, top_c)
    assert (out["scores"] == ref["scores"]).all()
    assert (out["sel"] == ref["sel"]).all()
    assert (out["ids"] == ref["ids"]).all() and (out["logits"] == ref["logits"]).all()
    assert int(out["best"][0]) == ref["best"]


def test_flash_head_ties_go_to_the_lower_index(cuda_dev):
    V, d, cs = 8 * 4, 64, 4
    W = synth.normal_bf16(23, 0, V * d, 0.02).reshape(V, d)
    W[12:16] = W[4:8]      # cluster 3 = cluster 1: equal scores
    W[5] = W[4]            # tokens 4 and 5 equal: equal logits
    x = synth.normal_bf16(24, 0, d, 1.0)
    Wd = torch.from_numpy(W.view(np.int16)).to(cuda_dev)
    _, _, out = _run(Wd, x, cs, 8)
    ref = fh.flash_head(W, *(lambda q, s: (fh.pack4(q), s))(*fh.quant4(fh.centroids(W, cs))), x, cs, 8)
    assert (out["sel"] == ref["sel"]).all()
    pos1, pos3 = list(out["sel"]).index(1), list(out["sel"]).index(3)
    assert pos1 < pos3
    assert int(out["best"][0]) == ref["best"]


@pytest.mark.parametrize("nc,top_c,equal", [(100, 37, True), (3000, 1024, False), (2000, 1500, False),
                                             (3000, 700, True)])
def test_flash_head_selection_paths(cuda_dev, nc, top_c, equal):
    """The selection against the oracle on both of its paths: top_c <= 1,024 (radix select of
    the cutoff, then ranks) and more (a full sort).  With every cluster equal, all scores tie
    and the top_c lowest cluster indices must come out in order."""
    d, cs = 64, 4
    W = synth.normal_bf16(25 + nc, 0, nc * cs * d, 0.02).reshape(nc * cs, d)
    if equal:
        W[:] = W[:cs].reshape(1, cs, d).repeat(nc, 0).reshape(nc * cs, d)
    x = synth.normal_bf16(26 + nc, 0, d, 1.0)
    Wd = torch.from_numpy(W.view(np.int16)).to(cuda_dev)
    C4, sc, out = _run(Wd, x, cs, top_c)
    assert (out["sel"] == fh.select(out["scores"], top_c)).all()
    if equal:
        assert (out["sel"] == np.arange(top_c)).all()
    assert int(out["best"][0]) == fh.best(out["ids"], out["logits"])


def test_flash_head_full_size_sampled(cuda_dev):
    """151,936 tokens x 2,048, top 512 of 4,748 clusters: sampled centroids, scores and logits
    against the oracle, the selection and the answer against the oracle on the device's values."""
    hs = synth.head_shape()
    V, d, cs, top_c = hs["V"], hs["d"], hs["cluster_size"], hs["top_c"]
    Wd = synth.normal_bf16_torch(synth.derive(synth.BASE_SEED + 6, 1), 0, V * d, 0.02, cuda_dev).view(V, d)
    x = synth.normal_bf16(synth.derive(synth.BASE_SEED + 6, 2), 0, d, 1.0)
    C4, sc, out = _run(Wd, x, cs, top_c)
    rng = np.random.default_rng(7)
    C4h, sch = C4.cpu().numpy(), sc.cpu().numpy()
    for c in rng.choice(hs["n_clusters"], 12, replace=False):
        rows = _u16(Wd[c * cs:(c + 1) * cs])
        q, s = fh.quant4(fh.centroids(rows, cs))
        assert (C4h[c] == fh.pack4(q)[0]).all() and sch[c] == s[0]
    assert (out["scores"] == fh.scores(C4h, sch, x)).all()
    assert (out["sel"] == fh.select(out["scores"], top_c)).all()
    for qi in rng.choice(top_c * cs, 48, replace=False):
        v = int(out["ids"][qi])
        assert v == out["sel"][qi // cs] * cs + qi % cs
        _, lg = fh.head(_u16(Wd[v:v + 1]), x, np.array([0], np.int32), 1)
        assert out["logits"][qi] == lg[0]
    assert int(out["best"][0]) == fh.best(out["ids"], out["logits"])
