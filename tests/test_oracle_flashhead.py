"""Pins of the FlashHead oracle against arithmetic that does not go through it."""
from fractions import Fraction
import importlib.util
import itertools
import os

import numpy as np

import synth

# The mutant test runs these pins against planted-mistake copies of the module.
_SRC = os.environ.get("TERNMOE_FLASHHEAD_SRC")
if _SRC:
    _spec = importlib.util.spec_from_file_location("flashhead_under_test", _SRC)
    fh = importlib.util.module_from_spec(_spec)
    _spec.loader.exec_module(fh)
else:
    from oracle import flashhead as fh


def _bits(vals):
    return synth.f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


def test_centroid_is_the_exact_mean():
    W = _bits(synth.uniform01(5, 0, 6 * 4) * 4 - 2).reshape(6, 4)
    C = fh.centroids(W, 3)
    Wf = synth.bf16_bits_to_f64(W)
    for c in range(2):
        for k in range(4):
            exact = sum(Fraction(float(Wf[3 * c + r, k])) for r in range(3)) / 3
            assert abs(Fraction(float(C[c, k])) - exact) <= abs(exact) * Fraction(1, 2 ** 52)
    # identical rows: the centroid is the row; a row and its negation: zero
    same = np.repeat(_bits([[0.5, -1.25, 3.0, 0.0]]), 4, axis=0)
    assert (fh.centroids(same, 4)[0] == [0.5, -1.25, 3.0, 0.0]).all()
    pm = _bits([[1.5, -2.0], [-1.5, 2.0]])
    assert (fh.centroids(pm, 2) == 0).all()


def test_quant4_hand_values_and_ties_to_even():
    C = np.array([[7.0, -3.5, 0.5, -0.5, 1.5, 2.5, -7.0, 0.0],
                  [0.0] * 8])
    q, s = fh.quant4(C)
    assert s.tolist() == [1.0, 0.0]
    assert q[0].tolist() == [7, -4, 0, 0, 2, 2, -7, 0]
    assert (q[1] == 0).all()
    q2, s2 = fh.quant4(np.array([[0.07, 0.01, -0.035, 0.0]]))
    assert s2[0] == 0.07 / 7.0 and q2[0].tolist() == [7, 1, -4, 0]   # -0.035/0.01 = -3.5 -> -4


def test_pack4_nibble_order_and_roundtrip():
    pairs = np.array(list(itertools.product(range(-7, 8), repeat=2)), dtype=np.int8).reshape(1, -1)
    p = fh.pack4(pairs)
    assert (fh.unpack4(p) == pairs).all()
    one = fh.pack4(np.array([[3, -2]], np.int8))
    assert one.tolist() == [[0x03 | (0xE << 4)]]   # element 0 low nibble, -2 = 0xE


def test_scores_are_exact():
    q = np.array([[7, -1, 0, 3], [-7, 2, 5, -3]], np.int8)
    s = np.array([0.25, 1.0 / 7.0])
    x = _bits([1.5, -0.75, 2.0, 0.125])
    got = fh.scores(fh.pack4(q), s, x)
    xf = synth.bf16_bits_to_f64(x)
    for c in range(2):
        dot = sum(Fraction(int(q[c, k])) * Fraction(float(xf[k])) for k in range(4))
        assert got[c] == float(dot) * s[c]


def test_select_bruteforce_with_ties():
    rng = np.random.default_rng(3)
    for _ in range(20):
        sc = rng.integers(-3, 4, size=37).astype(np.float64)
        sel = fh.select(sc, 9)
        ref = sorted(range(37), key=lambda i: (-sc[i], i))[:9]
        assert sel.tolist() == ref


def test_all_clusters_selected_is_the_exact_full_head():
    """With every cluster kept the approximate head is the full head: same logits, same answer."""
    V, d, cs = 64, 32, 8
    W = synth.normal_bf16(11, 0, V * d, 0.02).reshape(V, d)
    x = synth.normal_bf16(12, 0, d, 1.0)
    q, s = fh.quant4(fh.centroids(W, cs))
    r = fh.flash_head(W, fh.pack4(q), s, x, cs, V // cs)
    full = synth.bf16_bits_to_f64(W) @ synth.bf16_bits_to_f64(x)
    assert sorted(r["ids"].tolist()) == list(range(V))
    assert (r["logits"] == full[r["ids"]]).all()
    assert r["best"] == int(np.lexsort((np.arange(V), -full))[0])
    # the candidates are exactly the selected clusters' rows, in selection order
    assert (r["ids"].reshape(-1, cs)[:, 0] // cs == r["sel"]).all()


def test_best_breaks_ties_to_the_lower_token_id():
    ids = np.array([5, 3, 9, 1], np.int32)
    assert fh.best(ids, np.array([1.0, 1.0, 0.5, -2.0])) == 3
    assert fh.best(ids, np.array([0.0, -1.0, 2.0, 2.0])) == 1
    assert fh.best(ids[:1], np.array([-7.0])) == 5
