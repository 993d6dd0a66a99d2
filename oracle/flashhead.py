"""Oracle for a FlashHead-style approximate output head -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package's smoke check and the CPU-baseline leg of the benchmark may
use this module.  Plain numpy in fp64; it shares nothing with the CUDA library.

What it computes ("A 20B AI Model Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac
Mini", "The Architecture: Designed for the Hardware": the output projection to a ~151,000-token
vocabulary is clustered into 4,748 groups, the top 512 clusters are found by scoring 4-bit
centroids, and only their tokens get full-precision projections).  The pages leave the details
open; the readings taken here:
  - the vocabulary is stored cluster-major: cluster c holds tokens c*cs .. c*cs+cs-1 (cs equal
    for all clusters; 151,936 = 4,748 x 32);
  - a centroid is the mean of its cluster's bf16 unembedding rows (exact in fp64);
  - 4-bit centroids: symmetric int4 in [-7, 7], one fp64 scale per centroid = absmax / 7,
    q = clamp(rint(c / scale)) with ties to even; two values per byte, element 2j in the low
    nibble (two's complement); an all-zero centroid has scale 0 and q = 0;
  - score_c = scale_c * sum_k q_ck x_k, the sum exact in fp64;
  - the top `top_c` clusters by score, ties to the lower cluster index, in that order;
  - candidate logits: sum_k W_vk x_k over the selected clusters' tokens (bf16 x bf16 products
    are exact in fp64; the sum is exact here), in selection order then row order;
  - the answer is the candidate with the largest logit, ties to the lower token id.
"""
from __future__ import annotations

import numpy as np

import synth


def _f64(bits):
    return synth.bf16_bits_to_f64(np.ascontiguousarray(bits, dtype=np.uint16))


def centroids(W_bits, cluster_size):
    """Means of consecutive groups of `cluster_size` rows, fp64 [n_clusters, d]."""
    W = _f64(W_bits)
    V, d = W.shape
    assert V % cluster_size == 0
    return W.reshape(V // cluster_size, cluster_size, d).sum(axis=1) / cluster_size


def quant4(C):
    """int4 codes (int8 array, values in [-7, 7]) and fp64 scales of centroids C."""
    C = np.asarray(C, dtype=np.float64)
    absmax = np.abs(C).max(axis=1)
    scale = absmax / 7.0
    q = np.zeros(C.shape, dtype=np.int8)
    nz = scale > 0
    q[nz] = np.clip(np.rint(C[nz] / scale[nz, None]), -7, 7).astype(np.int8)
    return q, scale


def pack4(q):
    q = np.asarray(q, dtype=np.int8)
    assert q.shape[1] % 2 == 0
    lo = q[:, 0::2].astype(np.int16) & 0xF
    hi = q[:, 1::2].astype(np.int16) & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack4(p):
    p = np.asarray(p, dtype=np.uint8).astype(np.int16)
    lo = p & 0xF
    hi = p >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.int8)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    return q


def scores(C4, scale, x_bits):
    q = unpack4(C4).astype(np.float64)
    x = _f64(x_bits).reshape(-1)
    return (q @ x) * np.asarray(scale, dtype=np.float64)


def select(sc, top_c):
    """Indices of the top_c largest scores, larger first, ties to the lower index."""
    sc = np.asarray(sc, dtype=np.float64)
    order = np.lexsort((np.arange(sc.size), -sc))
    return order[:top_c].astype(np.int32)


def head(W_bits, x_bits, sel, cluster_size):
    """Candidate token ids and their exact logits, selection order then row order."""
    ids = (np.asarray(sel, dtype=np.int64)[:, None] * cluster_size + np.arange(cluster_size)[None, :]).reshape(-1)
    x = _f64(x_bits).reshape(-1)
    logits = _f64(W_bits[ids]) @ x
    return ids.astype(np.int32), logits


def best(ids, logits):
    order = np.lexsort((ids, -logits))
    return int(ids[order[0]])


def flash_head(W_bits, C4, scale, x_bits, cluster_size, top_c):
    sc = scores(C4, scale, x_bits)
    sel = select(sc, top_c)
    ids, lg = head(W_bits, x_bits, sel, cluster_size)
    return {"scores": sc, "sel": sel, "ids": ids, "logits": lg, "best": best(ids, lg)}
