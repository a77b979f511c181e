"""Exact softmax attention for one decode query -- float64 CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Source: SOCKET technical summary (gist.science/ja/paper/2602.06283), section
"中核メカニズム：ソフト LSH", step 4: after selection, exact attention is
computed on the chosen subset. Reading: the softmax is renormalised over the
subset (no importance weights) and the logit scale is 1/sqrt(d).
The dense decode baseline is the same computation over every cached key.
"""

from __future__ import annotations

import numpy as np


def exact_attention(q, Ks, Vs, scale: float) -> np.ndarray:
    """softmax(q . Ks^T * scale) . Vs for one query row.

    q: [d]; Ks, Vs: [m, d] with m >= 1. The softmax subtracts the max logit,
    exponentiates, and divides by the sum of weights.
    """
    q = np.asarray(q, dtype=np.float64)
    Ks = np.asarray(Ks, dtype=np.float64)
    Vs = np.asarray(Vs, dtype=np.float64)
    a = (Ks @ q) * scale
    w = np.exp(a - a.max())
    return (w @ Vs) / w.sum()


def attend_subset(Qg, K, V, idx, scale: float) -> np.ndarray:
    """Attention of each query head of a group over the selected keys only.

    Qg: [G, d]; K, V: [N, d]; idx: selected key indices. Returns [G, d].
    """
    idx = np.asarray(idx, dtype=np.int64)
    Ks = np.asarray(K)[idx]
    Vs = np.asarray(V)[idx]
    return np.stack([exact_attention(q, Ks, Vs, scale) for q in np.asarray(Qg)])


def dense_decode(Q, K, V, scale: float, N: int | None = None, pairs=None) -> np.ndarray:
    """Dense decode attention over the first N cached keys.

    Q: [B, Hq, d]; K, V: [B, Hkv, Ncap, d]. Returns O [B, Hq, d] float64 (NaN for
    pairs not in ``pairs`` when given).
    """
    B, Hq, d = np.shape(Q)
    Hkv = np.shape(K)[1]
    G = Hq // Hkv
    n = np.shape(K)[2] if N is None else N
    O = np.full((B, Hq, d), np.nan)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        for g in range(G):
            O[b, h * G + g] = exact_attention(Q[b, h * G + g], K[b, h, :n], V[b, h, :n], scale)
    return O
