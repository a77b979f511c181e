"""SOCKET soft-count attention estimator -- float64 CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Source: SOCKET technical summary ("SOCKET - SOft Collision Kernel EsTimator
for sparse attention", gist.science/ja/paper/2602.06283): section
"理論的基盤" (the soft LSH score approximates a kernel closely related to
softmax attention, an angular kernel) and "主要な貢献" item 4 (an end-to-end
error bound for the soft-count attention estimator, split into sampling
variance, finite-table error and soft-bucketisation bias).

The page prints no formula. The plainest reading, used here: the soft
collision count of key i for query head h,

    c_{h,i} = sum_l p_{h,l}(id_l(i)),

(the soft bucket probabilities of ``socket_ref.bucket_probabilities``, summed
over the L tables, with no value-norm weight) is the estimate of the kernel
value between q_h and k_i, and the estimator replaces the softmax weights of
exact attention by these counts over the selected keys S:

    o_h = sum_{i in S} c_{h,i} v_i / sum_{i in S} c_{h,i}.

It needs the values of the selected keys and their cached bucket IDs, not
their keys.
"""

from __future__ import annotations

import numpy as np

from .socket_ref import bucket_probabilities


def soft_counts(q, R, ids, L: int, P: int, tau: float) -> np.ndarray:
    """c_i = sum_l p_l(ids[i, l]) for one query row q and keys with IDs ids [n, L]."""
    p = bucket_probabilities(q, R, L, P, tau)               # [L, 2^P]
    ids = np.asarray(ids, dtype=np.int64)
    return p[np.arange(L)[None, :], ids].sum(axis=1)


def soft_count_attention(Qg, V, R, ids, idx, L: int, P: int, tau: float) -> np.ndarray:
    """The estimator for every query head of a group over the selected keys.

    Qg: [G, d]; V: [N, d] values; ids: [N, L] cached bucket IDs; idx: selected
    key indices. Returns [G, d]: o_h = sum_i c_{h,i} v_i / sum_i c_{h,i}.
    """
    idx = np.asarray(idx, dtype=np.int64)
    Vs = np.asarray(V, dtype=np.float64)[idx]
    ids_s = np.asarray(ids)[idx]
    out = []
    for q in np.asarray(Qg, dtype=np.float64):
        c = soft_counts(q, R, ids_s, L, P, tau)
        out.append((c @ Vs) / c.sum())
    return np.stack(out)
