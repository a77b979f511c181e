"""SOCKET soft-LSH scoring, selection and decode -- float64 CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Source: SOCKET technical summary ("SOCKET - SOft Collision Kernel EsTimator
for sparse attention", gist.science/ja/paper/2602.06283), section
"中核メカニズム：ソフト LSH", whose four numbered steps are:

1. pre-computation (prefill): keys are hashed into L independent tables by
   random projections; each key gets one bucket ID per table, and the norm of
   its value vector is cached;
2. soft assignment (decode): the query's projections onto the random
   hyperplanes give soft hash scores that go through a temperature-controlled
   softmax over *all* buckets of each table;
3. scoring: each key's score aggregates, over the L tables, the probability
   mass of the bucket that key sits in, weighted by the key's value norm;
4. selection: the top-k keys by that score are chosen deterministically and
   exact attention is computed on that subset (see ``attention_ref``).

The page prints no formula for step 2. The form used here is
p_l(b) = softmax_b( sum_j s_bj * z_lj / tau ), s_bj = +1 if bit j of b is
set else -1, z_lj = q_hat . r_lj -- the plain reading of "projections ... go
through a temperature softmax over all buckets". Readings adopted where the
page is silent (each one pinned by a test):

* the query is normalised before projecting (q_hat = q / |q|);
* bit j of a bucket ID is hyperplane j of the table, least significant bit
  first, and a projection of exactly 0 gives bit 0;
* the value norm is stored as the fp16 value nearest (ties to even) to the
  exact Euclidean norm, and scoring uses the stored fp16 value;
* with grouped-query attention one index set is chosen per KV head, scoring
  each key by the sum over the group's query heads;
* ties in the top-k go to the lower key index; the result is ascending.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import attend_subset


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def hash_key_ids(K, R, L: int, P: int):
    """Bucket IDs of keys in L tables of P hyperplanes each (step 1).

    K: [n, d] keys (any real dtype; used exactly, in float64).
    R: [L*P, d] hyperplanes; row l*P + j is hyperplane j of table l.
    Returns (ids [n, L] int64 in [0, 2^P), proj [n, L*P] float64), where
    bit j of ids[:, l] is 1 iff proj[:, l*P + j] > 0.
    """
    K = _f64(K)
    R = _f64(R)
    if R.shape[0] != L * P:
        raise ValueError("R must have L*P rows")
    proj = K @ R.T                                   # [n, L*P] random projections
    bits = (proj > 0).astype(np.int64).reshape(K.shape[0], L, P)
    weights = np.int64(1) << np.arange(P, dtype=np.int64)   # 2^j for hyperplane j
    ids = (bits * weights).sum(axis=2)
    return ids, proj


def value_norms_f16(V) -> np.ndarray:
    """Cached value norm of each key (step 1): fp16 nearest to |v|_2.

    V: [n, d]. Returns [n] float16. numpy rounds float64 -> float16 directly,
    to nearest with ties to even.
    """
    V = _f64(V)
    with np.errstate(over="ignore"):        # norms >= 65520 round to +inf, as fp16 does
        return np.sqrt((V * V).sum(axis=1)).astype(np.float16)


def _bucket_signs(P: int) -> np.ndarray:
    """s[b, j] = +1 if bit j of bucket b is set, else -1. Shape [2^P, P]."""
    b = np.arange(1 << P, dtype=np.int64)[:, None]
    j = np.arange(P, dtype=np.int64)[None, :]
    return np.where((b >> j) & 1, 1.0, -1.0)


def bucket_probabilities(q, R, L: int, P: int, tau: float) -> np.ndarray:
    """Soft assignment of one query to every bucket of every table (step 2).

    q: [d]; R: [L*P, d]. Returns p [L, 2^P] with each row summing to 1:
    p[l, b] = softmax over b of sum_j s_bj * z[l, j] / tau, z = R q_hat.
    The softmax is computed literally: subtract the row max, exponentiate,
    divide by the row sum.
    """
    q = _f64(q)
    R = _f64(R)
    q_hat = q / np.sqrt((q * q).sum())
    z = (R @ q_hat).reshape(L, P)                     # projections onto hyperplanes
    signs = _bucket_signs(P)                          # [2^P, P]
    logits = (z @ signs.T) / tau                      # [L, 2^P]
    logits = logits - logits.max(axis=1, keepdims=True)
    e = np.exp(logits)
    return e / e.sum(axis=1, keepdims=True)


def group_bucket_table(Qg, R, L: int, P: int, tau: float) -> np.ndarray:
    """Sum of the bucket probabilities of the query heads sharing a KV head.

    Qg: [G, d]. Returns T [L, 2^P], T[l, b] = sum_h p_h[l, b].
    """
    Qg = _f64(Qg)
    T = np.zeros((L, 1 << P), dtype=np.float64)
    for h in range(Qg.shape[0]):
        T += bucket_probabilities(Qg[h], R, L, P, tau)
    return T


def soft_collision_scores(T, ids, norms) -> np.ndarray:
    """Per-key soft collision score (step 3).

    T: [L, 2^P] (group-summed) bucket probabilities; ids: [n, L] bucket IDs;
    norms: [n] cached value norms (the stored fp16 values).
    score_i = norms_i * sum_l T[l, ids[i, l]].
    """
    T = _f64(T)
    ids = np.asarray(ids, dtype=np.int64)
    L = T.shape[0]
    mass = T[np.arange(L)[None, :], ids].sum(axis=1)
    return _f64(norms) * mass


def select_topk(scores, k: int) -> np.ndarray:
    """Deterministic top-k (step 4): the k largest scores, ties to lower index.

    Returns the chosen key indices in ascending order (int64).
    """
    scores = _f64(scores)
    if not 0 <= k <= scores.shape[0]:
        raise ValueError("k out of range")
    order = np.argsort(-scores, kind="stable")        # stable: equal scores keep index order
    return np.sort(order[:k])


def socket_decode_pair(Qg, K, V, R, ids, norms, L, P, tau, k, scale):
    """One (batch, kv-head) pair of the decode step, steps 2-4.

    Qg: [G, d] query heads of the group; K, V: [N, d] cached keys/values;
    ids: [N, L]; norms: [N] (the cache as given). Returns (O [G, d], idx [k],
    scores [N]).
    """
    T = group_bucket_table(Qg, R, L, P, tau)
    scores = soft_collision_scores(T, ids, norms)
    idx = select_topk(scores, k)
    O = attend_subset(Qg, K, V, idx, scale)
    return O, idx, scores


def socket_decode(Q, K, V, R, ids, norms, L, P, tau, k, scale, pairs=None):
    """Decode step over a batch.

    Q: [B, Hq, d]; K, V: [B, Hkv, N, d]; ids: [B, Hkv, N, L]; norms: [B, Hkv, N].
    Query head h reads KV head h // (Hq // Hkv). ``pairs`` optionally limits the
    work to a list of (b, kvh); the outputs of other pairs stay NaN / -1.
    Returns (O [B, Hq, d] float64, idx [B, Hkv, k] int64).
    """
    B, Hq, d = np.shape(Q)
    Hkv = np.shape(K)[1]
    G = Hq // Hkv
    O = np.full((B, Hq, d), np.nan)
    IDX = np.full((B, Hkv, k), -1, dtype=np.int64)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        o, idx, _ = socket_decode_pair(Q[b, h * G:(h + 1) * G], K[b, h], V[b, h], R,
                                       ids[b, h], norms[b, h], L, P, tau, k, scale)
        O[b, h * G:(h + 1) * G] = o
        IDX[b, h] = idx
    return O, IDX
