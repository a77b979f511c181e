"""Per-query-head index sets and the adaptive (cumulative-mass) k -- float64
CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Two selection variants around SOCKET's step 4 (SOCKET technical summary,
gist.science/ja/paper/2602.06283, section "中核メカニズム：ソフト LSH"):

* Per-query-head index sets. With grouped-query attention the main path
  chooses one index set per KV head from the group-summed soft table. Here
  every query head h scores the keys with its own soft assignment,
  score_{h,i} = |v_i| sum_l p_{h,l}(id_l(i)), takes its own top-k and attends
  over its own subset. For a group of one head the two agree.

* Adaptive k (Tactic digest, "Tactic: Adaptive Sparse Attention with
  Clustering and Distribution Fitting for Long-Context LLMs",
  aibr.jp/archives/79195, section 3 "中核となる技術的要素":
  the cumulative score p(I) = sum_{i in I} s_i of a token set I, and tokens
  are chosen until a target value of it is met, independently per head and
  query). Applied to SOCKET's soft scores: with s_i = score_i / sum_j score_j,
  k is the smallest count whose top-k by score (ties to the lower index)
  reaches the target mass fraction rho:

      k = min{ k >= 0 : sum of the k largest scores >= rho * sum of all },

  then clamped to [k_min, k_max] (and to N). The top-k set itself is the
  deterministic top-k of step 4 with that k.
"""

from __future__ import annotations

import numpy as np

from .attention_ref import attend_subset
from .socket_ref import bucket_probabilities, group_bucket_table, select_topk, soft_collision_scores


def per_head_scores(Qg, R, ids, norms, L: int, P: int, tau: float) -> np.ndarray:
    """score[h, i] = norms_i * sum_l p_{h,l}(ids[i, l]) for every head of the group: [G, N]."""
    Qg = np.asarray(Qg, dtype=np.float64)
    return np.stack([soft_collision_scores(bucket_probabilities(q, R, L, P, tau), ids, norms) for q in Qg])


def socket_decode_pair_per_head(Qg, K, V, R, ids, norms, L, P, tau, k, scale):
    """Decode of one (batch, kv-head) pair with one index set per query head.

    Returns (O [G, d], idx [G, k] ascending, scores [G, N]).
    """
    Qg = np.asarray(Qg, dtype=np.float64)
    scores = per_head_scores(Qg, R, ids, norms, L, P, tau)
    idx = np.stack([select_topk(s, k) for s in scores])
    O = np.stack([attend_subset(Qg[h:h + 1], K, V, idx[h], scale)[0] for h in range(Qg.shape[0])])
    return O, idx, scores


def adaptive_k(scores, mass: float, k_min: int, k_max: int) -> int:
    """Smallest k whose top-k scores hold the fraction `mass` of the total,
    clamped to [k_min, min(k_max, N)].

    The cumulative sums run over the scores in descending order (ties in
    index order) in float64. If rounding keeps the full sum below the target,
    the count is N.
    """
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.argsort(-s, kind="stable")
    cum = np.cumsum(s[order])
    target = mass * s.sum()
    if target <= 0.0:
        k = 0
    else:
        hit = np.nonzero(cum >= target)[0]
        k = int(hit[0]) + 1 if hit.size else n
    return int(max(k_min, min(k, k_max, n)))


def select_adaptive(scores, mass: float, k_min: int, k_max: int):
    """(ascending index set, k): the deterministic top-k with the adaptive k."""
    k = adaptive_k(scores, mass, k_min, k_max)
    return select_topk(scores, k), k


def socket_decode_pair_adaptive(Qg, K, V, R, ids, norms, L, P, tau, mass, k_min, k_max, scale, per_head=False):
    """Decode of one pair with the adaptive k: one unit (the group, from the
    group-summed table) or one unit per query head (per_head). Returns a list
    of (O [g, d], idx, k, scores) per unit, g = G or 1."""
    Qg = np.asarray(Qg, dtype=np.float64)
    if per_head:
        units = [(Qg[h:h + 1], per_head_scores(Qg[h:h + 1], R, ids, norms, L, P, tau)[0]) for h in range(len(Qg))]
    else:
        units = [(Qg, soft_collision_scores(group_bucket_table(Qg, R, L, P, tau), ids, norms))]
    out = []
    for q, s in units:
        idx, k = select_adaptive(s, mass, k_min, k_max)
        out.append((attend_subset(q, K, V, idx, scale), idx, k, s))
    return out
