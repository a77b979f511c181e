"""Pins of the per-query-head and adaptive-k selection oracle.

Expected values come from closed forms (uniform and geometric score
sequences), hand-built cases, pure-Python loops over a sorted list, and
reductions to other oracle functions that the pins of test_oracle_socket.py
already hold (a group of one head; a group whose heads are equal).
"""

import math

import numpy as np
import pytest
from scipy.special import softmax

from oracle import selection_ref as sr
from oracle import socket_ref as so


def _pair(seed, G=4, N=300, d=32, L=6, P=3):
    rng = np.random.default_rng(seed)
    Qg = rng.standard_normal((G, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    R = rng.standard_normal((L * P, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    norms = so.value_norms_f16(V)
    return Qg, K, V, R, ids, norms


# ---------------------------------------------------------------- per-head index sets

def test_per_head_with_one_head_is_the_group_decode():
    Qg, K, V, R, ids, norms = _pair(1, G=1)
    o, idx, s = sr.socket_decode_pair_per_head(Qg, K, V, R, ids, norms, 6, 3, 0.5, 40, 0.3)
    o_g, idx_g, s_g = so.socket_decode_pair(Qg, K, V, R, ids, norms, 6, 3, 0.5, 40, 0.3)
    np.testing.assert_array_equal(idx[0], idx_g)
    np.testing.assert_allclose(s[0], s_g, rtol=1e-13)
    np.testing.assert_allclose(o, o_g, rtol=1e-12, atol=1e-14)


def test_per_head_with_equal_heads_is_the_group_selection():
    # G copies of one query: the group table is G times each head's table, so
    # every head picks the group's set; each head's output is the group's
    Qg, K, V, R, ids, norms = _pair(2, G=1)
    Q4 = np.repeat(Qg, 4, axis=0)
    o, idx, s = sr.socket_decode_pair_per_head(Q4, K, V, R, ids, norms, 6, 3, 0.5, 25, 0.3)
    o_g, idx_g, s_g = so.socket_decode_pair(Q4, K, V, R, ids, norms, 6, 3, 0.5, 25, 0.3)
    for h in range(4):
        np.testing.assert_array_equal(idx[h], idx_g)
        np.testing.assert_allclose(4 * s[h], s_g, rtol=1e-13)
        np.testing.assert_allclose(o[h], o_g[h], rtol=1e-12, atol=1e-14)


def test_per_head_scores_follow_each_head_and_its_softmax():
    # head order permutes the per-head results; each output row is the
    # scipy softmax of that head's scaled logits over its own set
    Qg, K, V, R, ids, norms = _pair(3, G=3)
    o, idx, s = sr.socket_decode_pair_per_head(Qg, K, V, R, ids, norms, 6, 3, 0.4, 30, 0.25)
    o2, idx2, s2 = sr.socket_decode_pair_per_head(Qg[::-1], K, V, R, ids, norms, 6, 3, 0.4, 30, 0.25)
    np.testing.assert_array_equal(idx2, idx[::-1])
    np.testing.assert_allclose(o2, o[::-1], rtol=1e-12, atol=1e-14)
    assert not np.array_equal(idx[0], idx[1])       # the heads disagree on this draw
    for h in range(3):
        w = softmax(0.25 * K[idx[h]] @ Qg[h])
        np.testing.assert_allclose(o[h], w @ V[idx[h]], rtol=1e-12, atol=1e-14)
        # the head's scores: its own table, looked up per key
        p = so.bucket_probabilities(Qg[h], R, 6, 3, 0.4)
        want = [float(norms[i]) * math.fsum(p[l, ids[i, l]] for l in range(6)) for i in range(len(K))]
        np.testing.assert_allclose(s[h], want, rtol=1e-14)


# ---------------------------------------------------------------- adaptive k

@pytest.mark.parametrize("N,rho", [(100, 0.305), (1000, 0.9003), (37, 0.5), (64, 0.999)])
def test_adaptive_k_uniform_scores(N, rho):
    # N equal scores: the top-k hold k / N of the mass, so k = ceil(rho N)
    k = sr.adaptive_k(np.full(N, 0.7), rho, 1, N)
    assert k == math.ceil(rho * N)


@pytest.mark.parametrize("r,N,rho", [(0.9, 200, 0.5), (0.99, 1000, 0.8), (0.5, 40, 0.95)])
def test_adaptive_k_geometric_scores(r, N, rho):
    # s_i = r^i (shuffled): the top k hold (1 - r^k) / (1 - r^N) of the mass,
    # so k = ceil(log(1 - rho (1 - r^N)) / log r)
    rng = np.random.default_rng(int(1000 * r) + N)
    s = r ** rng.permutation(N).astype(np.float64)
    x = math.log(1 - rho * (1 - r ** N)) / math.log(r)
    assert abs(x - round(x)) > 1e-6          # not at a boundary
    assert sr.adaptive_k(s, rho, 1, N) == math.ceil(x)


def test_adaptive_k_one_dominant_key_and_clamps():
    s = np.array([1.0, 100.0, 1.0, 1.0])
    assert sr.adaptive_k(s, 0.9, 1, 4) == 1          # 100 / 103 >= 0.9
    assert sr.adaptive_k(s, 0.98, 1, 4) == 2         # 100 / 103 < 0.98 <= 101 / 103
    assert sr.adaptive_k(s, 0.9, 3, 4) == 3          # k_min
    assert sr.adaptive_k(s, 1.0, 1, 2) == 2          # k_max
    assert sr.adaptive_k(s, 1.0, 1, 99) == 4         # N
    idx, k = sr.select_adaptive(s, 0.9, 1, 4)
    assert k == 1 and idx.tolist() == [1]


def test_adaptive_selection_ties_go_to_lower_indices():
    s = np.array([1.0, 2.0, 2.0, 2.0, 1.0, 2.0])
    # total 10; target 0.5 -> 5 needs three of the 2s: keys 1, 2, 3
    idx, k = sr.select_adaptive(s, 0.5, 1, 6)
    assert k == 3 and idx.tolist() == [1, 2, 3]
    idx, k = sr.select_adaptive(s, 0.85, 1, 6)        # 8.5 -> four 2s and one 1 (key 0)
    assert k == 5 and idx.tolist() == [0, 1, 2, 3, 5]


@pytest.mark.parametrize("seed", range(6))
def test_adaptive_k_matches_a_python_loop(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 60))
    s = rng.choice([0.0, 0.5, 1.0, 3.0], size=n) * rng.integers(1, 4, size=n)
    rho = float(rng.uniform(0.05, 1.0))
    k_min, k_max = int(rng.integers(1, 4)), int(rng.integers(4, 80))
    # the loop: repeatedly take the largest remaining score (lowest index
    # first), stop once the running sum reaches the target
    total = math.fsum(s)
    left = list(range(n))
    run, k = 0.0, 0
    while left and run < rho * total:
        best = max(left, key=lambda i: (s[i], -i))
        left.remove(best)
        run += s[best]
        k += 1
    want = max(k_min, min(k, k_max, n))
    assert sr.adaptive_k(s, rho, k_min, k_max) == want
    idx, kk = sr.select_adaptive(s, rho, k_min, k_max)
    assert kk == want and len(idx) == want and np.all(np.diff(idx) > 0)


def test_adaptive_decode_units():
    Qg, K, V, R, ids, norms = _pair(4, G=2)
    group = sr.socket_decode_pair_adaptive(Qg, K, V, R, ids, norms, 6, 3, 0.5, 0.3, 2, 300, 0.2)
    assert len(group) == 1
    o, idx, k, s = group[0]
    o_g, idx_g, s_g = so.socket_decode_pair(Qg, K, V, R, ids, norms, 6, 3, 0.5, k, 0.2)
    np.testing.assert_array_equal(idx, idx_g)
    np.testing.assert_allclose(o, o_g, rtol=1e-12, atol=1e-14)
    heads = sr.socket_decode_pair_adaptive(Qg, K, V, R, ids, norms, 6, 3, 0.5, 0.3, 2, 300, 0.2, per_head=True)
    assert len(heads) == 2
    for h, (oh, idxh, kh, sh) in enumerate(heads):
        o1, idx1, _ = sr.socket_decode_pair_per_head(Qg[h:h + 1], K, V, R, ids, norms, 6, 3, 0.5, kh, 0.2)
        np.testing.assert_array_equal(idxh, idx1[0])
        np.testing.assert_allclose(oh, o1, rtol=1e-12, atol=1e-14)
        assert kh == sr.adaptive_k(sh, 0.3, 2, 300)
