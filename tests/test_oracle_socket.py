"""Pins of the SOCKET oracle against closed forms, invariants and brute force.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or bit order, a transposed operand, the softmax over the wrong
axis, double rounding of the norm) fails at least one of them. None of them
re-types the oracle's own formula: they use hand-worked fixtures, identities
that hold for the method (factorisation of the bucket softmax over bits, the
tau -> 0 and tau -> infinity limits), and independent brute force.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import socket_ref as so
from tests.conftest import GOLDEN


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


# ----------------------------------------------------------------- hashing (step 1)

def test_hash_ids_golden_basis():
    fx = _load("hash_ids_basis.json")
    for case in fx["cases"]:
        R = np.eye(4)
        ids, _ = so.hash_key_ids(np.array([case["key"]]), R, case["L"], case["P"])
        assert ids[0].tolist() == case["ids"], case["why"]


def test_hash_ids_negation_flips_every_bit():
    rng = np.random.default_rng(1)
    L, P, d = 6, 5, 16
    K = rng.standard_normal((200, d))
    R = rng.standard_normal((L * P, d))
    ids, proj = so.hash_key_ids(K, R, L, P)
    assert np.all(proj != 0)
    ids_neg, _ = so.hash_key_ids(-K, R, L, P)
    assert np.array_equal(ids_neg, ids ^ ((1 << P) - 1))


def test_hash_ids_scale_invariant_and_self_hyperplane():
    rng = np.random.default_rng(2)
    L, P, d = 4, 8, 32
    K = rng.standard_normal((64, d))
    R = rng.standard_normal((L * P, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    ids2, _ = so.hash_key_ids(7.5 * K, R, L, P)
    assert np.array_equal(ids, ids2)
    # a key equal to hyperplane j of table l projects to |r|^2 > 0 on it
    for l in range(L):
        for j in range(P):
            i, _ = so.hash_key_ids(R[l * P + j][None, :], R, L, P)
            assert (i[0, l] >> j) & 1 == 1


def test_hash_ids_brute_force_fsum():
    rng = np.random.default_rng(3)
    L, P, d = 3, 3, 8
    K = rng.standard_normal((10, d))
    R = rng.standard_normal((L * P, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    for n in range(K.shape[0]):
        for l in range(L):
            want = 0
            for j in range(P):
                dot = math.fsum(float(K[n, c]) * float(R[l * P + j, c]) for c in range(d))
                if dot > 0:
                    want |= 1 << j
            assert ids[n, l] == want


# ----------------------------------------------------------------- value norms

def test_value_norms_golden_rounding():
    fx = _load("value_norm_f16.json")
    for case in fx["cases"]:
        got = so.value_norms_f16(np.array([case["v"]], dtype=np.float64))[0]
        want = np.float16(np.inf) if case["norm_f16"] == "inf" else np.float16(case["norm_f16"])
        assert got.dtype == np.float16
        assert got == want or (np.isinf(got) and np.isinf(want)), case["why"]


def test_value_norms_match_scipy_norm_rounded():
    from scipy.linalg import norm
    rng = np.random.default_rng(4)
    V = rng.standard_normal((50, 128)) * 3
    got = so.value_norms_f16(V)
    want = np.array([np.float16(norm(v)) for v in V])
    assert np.array_equal(got, want)


# ----------------------------------------------------------------- soft assignment (step 2)

def test_soft_assignment_golden_2d():
    fx = _load("soft_assignment_2d.json")
    R = np.eye(2)
    for case in fx["cases"]:
        p = so.bucket_probabilities(np.array(case["q"]), R, 1, 2, case["tau"])
        assert np.allclose(p[0], case["p"], rtol=0, atol=fx["tolerance"])


@pytest.mark.parametrize("P,tau", [(1, 0.3), (4, 0.5), (8, 0.3), (8, 0.2), (10, 1.0)])
def test_soft_assignment_factorises_over_bits(P, tau):
    """p_l(b) = prod_j sigmoid(2 s_bj z_j / tau): the softmax over sign patterns factorises."""
    rng = np.random.default_rng(10 + P)
    d, L = 16, 3
    q = rng.standard_normal(d)
    R = rng.standard_normal((L * P, d))
    p = so.bucket_probabilities(q, R, L, P, tau)
    qn = math.sqrt(math.fsum(x * x for x in q))
    for l in range(L):
        z = [math.fsum(R[l * P + j, c] * q[c] / qn for c in range(d)) for j in range(P)]
        for b in range(0, 1 << P, max(1, (1 << P) // 64)):
            prod = 1.0
            for j in range(P):
                s = 1.0 if (b >> j) & 1 else -1.0
                prod *= _sigmoid(2.0 * s * z[j] / tau)
            assert p[l, b] == pytest.approx(prod, rel=1e-11, abs=1e-300)
        assert math.fsum(p[l]) == pytest.approx(1.0, abs=1e-12)


def test_soft_assignment_single_bit_is_logistic():
    rng = np.random.default_rng(5)
    d = 8
    for _ in range(5):
        q = rng.standard_normal(d)
        r = rng.standard_normal((1, d))
        tau = 0.25
        p = so.bucket_probabilities(q, r, 1, 1, tau)
        z = float(r[0] @ (q / np.linalg.norm(q)))
        assert p[0, 1] == pytest.approx(1.0 / (1.0 + math.exp(-2 * z / tau)), rel=1e-13)
        assert p[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(2 * z / tau)), rel=1e-13)


def test_soft_assignment_limits():
    rng = np.random.default_rng(6)
    d, L, P = 32, 5, 6
    q = rng.standard_normal(d)
    R = rng.standard_normal((L * P, d))
    # tau -> infinity: uniform over the 2^P buckets
    p_hot = so.bucket_probabilities(q, R, L, P, 1e12)
    assert np.allclose(p_hot, 2.0 ** -P, rtol=1e-9)
    # tau -> 0: one-hot at the query's own hard bucket (its sign pattern)
    p_cold = so.bucket_probabilities(q, R, L, P, 1e-9)
    qh = q / np.linalg.norm(q)
    for l in range(L):
        hard = sum(1 << j for j in range(P) if float(R[l * P + j] @ qh) > 0)
        assert p_cold[l, hard] == pytest.approx(1.0, abs=1e-12)
        assert p_cold[l].sum() == pytest.approx(1.0, abs=1e-12)


def test_soft_assignment_uses_unit_query():
    rng = np.random.default_rng(7)
    q = rng.standard_normal(16)
    R = rng.standard_normal((8, 16))
    assert np.allclose(so.bucket_probabilities(q, R, 2, 4, 0.3),
                       so.bucket_probabilities(11.0 * q, R, 2, 4, 0.3), rtol=1e-13)


def test_group_table_is_sum_over_heads():
    rng = np.random.default_rng(8)
    Qg = rng.standard_normal((4, 16))
    R = rng.standard_normal((12, 16))
    T = so.group_bucket_table(Qg, R, 3, 4, 0.3)
    assert np.allclose(T.sum(axis=1), 4.0, atol=1e-12)        # each head's row sums to 1
    T_rev = so.group_bucket_table(Qg[::-1], R, 3, 4, 0.3)
    assert np.allclose(T, T_rev, rtol=1e-14)
    T1 = so.group_bucket_table(Qg[:1], R, 3, 4, 0.3)
    assert np.array_equal(T1, so.bucket_probabilities(Qg[0], R, 3, 4, 0.3))


# ----------------------------------------------------------------- scoring (step 3)

def test_scores_hand_example():
    T = np.array([[0.1, 0.9], [0.7, 0.3]])          # L = 2 tables, P = 1
    ids = np.array([[0, 0], [1, 0], [1, 1], [0, 1]])
    norms = np.array([1.0, 2.0, 0.5, 4.0], dtype=np.float16)
    got = so.soft_collision_scores(T, ids, norms)
    assert np.allclose(got, [0.8, 3.2, 0.6, 1.6], rtol=1e-15)


def test_scores_tau_to_zero_is_norm_times_hard_collisions():
    """Theorem 3's limit: as tau -> 0 the soft score is |v| times the hard collision count."""
    rng = np.random.default_rng(9)
    d, L, P, G, n = 32, 10, 4, 3, 300
    Qg = rng.standard_normal((G, d))
    R = rng.standard_normal((L * P, d))
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    norms = so.value_norms_f16(V)
    # keep the case away from projections where tau = 1e-6 is not yet a hard limit
    z = np.stack([R @ (q / np.linalg.norm(q)) for q in Qg])
    assert np.abs(z).min() > 1e-3
    T = so.group_bucket_table(Qg, R, L, P, 1e-6)
    s = so.soft_collision_scores(T, ids, norms)
    for i in range(n):
        coll = 0
        for h in range(G):
            for l in range(L):
                hard = sum(1 << j for j in range(P) if z[h, l * P + j] > 0)
                coll += int(ids[i, l] == hard)
        assert s[i] == pytest.approx(float(norms[i]) * coll, rel=1e-9, abs=1e-9)


def test_scores_bounds_and_uniform_limit():
    rng = np.random.default_rng(11)
    d, L, P, G, n = 16, 6, 3, 2, 100
    Qg = rng.standard_normal((G, d))
    R = rng.standard_normal((L * P, d))
    ids = rng.integers(0, 1 << P, size=(n, L))
    norms = np.abs(rng.standard_normal(n)).astype(np.float16)
    s = so.soft_collision_scores(so.group_bucket_table(Qg, R, L, P, 0.3), ids, norms)
    assert np.all(s >= 0) and np.all(s <= G * L * norms.astype(np.float64) + 1e-12)
    s_hot = so.soft_collision_scores(so.group_bucket_table(Qg, R, L, P, 1e12), ids, norms)
    assert np.allclose(s_hot, norms.astype(np.float64) * G * L / 2 ** P, rtol=1e-9)


# ----------------------------------------------------------------- selection (step 4)

def test_select_brute_force_with_ties():
    rng = np.random.default_rng(12)
    for trial in range(30):
        n = int(rng.integers(1, 64))
        s = rng.integers(0, 6, size=n).astype(np.float64)   # many exact ties
        for k in range(0, n + 1):
            want = sorted(sorted(range(n), key=lambda i: (-s[i], i))[:k])
            assert select_list(s, k) == want


def select_list(s, k):
    return so.select_topk(s, k).tolist()


def test_select_degenerate():
    assert select_list(np.full(10, 3.0), 4) == [0, 1, 2, 3]
    assert select_list(np.arange(10.0), 10) == list(range(10))
    assert select_list(np.arange(10.0), 0) == []
    assert select_list(np.arange(10.0), 3) == [7, 8, 9]
    with pytest.raises(ValueError):
        so.select_topk(np.arange(3.0), 4)


# ----------------------------------------------------------------- end to end

def test_decode_pair_full_selection_is_dense_softmax():
    """k = N: attention over the selection is ordinary softmax attention (scipy)."""
    from scipy.special import softmax
    rng = np.random.default_rng(13)
    G, d, N, L, P = 2, 16, 40, 4, 3
    Qg = rng.standard_normal((G, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    R = rng.standard_normal((L * P, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    norms = so.value_norms_f16(V)
    O, idx, _ = so.socket_decode_pair(Qg, K, V, R, ids, norms, L, P, 0.3, N, 0.25)
    assert idx.tolist() == list(range(N))
    for h in range(G):
        w = softmax(K @ Qg[h] * 0.25)
        assert np.allclose(O[h], w @ V, rtol=1e-12, atol=1e-14)
