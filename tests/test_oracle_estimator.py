"""Pins of the soft-count attention estimator oracle (oracle/estimator_ref.py).

Expected values are worked by hand with math.exp or computed by pure-Python
loops written from the definition, never by the oracle itself.
"""

import math

import numpy as np

from oracle import estimator_ref as eo


def _sigmoid(x):
    return 1.0 / (1.0 + math.exp(-x))


def test_one_hyperplane_worked_case():
    """L = 1, P = 1, hyperplane e_0, q = e_0: z = 1, so bucket 1 (bit set)
    has probability sigmoid(2 / tau) and bucket 0 sigmoid(-2 / tau). The
    estimate is the values averaged with those weights."""
    d, tau = 4, 0.5
    R = np.zeros((1, d))
    R[0, 0] = 1.0
    q = np.array([1.0, 0.0, 0.0, 0.0])
    ids = np.array([[1], [0], [1], [0], [0]])
    V = np.arange(5 * d, dtype=np.float64).reshape(5, d) / 7.0
    idx = [0, 1, 3, 4]
    w1, w0 = _sigmoid(2.0 / tau), _sigmoid(-2.0 / tau)
    weights = {0: w1, 1: w0, 3: w0, 4: w0}
    want = [math.fsum(weights[i] * V[i, c] for i in idx) / math.fsum(weights.values()) for c in range(d)]
    got = eo.soft_count_attention(q[None], V, R, ids, idx, 1, 1, tau)[0]
    assert np.allclose(got, want, rtol=1e-14, atol=0)
    c = eo.soft_counts(q, R, ids, 1, 1, tau)
    assert np.allclose(c, [w1, w0, w1, w0, w0], rtol=1e-15)


def test_uniform_limit_is_the_mean_of_the_selected_values():
    """tau -> infinity makes every bucket equally likely: every key gets the
    count L / 2^P, and the estimate is the plain mean of the selected values."""
    rng = np.random.default_rng(51)
    G, d, N, L, P = 3, 16, 40, 5, 3
    Qg = rng.standard_normal((G, d))
    V = rng.standard_normal((N, d))
    R = rng.standard_normal((L * P, d))
    ids = rng.integers(0, 2 ** P, size=(N, L))
    idx = [1, 4, 9, 22, 39]
    c = eo.soft_counts(Qg[0], R, ids, L, P, 1e12)
    assert np.allclose(c, L / 2 ** P, rtol=1e-9)
    got = eo.soft_count_attention(Qg, V, R, ids, idx, L, P, 1e12)
    assert np.allclose(got, np.repeat(V[idx].mean(axis=0)[None], G, axis=0), rtol=1e-9, atol=1e-12)


def test_brute_force_loop_over_tables_and_buckets():
    """Pure-Python loops over heads, tables and sign patterns, with the
    softmax written out per table."""
    rng = np.random.default_rng(52)
    G, d, N, L, P, tau = 2, 6, 12, 3, 2, 0.7
    Qg = rng.standard_normal((G, d))
    V = rng.standard_normal((N, d))
    R = rng.standard_normal((L * P, d))
    ids = rng.integers(0, 2 ** P, size=(N, L))
    idx = [0, 3, 5, 6, 11]
    got = eo.soft_count_attention(Qg, V, R, ids, idx, L, P, tau)
    for h in range(G):
        qn = math.sqrt(math.fsum(x * x for x in Qg[h]))
        counts = []
        for i in idx:
            c = 0.0
            for l in range(L):
                z = [math.fsum(Qg[h, t] / qn * R[l * P + j, t] for t in range(d)) for j in range(P)]
                logits = []
                for b in range(2 ** P):
                    logits.append(sum((1.0 if (b >> j) & 1 else -1.0) * z[j] for j in range(P)) / tau)
                m = max(logits)
                e = [math.exp(x - m) for x in logits]
                c += e[ids[i, l]] / math.fsum(e)
            counts.append(c)
        want = [math.fsum(counts[n] * V[i, t] for n, i in enumerate(idx)) / math.fsum(counts) for t in range(d)]
        assert np.allclose(got[h], want, rtol=1e-12, atol=1e-14)
