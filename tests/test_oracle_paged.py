"""Pins of the paged KV gather oracle.

Expected values: a hand-built pool and page table read element by element,
the identity page table (which turns the pool back into the contiguous cache
of attention_ref, pinned in test_oracle_attention_hata.py), invariance under
any permutation of the physical pages, page size 1 and one page per pair, and
scipy's softmax.
"""

import numpy as np
import pytest
from scipy.special import softmax

from oracle import attention_ref as ao
from oracle import paged_ref as pr
from oracle import socket_ref as so


def test_paged_rows_hand_built():
    # 4 physical pages of 2 rows, d = 3; row r of page p holds (p, r, p + r)
    pool = np.array([[[p, r, p + r] for r in range(2)] for p in range(4)], dtype=np.float64)
    table = [3, 0, 2]                          # logical pages 0, 1, 2 -> physical 3, 0, 2
    rows = pr.paged_rows(pool, table, [0, 3, 4, 1, 5], 2)
    want = [[3, 0, 3], [0, 1, 1], [2, 0, 2], [3, 1, 4], [2, 1, 3]]
    np.testing.assert_array_equal(rows, want)


def _contiguous_to_pool(K, page_size, order):
    """Pages of K [N, d] (N a multiple of page_size) stored at physical slots `order`."""
    n_pages = K.shape[0] // page_size
    pool = np.zeros((n_pages, page_size, K.shape[1]))
    table = np.zeros(n_pages, dtype=np.int64)
    for logical, physical in enumerate(order):
        pool[physical] = K[logical * page_size:(logical + 1) * page_size]
        table[logical] = physical
    return pool, table


@pytest.mark.parametrize("page_size", [1, 4, 16, 64])
def test_paged_attention_equals_contiguous(page_size):
    rng = np.random.default_rng(page_size)
    N, d, G = 256, 16, 3
    K, V = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    Qg = rng.standard_normal((G, d))
    idx = np.sort(rng.choice(N, 37, replace=False))
    want = ao.attend_subset(Qg, K, V, idx, 0.25)
    n_pages = N // page_size
    for order in [np.arange(n_pages), rng.permutation(n_pages)]:
        Kp, table = _contiguous_to_pool(K, page_size, order)
        Vp, table_v = _contiguous_to_pool(V, page_size, order)
        assert np.array_equal(table, table_v)
        got = pr.attend_subset_paged(Qg, Kp, Vp, table, idx, page_size, 0.25)
        np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)
        # and the textbook softmax over the gathered rows
        for h in range(G):
            w = softmax(0.25 * K[idx] @ Qg[h])
            np.testing.assert_allclose(got[h], w @ V[idx], rtol=1e-12, atol=1e-14)


def test_one_page_per_pair_and_shared_pool():
    # two pairs in one pool, each with a single page of all its keys
    rng = np.random.default_rng(7)
    N, d = 32, 8
    K0, K1 = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    pool = np.stack([K1, K0])                 # pair 0 -> page 1, pair 1 -> page 0
    np.testing.assert_array_equal(pr.paged_rows(pool, [1], np.arange(N), N), K0)
    np.testing.assert_array_equal(pr.paged_rows(pool, [0], [5, 2], N), K1[[5, 2]])


def test_paged_decode_pair_matches_the_contiguous_decode():
    rng = np.random.default_rng(11)
    N, d, G, L, P, ps = 512, 32, 2, 8, 4, 32
    K, V = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    Qg = rng.standard_normal((G, d))
    R = rng.standard_normal((L * P, d))
    ids, _ = so.hash_key_ids(K, R, L, P)
    norms = so.value_norms_f16(V)
    order = rng.permutation(N // ps)
    Kp, table = _contiguous_to_pool(K, ps, order)
    Vp, _ = _contiguous_to_pool(V, ps, order)
    o, idx, s = pr.socket_decode_pair_paged(Qg, Kp, Vp, table, ps, R, ids, norms, L, P, 0.5, 40, 0.2)
    o_c, idx_c, s_c = so.socket_decode_pair(Qg, K, V, R, ids, norms, L, P, 0.5, 40, 0.2)
    np.testing.assert_array_equal(idx, idx_c)
    np.testing.assert_array_equal(s, s_c)
    np.testing.assert_allclose(o, o_c, rtol=1e-13, atol=1e-15)
