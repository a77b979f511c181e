"""Pins of the oracle's composed functions: the hard-hash decode of one pair
and the batch wrappers with their query-head -> KV-head mapping.

The parts (codes, Hamming scores, top-k, subset attention, soft tables) are
pinned elsewhere; these tests pin how they are put together. A wrong operand
(query codes taken from the keys, or from the wrong hyperplane matrix), a
wrong head slice of a group, or a wrong KV head for a query head fails one of
them. Expected values come from hand-built codes and scipy's softmax, never
from the oracle itself.
"""

import numpy as np
import pytest
from scipy.special import softmax

from oracle import hata_ref as ho
from oracle import socket_ref as so


def _softmax_attention(q, Ks, Vs, scale):
    return softmax(Ks @ q * scale) @ Vs


# ----------------------------------------------------------------- hard-hash decode of one pair

def _bits_to_codes(bits):
    """[n, 128] 0/1 -> [n, 16] uint8, bit m in byte m // 8 at bit m % 8 (written out, no numpy packbits)."""
    bits = np.asarray(bits, dtype=np.int64)
    out = np.zeros((bits.shape[0], 16), dtype=np.uint8)
    for i in range(bits.shape[0]):
        for m in range(128):
            if bits[i, m]:
                out[i, m // 8] |= np.uint8(1 << (m % 8))
    return out


def test_hata_decode_pair_hand_built_codes():
    """Identity hyperplanes (d = 128) make a query's code its sign pattern, so
    the match count of a hand-built key code is known by construction."""
    d, G, N, k, scale = 128, 2, 12, 4, 0.3
    rng = np.random.default_rng(31)
    R128 = np.eye(d)
    mag = rng.uniform(0.5, 2.0, size=(G, d))
    sgn = np.where(rng.integers(0, 2, size=(G, d)) == 1, 1.0, -1.0)
    Qg = mag * sgn
    qbits = (sgn > 0).astype(np.int64)                   # the query codes, by construction
    # key i agrees with head 0 on a[i] bits and with head 1 on b[i] bits: flip
    # a chosen number of head 0's bits (heads agree on no bit: head 1 = ~head 0)
    Qg[1] = -Qg[0]
    qbits[1] = 1 - qbits[0]
    flips = [0, 5, 64, 3, 127, 30, 5, 100, 2, 64, 7, 128]
    kbits = np.zeros((N, d), dtype=np.int64)
    for i, f in enumerate(flips):
        kbits[i] = qbits[0]
        kbits[i, :f] = 1 - kbits[i, :f]
    kcodes = _bits_to_codes(kbits)
    # score = (128 - f) + f = 128 for every key: all tie, so the lowest indices win
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    O, idx, scores = ho.hata_decode_pair(Qg, K, V, R128, kcodes, k, scale)
    assert scores.tolist() == [128] * N
    assert idx.tolist() == [0, 1, 2, 3]
    # now make head 1 agree with head 0: score = 2 * (128 - f)
    Qg[1] = Qg[0] * 0.5
    O, idx, scores = ho.hata_decode_pair(Qg, K, V, R128, kcodes, k, scale)
    assert scores.tolist() == [2 * (128 - f) for f in flips]
    # the 4 largest: f = 0, 2, 3, 5 (indices 0, 8, 3, and the first f = 5 at index 1)
    assert idx.tolist() == [0, 1, 3, 8]
    for h in range(G):
        want = _softmax_attention(Qg[h], K[[0, 1, 3, 8]], V[[0, 1, 3, 8]], scale)
        assert np.allclose(O[h], want, rtol=1e-12, atol=1e-14)


def test_hata_decode_pair_planted_query_key_is_selected():
    """A key equal to a query head matches all 128 of that head's bits; with
    random hyperplanes and k = 1 it is the selection, and the output is its value."""
    rng = np.random.default_rng(32)
    d, G, N = 64, 3, 500
    R128 = rng.standard_normal((128, d))
    Qg = rng.standard_normal((G, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    pos = 317
    K[pos] = Qg[1]
    # G identical query heads make the planted key score the maximum 128 * G
    Qs = np.repeat(Qg[1:2], G, axis=0)
    kcodes, _ = ho.binary_codes(K, R128)
    O, idx, scores = ho.hata_decode_pair(Qs, K, V, R128, kcodes, 1, d ** -0.5)
    assert idx.tolist() == [pos] and scores[pos] == 128 * G
    assert np.array_equal(O, np.repeat(V[pos][None], G, axis=0))
    # with the distinct heads the planted key still matches head 1 fully
    O, idx, scores = ho.hata_decode_pair(Qg, K, V, R128, kcodes, 8, d ** -0.5)
    assert pos in idx.tolist()
    qc, _ = ho.binary_codes(Qg[1:2], R128)
    assert np.array_equal(qc[0], kcodes[pos])


# ----------------------------------------------------------------- batch wrappers

def _random_batch(seed, B=2, Hq=6, Hkv=3, N=50, d=16, L=4, P=3):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    R = rng.standard_normal((L * P, d))
    return Q, K, V, R


def test_socket_decode_batch_head_mapping():
    """Query head h reads KV head h // G, and the selection of KV head j uses
    the tables of query heads j*G .. j*G + G - 1: checked head by head with
    scipy's softmax over the selected rows, and the index set against the top-k
    of the group's soft scores."""
    B, Hq, Hkv, N, d, L, P, tau, k, scale = 2, 6, 3, 50, 16, 4, 3, 0.4, 9, 0.25
    Q, K, V, R = _random_batch(41, B, Hq, Hkv, N, d, L, P)
    ids = np.zeros((B, Hkv, N, L), dtype=np.int64)
    norms = np.zeros((B, Hkv, N), dtype=np.float16)
    for b in range(B):
        for j in range(Hkv):
            ids[b, j], _ = so.hash_key_ids(K[b, j], R, L, P)
            norms[b, j] = so.value_norms_f16(V[b, j])
    O, IDX = so.socket_decode(Q, K, V, R, ids, norms, L, P, tau, k, scale)
    G = Hq // Hkv
    for b in range(B):
        for j in range(Hkv):
            T = so.group_bucket_table(Q[b, j * G:(j + 1) * G], R, L, P, tau)
            s = so.soft_collision_scores(T, ids[b, j], norms[b, j])
            want = sorted(sorted(range(N), key=lambda i: (-s[i], i))[:k])
            assert IDX[b, j].tolist() == want
        for h in range(Hq):
            j = h // G
            sel = IDX[b, j]
            assert np.allclose(O[b, h], _softmax_attention(Q[b, h], K[b, j][sel], V[b, j][sel], scale),
                               rtol=1e-12, atol=1e-14)
    # the selection differs between KV heads (so a wrong mapping could not pass by accident)
    assert not np.array_equal(IDX[0, 0], IDX[0, 1])
    # a subset of pairs leaves the others untouched
    O2, IDX2 = so.socket_decode(Q, K, V, R, ids, norms, L, P, tau, k, scale, pairs=[(1, 2)])
    assert np.array_equal(IDX2[1, 2], IDX[1, 2]) and np.all(IDX2[0] == -1)
    assert np.array_equal(O2[1, 4:6], O[1, 4:6]) and np.isnan(O2[0]).all() and np.isnan(O2[1, :4]).all()


def test_hata_decode_batch_head_mapping():
    B, Hq, Hkv, N, d, k, scale = 2, 8, 2, 60, 32, 6, 0.2
    rng = np.random.default_rng(42)
    Q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    R128 = rng.standard_normal((128, d))
    kcodes = np.zeros((B, Hkv, N, 16), dtype=np.uint8)
    for b in range(B):
        for j in range(Hkv):
            kcodes[b, j], _ = ho.binary_codes(K[b, j], R128)
    O, IDX = ho.hata_decode(Q, K, V, R128, kcodes, k, scale)
    G = Hq // Hkv
    for b in range(B):
        for j in range(Hkv):
            # matches counted bit by bit from the projection signs
            qbits = (Q[b, j * G:(j + 1) * G] @ R128.T > 0)
            kbits = (K[b, j] @ R128.T > 0)
            s = np.array([sum(int((qbits[h] == kbits[i]).sum()) for h in range(G)) for i in range(N)])
            want = sorted(sorted(range(N), key=lambda i: (-s[i], i))[:k])
            assert IDX[b, j].tolist() == want
        for h in range(Hq):
            j = h // G
            sel = IDX[b, j]
            assert np.allclose(O[b, h], _softmax_attention(Q[b, h], K[b, j][sel], V[b, j][sel], scale),
                               rtol=1e-12, atol=1e-14)
    assert not np.array_equal(IDX[0, 0], IDX[0, 1])
