"""HATA-style hard-hash (Hamming) scoring and decode -- CPU oracle.

TEST INFRASTRUCTURE: see the package docstring for who may import this.

Source: HATA digest ("HATA: Hash-Aware Top-k Attention",
aibr.jp/archives/117328), section 3 "中核となる技術的要素": queries and keys
are mapped to binary hash codes, and the top-k keys are ranked by comparing
codes instead of computing exact q.k scores; section 2 states that only the
rank order has to be preserved. The learned hash functions of the page need
training and weights; seeded random hyperplanes stand in for them. Readings
(each one pinned by a test):

* code bit m of a row x is [x . r_m > 0] for 128 hyperplanes r_m, packed
  least significant bit first: bit m goes to byte m // 8, bit m % 8;
* the similarity of a query head and a key is the number of equal code bits,
  128 - Hamming distance; with grouped-query attention the key's score is the
  sum over the group's query heads (larger is better, no value-norm weight);
* selection and exact attention are the SOCKET steps (ties to lower index).
"""

from __future__ import annotations

import numpy as np

from .attention_ref import attend_subset
from .socket_ref import select_topk

CODE_BITS = 128
CODE_BYTES = CODE_BITS // 8


def binary_codes(X, R128):
    """128-bit sign codes of the rows of X.

    X: [n, d]; R128: [128, d]. Returns (codes [n, 16] uint8, proj [n, 128]
    float64) with bit m of the code equal to [proj[:, m] > 0].
    """
    X = np.asarray(X, dtype=np.float64)
    R128 = np.asarray(R128, dtype=np.float64)
    if R128.shape[0] != CODE_BITS:
        raise ValueError("R128 must have 128 rows")
    proj = X @ R128.T
    bits = (proj > 0).astype(np.uint8).reshape(X.shape[0], CODE_BYTES, 8)
    weights = (1 << np.arange(8)).astype(np.uint8)
    codes = (bits * weights).sum(axis=2).astype(np.uint8)
    return codes, proj


def _popcount8(x: np.ndarray) -> np.ndarray:
    """Number of set bits of each uint8 (via unpackbits)."""
    return np.unpackbits(np.asarray(x, dtype=np.uint8)[..., None], axis=-1).sum(axis=-1)


def hamming_match_scores(qcodes, kcodes) -> np.ndarray:
    """Score of each key: sum over query heads of the number of equal code bits.

    qcodes: [G, 16] uint8; kcodes: [n, 16] uint8. Returns int64 [n] in [0, 128*G].
    """
    qcodes = np.asarray(qcodes, dtype=np.uint8)
    kcodes = np.asarray(kcodes, dtype=np.uint8)
    total = np.zeros(kcodes.shape[0], dtype=np.int64)
    for h in range(qcodes.shape[0]):
        hamming = _popcount8(np.bitwise_xor(kcodes, qcodes[h][None, :])).sum(axis=1)
        total += CODE_BITS - hamming.astype(np.int64)
    return total


def hata_decode_pair(Qg, K, V, R128, kcodes, k, scale):
    """One (batch, kv-head) pair: query codes, Hamming scores, top-k, attention.

    Returns (O [G, d], idx [k], scores [N] int64).
    """
    qcodes, _ = binary_codes(Qg, R128)
    scores = hamming_match_scores(qcodes, kcodes)
    idx = select_topk(scores.astype(np.float64), k)
    O = attend_subset(Qg, K, V, idx, scale)
    return O, idx, scores


def hata_decode(Q, K, V, R128, kcodes, k, scale, pairs=None):
    """Batch version: Q [B, Hq, d], K/V [B, Hkv, N, d], kcodes [B, Hkv, N, 16]."""
    B, Hq, d = np.shape(Q)
    Hkv = np.shape(K)[1]
    G = Hq // Hkv
    O = np.full((B, Hq, d), np.nan)
    IDX = np.full((B, Hkv, k), -1, dtype=np.int64)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        o, idx, _ = hata_decode_pair(Q[b, h * G:(h + 1) * G], K[b, h], V[b, h], R128,
                                     kcodes[b, h], k, scale)
        O[b, h * G:(h + 1) * G] = o
        IDX[b, h] = idx
    return O, IDX
