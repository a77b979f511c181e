"""Pins of the attention and hard-hash oracles, and end-to-end oracle checks."""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention_ref as ao
from oracle import hata_ref as ho
from oracle import socket_ref as so
from tests.conftest import GOLDEN
from hash_scored_top_b200 import workloads as wl


# ----------------------------------------------------------------- exact attention

def test_attention_brute_force_math_exp():
    rng = np.random.default_rng(20)
    d, m = 6, 9
    q = rng.standard_normal(d)
    Ks = rng.standard_normal((m, d))
    Vs = rng.standard_normal((m, d))
    scale = 0.7
    logits = [scale * math.fsum(q[c] * Ks[i, c] for c in range(d)) for i in range(m)]
    w = [math.exp(a) for a in logits]                 # no max shift: small logits here
    Z = math.fsum(w)
    want = [math.fsum(w[i] * Vs[i, c] for i in range(m)) / Z for c in range(d)]
    assert np.allclose(ao.exact_attention(q, Ks, Vs, scale), want, rtol=1e-13, atol=1e-15)


def test_attention_special_cases():
    rng = np.random.default_rng(21)
    d = 16
    q = rng.standard_normal(d)
    K = rng.standard_normal((30, d))
    V = rng.standard_normal((30, d))
    # a single selected key returns its value row
    assert np.array_equal(ao.attend_subset(q[None], K, V, [17], 0.1)[0], V[17])
    # identical selected keys: uniform weights, the mean of the selected values
    Kt = np.repeat(K[:1], 30, axis=0)
    assert np.allclose(ao.attend_subset(q[None], Kt, V, [2, 5, 11], 0.3)[0],
                       V[[2, 5, 11]].mean(axis=0), rtol=1e-13)
    # zero scale: the mean of all values
    assert np.allclose(ao.exact_attention(q, K, V, 0.0), V.mean(axis=0), rtol=1e-12)
    # a dominant logit selects its value row; huge logits must not overflow
    K2 = K.copy()
    K2[4] = 1e4 * q
    assert np.allclose(ao.exact_attention(q, K2, V, 1.0), V[4], rtol=0, atol=1e-12)


def test_dense_decode_gqa_mapping():
    rng = np.random.default_rng(22)
    B, Hq, Hkv, N, d = 2, 6, 3, 12, 8
    Q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N + 4, d))
    V = rng.standard_normal((B, Hkv, N + 4, d))
    O = ao.dense_decode(Q, K, V, 0.5, N=N)
    from scipy.special import softmax
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            w = softmax(K[b, kv, :N] @ Q[b, h] * 0.5)
            assert np.allclose(O[b, h], w @ V[b, kv, :N], rtol=1e-12)


# ----------------------------------------------------------------- hard hash

def test_hata_codes_golden_basis():
    with open(os.path.join(GOLDEN, "hata_codes_basis.json")) as f:
        fx = json.load(f)
    R = np.eye(128)
    even = np.where(np.arange(128) % 2 == 0, 1.0, -1.0)
    xs = {"85": even, "170": -even, "255": np.ones(128)}
    want = {"85": 85, "170": 170, "255": 255}
    codes = {}
    for key, x in xs.items():
        c, _ = ho.binary_codes(x[None], R)
        assert c.dtype == np.uint8 and c.shape == (1, 16)
        assert np.all(c == want[key])
        codes[key] = c
    for a, b, matches in fx["match_scores"]["pairs"]:
        assert ho.hamming_match_scores(codes[a], codes[b])[0] == matches


def test_hata_scores_brute_force_python_bits():
    rng = np.random.default_rng(23)
    G, n = 3, 40
    q = rng.integers(0, 256, size=(G, 16), dtype=np.uint8)
    k = rng.integers(0, 256, size=(n, 16), dtype=np.uint8)
    got = ho.hamming_match_scores(q, k)
    for i in range(n):
        want = 0
        for h in range(G):
            qi = int.from_bytes(q[h].tobytes(), "little")
            ki = int.from_bytes(k[i].tobytes(), "little")
            want += 128 - bin(qi ^ ki).count("1")
        assert got[i] == want


def test_hata_self_and_complement():
    rng = np.random.default_rng(24)
    d = 64
    R = rng.standard_normal((128, d))
    Qg = rng.standard_normal((4, d))
    qc, proj = ho.binary_codes(Qg, R)
    assert np.all(proj != 0)
    kc, _ = ho.binary_codes(np.concatenate([Qg, -Qg]), R)
    s = ho.hamming_match_scores(qc[:1], kc)
    assert s[0] == 128 and s[4] == 0
    # a key equal to a query head scores 128 for that head
    s_all = ho.hamming_match_scores(qc, kc[:4])
    for h in range(4):
        assert s_all[h] >= 128
    assert np.all(s_all <= 128 * 4)


# ----------------------------------------------------------------- end to end with the workloads

def _oracle_pair(w, inp, b, h):
    G = w.G
    K = inp["K"][b, h, :w.N].double().numpy()
    V = inp["V"][b, h, :w.N].double().numpy()
    Qg = inp["Q"][b, h * G:(h + 1) * G].double().numpy()
    R = inp["R"].double().numpy()
    ids, _ = so.hash_key_ids(K, R, w.L, w.P)
    norms = so.value_norms_f16(V)
    return so.socket_decode_pair(Qg, K, V, R, ids, norms, w.L, w.P, w.tau, w.k, w.scale)


def test_planted_needles_selected_tiny():
    """The needle-in-a-haystack check: every planted needle key is selected."""
    w = wl.TINY_F32
    inp = wl.make_inputs(w, "cpu")
    O, idx, scores = _oracle_pair(w, inp, 0, 0)
    needles = set(inp["needle_pos"][0, 0].tolist())
    assert needles <= set(idx.tolist())
    assert len(idx) == w.k and np.all(np.diff(idx) > 0)


def test_planted_needles_selected_gqa_pair():
    w = wl.shrink(wl.LLAMA_8B, B=1, Hkv=1, Hq=4, N=16384, k=16384 // 33)
    inp = wl.make_inputs(w, "cpu")
    _, idx, _ = _oracle_pair(w, inp, 0, 0)
    assert set(inp["needle_pos"][0, 0].tolist()) <= set(idx.tolist())


def test_oracle_is_deterministic():
    w = wl.shrink(wl.LLAMA_1B, B=1, Hkv=2, Hq=8, N=2048, k=62)
    a = wl.make_inputs(w, "cpu")
    b = wl.make_inputs(w, "cpu")
    for key in ("Q", "K", "V", "R"):
        assert torch.equal(a[key], b[key])
    o1, i1, _ = _oracle_pair(w, a, 0, 1)
    o2, i2, _ = _oracle_pair(w, b, 0, 1)
    assert np.array_equal(i1, i2) and np.array_equal(o1, o2)
