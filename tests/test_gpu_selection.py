"""GPU parity of the selection variants against the oracle, through the C ABI:
per-query-head index sets (socket_decode_heads) and the adaptive k
(socket_decode_adaptive, group and per-head units).

The adaptive k is an integer decided by floating-point sums. The GPU scores
are f32 (relative error below 6e-7 against the oracle's float64 scores), so
the test accepts any k between the oracle's smallest k whose cumulative mass
reaches mass * S * (1 - 2e-6) and the smallest reaching mass * S * (1 + 2e-6),
both clamped as the entry point clamps; for that k the index set must be a
valid top-k of the oracle's scores (near ties as in the plain top-k tests)
and, where it equals the oracle's set, the output must match the oracle's
attention over it.
"""

import numpy as np
import pytest
import torch

from oracle import attention_ref as ao
from oracle import selection_ref as sr
from oracle import socket_ref as so
from hash_scored_top_b200 import workloads as wl
from tests import parity as pa

pytestmark = pytest.mark.gpu

DEV = "cuda"
MASS_REL = 2e-6


@pytest.fixture(scope="module")
def api():
    from hash_scored_top_b200 import build
    build.build()
    from hash_scored_top_b200 import api as _api
    return _api


def _w(name):
    return {
        "tiny_f32": wl.TINY_F32,
        "llama1b_ragged": wl.shrink(wl.LLAMA_1B, B=1, Hkv=2, Hq=8, N=9001, k=9001 // 33),
        "qwen_l48_g8": wl.shrink(wl.QWEN3_30B, B=1, Hkv=2, Hq=16, N=6000, k=6000 // 50),
        "d64_g1": wl.shrink(wl.LLAMA_1B, B=2, Hkv=1, Hq=1, N=3000, k=100, L=20, P=6, tau=0.4),
        "g2_small_n": wl.shrink(wl.LLAMA_8B, B=1, Hkv=3, Hq=6, N=70, k=9, needles=0, L=5, P=3, tau=0.7),
        "llama8b_g4": wl.shrink(wl.LLAMA_8B, B=2, Hkv=2, Hq=8, N=12000, k=12000 // 33),
    }[name]


def _cache(w, inp):
    ids_nat, norms, _ = pa.oracle_socket_cache(inp, w)
    ids, nrm = pa.to_device_cache(ids_nat, norms, DEV)
    return ids, nrm, ids_nat, norms


# ---------------------------------------------------------------- per-head index sets

@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "qwen_l48_g8", "g2_small_n", "llama8b_g4"])
def test_decode_heads_matches_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms = _cache(w, inp)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hq, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode_heads(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O,
                            idx)
    api.check_status()
    R = inp["R"].double().cpu().numpy()
    tol = pa.out_tol(w)
    compared = units = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            o_ref, idx_ref, s_ref = sr.socket_decode_pair_per_head(Qg, K, V, R, ids_nat[b, h, : w.N],
                                                                   norms[b, h, : w.N], w.L, w.P, w.tau, w.k, w.scale)
            for g in range(w.G):
                units += 1
                got = idx[b, h * w.G + g].cpu().numpy()
                assert pa.check_selection(s_ref[g], got, w.k) == [], (b, h, g)
                if np.array_equal(got, idx_ref[g]):
                    compared += 1
                    err = pa.row_rel_err(O[b, h * w.G + g:h * w.G + g + 1].cpu().numpy(), o_ref[g:g + 1])
                    assert err < tol, (err, b, h, g)
    assert compared >= max(1, (3 * units) // 4)


def test_decode_heads_with_one_head_is_the_decode(api):
    # G = 1: the per-head units are the pairs; same kernels, same bits
    w = _w("d64_g1")
    inp = wl.make_inputs(w, DEV)
    ids, nrm, _, _ = _cache(w, inp)
    O1 = torch.empty(w.B, w.Hq, w.d, device=DEV)
    O2 = torch.empty_like(O1)
    i1 = torch.empty(w.B, w.Hq, w.k, dtype=torch.int32, device=DEV)
    i2 = torch.empty_like(i1)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O1, i1)
    api.socket_decode_heads(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O2,
                            i2)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2)
    assert torch.equal(O1, O2)


# ---------------------------------------------------------------- adaptive k

def _k_band(s, mass, k_min, k_max):
    s = np.asarray(s, dtype=np.float64)
    n = len(s)
    cum = np.cumsum(np.sort(s)[::-1])
    S = s.sum()

    def first(t):
        hit = np.nonzero(cum >= t)[0]
        return int(hit[0]) + 1 if hit.size else n

    clamp = lambda k: max(k_min, min(k, k_max, n))  # noqa: E731
    return clamp(first(mass * S * (1 - MASS_REL))), clamp(first(mass * S * (1 + MASS_REL)))


def _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, mass, k_min, k_max, per_head):
    U = w.Hq if per_head else w.Hkv
    gu = 1 if per_head else w.G
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, U, k_max, dtype=torch.int32, device=DEV)
    kc = torch.empty(w.B, U, dtype=torch.int32, device=DEV)
    api.socket_decode_adaptive(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, mass, k_min,
                               k_max, w.scale, O, idx, kc, per_head=per_head)
    api.check_status()
    R = inp["R"].double().cpu().numpy()
    tol = pa.out_tol(w)
    compared = units = 0
    ks = []
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            ref = sr.socket_decode_pair_adaptive(Qg, K, V, R, ids_nat[b, h, : w.N], norms[b, h, : w.N], w.L, w.P,
                                                 w.tau, mass, k_min, k_max, w.scale, per_head=per_head)
            for j, (o_ref, idx_ref, k_ref, s_ref) in enumerate(ref):
                units += 1
                u = h * w.G + j if per_head else h
                k = int(kc[b, u])
                lo, hi = _k_band(s_ref, mass, k_min, k_max)
                assert lo <= k <= hi, (b, h, j, k, lo, hi, k_ref)
                ks.append(k)
                row = idx[b, u].cpu().numpy()
                assert (row[k:] == -1).all()
                got = row[:k]
                assert pa.check_selection(s_ref, got, k) == [], (b, h, j)
                want = so.select_topk(s_ref, k)
                if np.array_equal(got, want):
                    compared += 1
                    q = Qg[j:j + 1] if per_head else Qg
                    o_want = ao.attend_subset(q, K, V, want, w.scale)
                    r0 = h * w.G + j if per_head else h * w.G
                    err = pa.row_rel_err(O[b, r0:r0 + gu].cpu().numpy(), o_want)
                    assert err < tol, (err, b, h, j)
    assert compared >= max(1, (3 * units) // 4)
    return O, idx, kc, ks


@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "qwen_l48_g8", "d64_g1", "g2_small_n", "llama8b_g4"])
@pytest.mark.parametrize("per_head", [False, True])
@pytest.mark.parametrize("mass", [0.3, 0.9])
def test_decode_adaptive_matches_oracle(api, name, per_head, mass):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms = _cache(w, inp)
    _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, mass, 1, w.N, per_head)


def test_decode_adaptive_clamps_and_is_deterministic(api):
    w = _w("llama8b_g4")
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms = _cache(w, inp)
    # a tiny target: every unit takes k_min keys (its top k_min)
    _, _, kc, ks = _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, 1e-6, 17, 900, False)
    assert ks == [17] * len(ks)
    # the whole mass, capped: every unit takes k_max keys
    _, _, kc, ks = _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, 1.0, 5, 333, True)
    assert ks == [333] * len(ks)
    # repeated calls give the same bits
    a = _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, 0.6, 1, w.N, True)
    b = _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, 0.6, 1, w.N, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_decode_adaptive_rejects_bad_arguments(api):
    w = _w("g2_small_n")
    inp = wl.make_inputs(w, DEV)
    ids, nrm, _, _ = _cache(w, inp)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, 9, dtype=torch.int32, device=DEV)
    kc = torch.empty(w.B, w.Hkv, dtype=torch.int32, device=DEV)
    for mass, k_min, k_max in [(0.0, 1, 9), (1.5, 1, 9), (0.5, 0, 9), (0.5, 10, 9)]:
        with pytest.raises(RuntimeError):
            api.socket_decode_adaptive(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, mass,
                                       k_min, k_max, w.scale, O, idx, kc)


def test_decode_heads_over_several_waves(api):
    """128 query-head units of 40K keys need 2-CTA clusters, 256 CTAs: more
    than one wave, so the decode builds the units' tables once in a table
    kernel and the selection copies them. Sampled units against the oracle."""
    w = wl.shrink(wl.LLAMA_8B, B=4, Hkv=8, Hq=32, N=40000, k=40000 // 33, needles=0)
    inp = wl.make_inputs(w, DEV)
    sample = [(0, 0), (1, 3), (2, 5), (3, 7)]
    ids_nat, norms, _ = pa.oracle_socket_cache(inp, w, sample)
    # every pair needs a cache; the sampled pairs carry the oracle's
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    nrm = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, nrm)
    ids_o, nrm_o = pa.to_device_cache(ids_nat, norms, DEV)
    for b, h in sample:
        ids[b, h] = ids_o[b, h]
        nrm[b, h] = nrm_o[b, h]
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hq, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode_heads(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O,
                            idx)
    api.check_status()
    R = inp["R"].double().cpu().numpy()
    compared = 0
    for b, h in sample:
        Qg, K, V = pa.pair_arrays(inp, w, b, h)
        o_ref, idx_ref, s_ref = sr.socket_decode_pair_per_head(Qg, K, V, R, ids_nat[b, h, : w.N], norms[b, h, : w.N],
                                                               w.L, w.P, w.tau, w.k, w.scale)
        for g in range(w.G):
            got = idx[b, h * w.G + g].cpu().numpy()
            assert pa.check_selection(s_ref[g], got, w.k) == [], (b, h, g)
            if np.array_equal(got, idx_ref[g]):
                compared += 1
                err = pa.row_rel_err(O[b, h * w.G + g:h * w.G + g + 1].cpu().numpy(), o_ref[g:g + 1])
                assert err < pa.out_tol(w), (err, b, h, g)
    assert compared >= 12


@pytest.mark.parametrize("name,per_head,mass,k_min,k_max", [
    ("llama8b_100k", False, 0.3, 1, None),       # 4-CTA clusters, k from the mass search
    ("llama8b_100k", True, 0.6, 1, None),
    ("llama8b_100k", False, 1e-6, 17, 900),      # clamped: the count search across 4 CTAs
    ("llama8b_100k", True, 1.0, 5, 333),
    ("ties_60k", False, 0.4, 1, None),           # many exactly equal scores across 2 CTAs
    ("ties_60k", True, 0.05, 1, None),
])
def test_decode_adaptive_multi_cta(api, name, per_head, mass, k_min, k_max):
    """Units of more keys than one CTA holds (the adaptive top-k then runs in
    clusters of 2 or 4 CTAs: cluster-wide mass sums and resolves, tie quotas and
    output offsets across CTAs); N is not a multiple of 4, so the last CTA's
    slice is ragged. In the tie-heavy shape (2 tables of 2 hyperplanes: 16
    bucket combinations times the f16 norms) about 89% of the keys share
    their score with another key (19.5K distinct scores over 60K keys)."""
    w = {"llama8b_100k": wl.shrink(wl.LLAMA_8B, B=1, Hkv=2, Hq=8, N=100003, k=100003 // 33),
         "ties_60k": wl.shrink(wl.LLAMA_8B, B=1, Hkv=2, Hq=4, N=60001, k=60001 // 33, needles=0, L=2, P=2,
                               tau=0.7)}[name]
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms = _cache(w, inp)
    _adaptive_and_compare(api, w, inp, ids, nrm, ids_nat, norms, mass, k_min, k_max if k_max else w.N, per_head)
