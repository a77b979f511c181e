"""GPU parity of the SOCKET path against the oracle, through the C ABI.

Sizes here finish in seconds on the oracle and still span several tiles,
several CTAs of a cluster and ragged tails. Full-size workloads are covered
by test_gpu_fullsize.py on sampled pairs.
"""

import numpy as np
import pytest
import torch

from oracle import attention_ref as ao
from oracle import socket_ref as so
from hash_scored_top_b200 import workloads as wl
from tests import parity as pa

pytestmark = pytest.mark.gpu

DEV = "cuda"


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
        "llama8b_needles": wl.shrink(wl.LLAMA_8B, B=2, Hkv=2, Hq=8, N=12000, k=12000 // 33),
        "qwen_l48_g8": wl.shrink(wl.QWEN3_30B, B=1, Hkv=2, Hq=16, N=10000, k=10000 // 50),
        "d64_g1": wl.shrink(wl.LLAMA_1B, B=2, Hkv=1, Hq=1, N=3000, k=100, L=20, P=6, tau=0.4),
        "g2_small_n": wl.shrink(wl.LLAMA_8B, B=1, Hkv=3, Hq=6, N=70, k=9, needles=0, L=5, P=3, tau=0.7),
        # 160 pairs: more than one wave of score CTAs, one CTA per pair
        "many_pairs": wl.shrink(wl.LLAMA_8B, B=10, Hkv=16, Hq=16, N=777, k=25, needles=0, L=8, P=4, tau=0.5),
    }[name]


def _cache(api, w, inp, pairs=None):
    ids_nat, norms, proj = pa.oracle_socket_cache(inp, w, pairs)
    ids, nrm = pa.to_device_cache(ids_nat, norms, DEV)
    return ids, nrm, ids_nat, norms, proj


# ---------------------------------------------------------------- step 1: hashing

@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "qwen_l48_g8", "d64_g1"])
def test_hash_keys_match_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms)
    torch.cuda.synchronize()
    gpu_nat = api.ids_to_natural(ids, w.L).cpu().numpy()
    ref_nat, ref_norms, proj = pa.oracle_socket_cache(inp, w)
    R = inp["R"].double().cpu().numpy()
    total_robust = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            K = inp["K"][b, h, : w.N].double().cpu().numpy()
            robust = pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, w.L, w.P).all(axis=2)
            total_robust += int(robust.sum())
            assert pa.check_ids(gpu_nat[b, h, : w.N], ref_nat[b, h, : w.N], robust) == 0
            assert np.array_equal(norms[b, h, : w.N].cpu().numpy(), ref_norms[b, h, : w.N])
    assert total_robust >= 0.99 * w.B * w.Hkv * w.N * w.L


# bf16 keys with P = 8 go through the tensor-core prefill kernel: L = 10 pads
# the last 4-table block and the 16-byte ID row; L = 64 needs two 256-column
# MMA chunks and leaves room for one key stage; L = 5 at d = 64 pads rows of
# R past 8L; Ncap not a multiple of 128 leaves a partial last tile.
@pytest.mark.parametrize("L,d,N,B,Hkv", [(10, 128, 700, 1, 2), (64, 128, 300, 1, 1), (5, 64, 333, 2, 1)])
def test_hash_keys_tensor_core_shapes(api, L, d, N, B, Hkv):
    w = wl.shrink(wl.LLAMA_1B, B=B, Hkv=Hkv, Hq=Hkv, d=d, N=N, L=L, P=8, k=N // 10, outlier_channels=0)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms, 0, w.N)
    # the same keys in two ranges that split a 128-key tile
    ids2 = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms2 = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    cut = 77
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids2, norms2, 0, cut)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids2, norms2, cut, w.N - cut)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(norms, norms2)
    gpu_nat = api.ids_to_natural(ids, w.L).cpu().numpy()
    ref_nat, ref_norms, proj = pa.oracle_socket_cache(inp, w)
    R = inp["R"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            K = inp["K"][b, h, : w.N].double().cpu().numpy()
            robust = pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, w.L, w.P).all(axis=2)
            assert pa.check_ids(gpu_nat[b, h, : w.N], ref_nat[b, h, : w.N], robust) == 0
            assert np.array_equal(norms[b, h, : w.N].cpu().numpy(), ref_norms[b, h, : w.N])
    assert np.all(gpu_nat[:, :, w.N:] == 0)


def test_hash_keys_append_touches_only_the_range(api):
    w = _w("llama1b_ragged")
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms, 0, w.N - 1)
    before_ids, before_norms = ids.clone(), norms.clone()
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms, w.N - 1, 1)   # append one token
    full_ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    full_norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, full_ids, full_norms, 0, w.N)
    torch.cuda.synchronize()
    assert torch.equal(norms, full_norms)
    nat_b, nat_a = api.ids_to_natural(before_ids, w.L), api.ids_to_natural(ids, w.L)
    nat_full = api.ids_to_natural(full_ids, w.L)
    assert torch.equal(nat_b[:, :, : w.N - 1], nat_a[:, :, : w.N - 1])
    assert torch.equal(nat_a[:, :, : w.N - 1], nat_full[:, :, : w.N - 1])
    assert torch.equal(nat_a[:, :, w.N:], torch.zeros_like(nat_a[:, :, w.N:]))
    # the appended key: the few-key kernel and the bulk kernel add the f32
    # projection up in different orders, so they may disagree only on a table
    # with a projection inside the f32 rounding band around zero
    R = inp["R"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            k = inp["K"][b, h, w.N - 1 : w.N].double().cpu().numpy()
            robust = pa.sign_band(k, R, k @ R.T).reshape(1, w.L, w.P).all(axis=2)
            got = nat_a[b, h, w.N - 1 : w.N].cpu().numpy()
            ref = nat_full[b, h, w.N - 1 : w.N].cpu().numpy()
            assert pa.check_ids(got, ref, robust) == 0


# ---------------------------------------------------------------- steps 2-3: scores

@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "qwen_l48_g8", "d64_g1", "g2_small_n", "many_pairs"])
def test_scores_match_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids, nrm, ids_nat, norms, _ = _cache(api, w, inp)
    scores = torch.full((w.B, w.Hkv, Ncap), -7.0, device=DEV)
    api.socket_score(inp["Q"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, scores)
    torch.cuda.synchronize()
    R = inp["R"].double().cpu().numpy()
    worst = 0.0
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg, _, _ = pa.pair_arrays(inp, w, b, h)
            T = so.group_bucket_table(Qg, R, w.L, w.P, w.tau)
            ref = so.soft_collision_scores(T, ids_nat[b, h, : w.N], norms[b, h, : w.N])
            got = scores[b, h, : w.N].double().cpu().numpy()
            worst = max(worst, float(np.max(np.abs(got - ref) / np.maximum(ref, 1e-30))))
            assert np.all(scores[b, h, w.N:].cpu().numpy() == -7.0)      # tail untouched
    assert worst <= pa.SCORE_REL_TOL, worst


# ---------------------------------------------------------------- step 4: selection

@pytest.mark.parametrize("N,ks,kind", [
    (70, [1, 9, 69, 70], "ties"),
    (5000, [1, 7, 165, 4999], "ties"),
    (33001, [1, 1000, 33001], "random"),
    (102400, [3103], "random"),
    (4096, [1, 128, 4096], "equal"),
])
def test_topk_matches_oracle_exactly(api, N, ks, kind):
    g = torch.Generator(device="cpu").manual_seed(N)
    B, Hkv = 2, 2
    Ncap = (N + 31) // 32 * 32
    if kind == "ties":
        s = torch.randint(0, 20, (B, Hkv, Ncap), generator=g).float() * 0.25
    elif kind == "equal":
        s = torch.full((B, Hkv, Ncap), 1.5)
    else:
        s = torch.rand(B, Hkv, Ncap, generator=g) * 10
    scores = s.to(DEV)
    for k in ks:
        idx = torch.empty(B, Hkv, k, dtype=torch.int32, device=DEV)
        api.socket_topk(scores, N, k, idx)
        torch.cuda.synchronize()
        for b in range(B):
            for h in range(Hkv):
                want = so.select_topk(s[b, h, :N].double().numpy(), k)
                assert np.array_equal(idx[b, h].cpu().numpy(), want), (N, k, kind, b, h)


# ---------------------------------------------------------------- step 4: attention over the subset

@pytest.mark.parametrize("dtype,d,G,k", [
    ("bf16", 128, 4, 1), ("bf16", 128, 4, 17), ("bf16", 128, 4, 1000), ("bf16", 128, 8, 300),
    ("bf16", 64, 4, 129), ("bf16", 128, 1, 33), ("bf16", 64, 2, 250), ("f32", 128, 1, 128), ("f32", 64, 3, 77),
])
def test_sparse_attend_matches_oracle(api, dtype, d, G, k):
    torch.manual_seed(k * 7 + d + G)
    B, Hkv, N = 2, 2, 4096
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Q = torch.randn(B, Hkv * G, d).to(dt)
    K = torch.randn(B, Hkv, N, d).to(dt)
    V = torch.randn(B, Hkv, N, d).to(dt)
    idx = torch.stack([torch.stack([torch.randperm(N)[:k].sort().values for _ in range(Hkv)]) for _ in range(B)])
    O = torch.empty(B, Hkv * G, d, device=DEV)
    api.socket_sparse_attend(Q.to(DEV), K.to(DEV), V.to(DEV), idx.int().to(DEV), d ** -0.5, O)
    torch.cuda.synchronize()
    tol = pa.BF16_TOL if dtype == "bf16" else pa.F32_TOL
    for b in range(B):
        for h in range(Hkv):
            ref = ao.attend_subset(Q[b, h * G:(h + 1) * G].double().numpy(), K[b, h].double().numpy(),
                                   V[b, h].double().numpy(), idx[b, h].numpy(), d ** -0.5)
            err = pa.row_rel_err(O[b, h * G:(h + 1) * G].cpu().numpy(), ref)
            assert err < tol, (err, b, h)


# ---------------------------------------------------------------- fused decode

def _decode_and_compare(api, w, inp, ids, nrm, ids_nat, norms, tol, use_chain=False):
    Ncap = inp["K"].shape[2]
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    if use_chain:
        scores = torch.empty(w.B, w.Hkv, Ncap, device=DEV)
        api.socket_score(inp["Q"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, scores)
        api.socket_topk(scores, w.N, w.k, idx)
        api.socket_sparse_attend(inp["Q"], inp["K"], inp["V"], idx, w.scale, O)
    else:
        api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
    api.check_status()
    R = inp["R"].double().cpu().numpy()
    compared = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            o_ref, idx_ref, s_ref = so.socket_decode_pair(Qg, K, V, R, ids_nat[b, h, : w.N], norms[b, h, : w.N],
                                                          w.L, w.P, w.tau, w.k, w.scale)
            got = idx[b, h].cpu().numpy()
            assert pa.check_selection(s_ref, got, w.k) == [], (b, h)
            if np.array_equal(got, idx_ref):
                compared += 1
                err = pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref)
                assert err < tol, (err, b, h)
    assert compared >= max(1, (w.B * w.Hkv * 3) // 4)
    return O, idx


@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "llama8b_needles", "qwen_l48_g8", "d64_g1",
                                  "g2_small_n"])
def test_fused_decode_matches_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms, _ = _cache(api, w, inp)
    O, idx = _decode_and_compare(api, w, inp, ids, nrm, ids_nat, norms, pa.out_tol(w))
    if w.needles:
        for b in range(w.B):
            for h in range(w.Hkv):
                assert set(inp["needle_pos"][b, h].tolist()) <= set(idx[b, h].cpu().tolist())
    # the unfused chain selects exactly the same keys
    O2, idx2 = _decode_and_compare(api, w, inp, ids, nrm, ids_nat, norms, pa.out_tol(w), use_chain=True)
    assert torch.equal(idx, idx2)


@pytest.mark.parametrize("name", ["tiny_f32", "llama8b_needles", "qwen_l48_g8", "g2_small_n"])
def test_select_only_matches_decode_and_oracle(api, name):
    """socket_select returns the decode step's index list: a valid top-k of the
    oracle's scores, identical to what socket_decode selects."""
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms, _ = _cache(api, w, inp)
    sel = torch.full((w.B, w.Hkv, w.k), -1, dtype=torch.int32, device=DEV)
    api.socket_select(inp["Q"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, sel)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
    api.check_status()
    assert torch.equal(sel, idx)
    R = inp["R"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg = inp["Q"][b, h * w.G:(h + 1) * w.G].double().cpu().numpy()
            s_ref = so.soft_collision_scores(so.group_bucket_table(Qg, R, w.L, w.P, w.tau), ids_nat[b, h, : w.N],
                                             norms[b, h, : w.N])
            assert pa.check_selection(s_ref, sel[b, h].cpu().numpy(), w.k) == [], (b, h)


@pytest.mark.parametrize("name", ["llama8b_needles", "qwen_l48_g8", "tiny_f32"])
def test_decode_append_equals_hash_then_decode(api, name):
    """socket_decode_append = socket_hash_keys of key N - 1, then socket_decode."""
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    nrm = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, nrm, 0, w.N - 1)   # the cache before the step
    ids2, nrm2 = ids.clone(), nrm.clone()
    O1 = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx1 = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode_append(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale,
                             O1, idx1)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids2, nrm2, w.N - 1, 1)
    O2 = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx2 = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids2, nrm2, w.N, w.L, w.P, w.tau, w.k, w.scale, O2, idx2)
    api.check_status()
    assert torch.equal(ids, ids2) and torch.equal(nrm, nrm2)
    assert torch.equal(idx1, idx2) and torch.equal(O1, O2)


@pytest.mark.parametrize("name,pinned", [("llama8b_needles", True), ("tiny_f32", True), ("llama8b_needles", False)])
def test_decode_step_from_host_buffers(api, name, pinned):
    """socket_decode_step_host copies the query and the new token's K/V rows in
    from host memory (the rows into position N - 1 of every pair), runs
    socket_decode_append and copies O out: the cache, the hashed rows and O
    equal those of the device-resident step bit for bit. Pinned buffers are
    read and written by a copy kernel; pageable ones by DMA copies."""
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    nrm = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, nrm, 0, w.N - 1)   # the cache before the step
    ids2, nrm2 = ids.clone(), nrm.clone()
    # reference: the rows already in the device cache, the device-resident step
    O1 = torch.empty(w.B, w.Hq, w.d, device=DEV)
    api.socket_decode_append(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O1)
    # the host-buffer step: the cache's row N - 1 and the query start as garbage
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t)
    q_host = pin(inp["Q"].cpu())
    k_host = pin(inp["K"][:, :, w.N - 1].contiguous().cpu())
    v_host = pin(inp["V"][:, :, w.N - 1].contiguous().cpu())
    K2, V2 = inp["K"].clone(), inp["V"].clone()
    K2[:, :, w.N - 1] = 7.0
    V2[:, :, w.N - 1] = -3.0
    Q2 = torch.full_like(inp["Q"], 5.0)
    O2 = torch.empty_like(O1)
    o_host = pin(torch.full((w.B, w.Hq, w.d), float("nan")))
    api.socket_decode_step_host(q_host, k_host, v_host, Q2, K2, V2, inp["R"], ids2, nrm2, w.N, w.L, w.P, w.tau, w.k,
                                w.scale, O2, o_host)
    torch.cuda.synchronize()
    api.check_status()
    assert torch.equal(K2, inp["K"]) and torch.equal(V2, inp["V"]) and torch.equal(Q2, inp["Q"])
    assert torch.equal(ids, ids2) and torch.equal(nrm, nrm2)
    assert torch.equal(O2, O1) and torch.equal(o_host, O1.cpu())


@pytest.mark.parametrize("case", ["all_equal", "all_zero", "above_range"])
def test_fused_selection_fallback_cases(api, case):
    """Score distributions the binned selection hands to the exact radix path:
    every key in the same buckets (the boundary bin holds all keys), every
    score 0 (below the bins' range), and a few keys above the range. The
    selection must still be a valid top-k of the oracle's scores."""
    w = _w("llama8b_needles")
    inp = wl.make_inputs(w, DEV)
    ids_nat, norms, _ = pa.oracle_socket_cache(inp, w)
    if case == "all_equal":
        ids_nat[...] = ids_nat[:, :, :1, :]          # every key in the same buckets
        norms[...] = np.float16(1.5)
    elif case == "all_zero":
        norms[...] = np.float16(0.0)
    else:                                            # f16 max norm: scores far above 2^16
        norms[:, :, 100:140] = np.float16(60000.0)
    ids, nrm = pa.to_device_cache(ids_nat, norms, DEV)
    sel = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_select(inp["Q"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, sel)
    api.check_status()
    R = inp["R"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg = inp["Q"][b, h * w.G:(h + 1) * w.G].double().cpu().numpy()
            s_ref = so.soft_collision_scores(so.group_bucket_table(Qg, R, w.L, w.P, w.tau), ids_nat[b, h, : w.N],
                                             norms[b, h, : w.N])
            got = sel[b, h].cpu().numpy()
            # keys with equal bucket IDs sum their table values in a key-dependent
            # (rotated) order, so "all equal" scores agree only within the near-tie
            # window; zero scores are exact ties and go to the lowest indices
            assert pa.check_selection(s_ref, got, w.k) == [], (b, h)
            if case == "all_zero":
                assert np.array_equal(got, np.arange(w.k)), (b, h)


def test_fused_decode_is_deterministic(api):
    w = _w("llama8b_needles")
    inp = wl.make_inputs(w, DEV)
    ids, nrm, *_ = _cache(api, w, inp)
    outs = []
    for _ in range(3):
        O = torch.empty(w.B, w.Hq, w.d, device=DEV)
        idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
        api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
        outs.append((O, idx))
    torch.cuda.synchronize()
    for O, idx in outs[1:]:
        assert torch.equal(O, outs[0][0]) and torch.equal(idx, outs[0][1])


@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged"])
def test_decode_with_k_equal_n_is_dense_attention(api, name):
    w = _w(name)
    w = wl.shrink(w, k=w.N)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, *_ = _cache(api, w, inp)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
    api.check_status()
    assert torch.equal(idx.cpu(), torch.arange(w.N, dtype=torch.int32).expand(w.B, w.Hkv, w.N))
    ref = ao.dense_decode(inp["Q"].double().cpu().numpy(), inp["K"].double().cpu().numpy(),
                          inp["V"].double().cpu().numpy(), w.scale, N=w.N)
    assert pa.row_rel_err(O.cpu().numpy(), ref) < pa.out_tol(w)


def test_decode_k_one_picks_the_top_key(api):
    w = wl.shrink(_w("llama8b_needles"), k=1)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms, _ = _cache(api, w, inp)
    O, idx = _decode_and_compare(api, w, inp, ids, nrm, ids_nat, norms, pa.BF16_TOL)
    # a single selected key: the output is that key's value row
    for b in range(w.B):
        for h in range(w.Hkv):
            v = inp["V"][b, h, idx[b, h, 0].item()].float()
            assert torch.allclose(O[b, h * w.G:(h + 1) * w.G], v.expand(w.G, -1), rtol=0, atol=1e-6)


# ---------------------------------------------------------------- dense decode

@pytest.mark.parametrize("name", ["tiny_f32", "llama1b_ragged", "qwen_l48_g8"])
def test_dense_decode_matches_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    api.dense_decode(inp["Q"], inp["K"], inp["V"], w.N, w.scale, O)
    torch.cuda.synchronize()
    ref = ao.dense_decode(inp["Q"].double().cpu().numpy(), inp["K"].double().cpu().numpy(),
                          inp["V"].double().cpu().numpy(), w.scale, N=w.N)
    assert pa.row_rel_err(O.cpu().numpy(), ref) < pa.out_tol(w)


# ---------------------------------------------------------------- append + decode against the oracle

@pytest.mark.parametrize("name", ["llama8b_needles", "tiny_f32", "qwen_l48_g8"])
def test_decode_append_matches_oracle(api, name):
    """socket_decode_append against the oracle alone. Keys 0 .. N-2 of the
    cache are the oracle's own hashing; the call hashes key N-1 on the GPU.
    Its bucket IDs must equal the oracle's outside the f32 sign band and its
    norm bit-exactly; where the whole row equals the oracle's, the selection
    must be a valid top-k of the oracle's scores over its own cache, and the
    output within the attention tolerance where the sets agree."""
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    ids_nat, norms, proj = pa.oracle_socket_cache(inp, w)
    before_nat = ids_nat.copy()
    before_norms = norms.copy()
    before_nat[:, :, w.N - 1] = 0
    before_norms[:, :, w.N - 1] = 0
    ids, nrm = pa.to_device_cache(before_nat, before_norms, DEV)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode_append(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale,
                             O, idx)
    api.check_status()
    got_nat = api.ids_to_natural(ids, w.L).cpu().numpy()
    got_norms = nrm.cpu().numpy()
    R = inp["R"].double().cpu().numpy()
    compared = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            # keys before N-1 are untouched
            assert np.array_equal(got_nat[b, h, : w.N - 1], before_nat[b, h, : w.N - 1])
            assert np.array_equal(got_norms[b, h, : w.N - 1], before_norms[b, h, : w.N - 1])
            k_row = inp["K"][b, h, w.N - 1: w.N].double().cpu().numpy()
            robust = pa.sign_band(k_row, R, proj[(b, h)][w.N - 1: w.N]).reshape(1, w.L, w.P).all(axis=2)
            assert pa.check_ids(got_nat[b, h, w.N - 1: w.N], ids_nat[b, h, w.N - 1: w.N], robust) == 0, (b, h)
            assert got_norms[b, h, w.N - 1] == norms[b, h, w.N - 1], (b, h)
            if not np.array_equal(got_nat[b, h, w.N - 1], ids_nat[b, h, w.N - 1]):
                continue                       # a table inside the sign band: scores differ legitimately
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            o_ref, idx_ref, s_ref = so.socket_decode_pair(Qg, K, V, R, ids_nat[b, h, : w.N], norms[b, h, : w.N],
                                                          w.L, w.P, w.tau, w.k, w.scale)
            got = idx[b, h].cpu().numpy()
            assert pa.check_selection(s_ref, got, w.k) == [], (b, h)
            if np.array_equal(got, idx_ref):
                compared += 1
                err = pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref)
                assert err < pa.out_tol(w), (err, b, h)
    assert compared >= max(1, (w.B * w.Hkv * 3) // 4)


def test_hash_keys_sign_band_statistics(api, capsys):
    """Reports, for the 8B-like shape, how many (key, table) bucket IDs fall
    inside the literal 1e-6 band of the spec and inside the wider f32 band
    used by the parity tests, and how many of each actually differ from the
    oracle. Asserts that nothing outside the wider band differs."""
    w = _w("llama8b_needles")
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms)
    torch.cuda.synchronize()
    gpu_nat = api.ids_to_natural(ids, w.L).cpu().numpy()
    ref_nat, _, proj = pa.oracle_socket_cache(inp, w)
    R = inp["R"].double().cpu().numpy()
    tot = lit_band = f32_band = diff_lit = diff_f32 = diff_out = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            K = inp["K"][b, h, : w.N].double().cpu().numpy()
            pr = proj[(b, h)].reshape(w.N, w.L, w.P)
            in_lit = (np.abs(pr) < 1e-6).any(axis=2)
            in_f32 = ~pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, w.L, w.P).all(axis=2)
            diff = gpu_nat[b, h, : w.N] != ref_nat[b, h, : w.N]
            tot += diff.size
            lit_band += int(in_lit.sum())
            f32_band += int(in_f32.sum())
            diff_lit += int((diff & in_lit).sum())
            diff_f32 += int((diff & in_f32).sum())
            diff_out += int((diff & ~in_f32).sum())
    with capsys.disabled():
        print(f"\n[sign band] {tot} IDs; in the 1e-6 band {lit_band}, in the f32 band {f32_band} "
              f"({f32_band / tot:.2e}); differing: {diff_lit} in the 1e-6 band, {diff_f32} in the f32 band, "
              f"{diff_out} outside it")
    assert diff_out == 0


def test_hash_tc_wait_timeout_drains_and_recovers(api):
    """The tensor-core hashing kernel's failure path: with its main-loop wait
    limit lowered to one clock (test hook), its waits give up while its TMA
    copies and MMAs are in flight. It must stop, drain what it issued, free its
    tensor memory and report SK_ERR_TIMEOUT; with the limit restored the next
    call on the same context is bit-identical to a run before the failure."""
    from hash_scored_top_b200 import _lib
    w = wl.shrink(wl.LLAMA_8B, B=1, Hkv=2, Hq=8, N=8192, k=256)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids0, nrm0 = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV), api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids0, nrm0, 0, w.N)
    api.check_status()
    ids1, nrm1 = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV), api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    try:
        assert _lib.lib.sk_test_set_wait_limit(1) == 0
        api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids1, nrm1, 0, w.N)
        with pytest.raises(RuntimeError, match="bounded wait"):
            api.check_status()
    finally:
        assert _lib.lib.sk_test_set_wait_limit(0) == 0
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids1, nrm1, 0, w.N)
    api.check_status()
    assert torch.equal(ids0, ids1) and torch.equal(nrm0, nrm1)


@pytest.mark.parametrize("tau", [1e-3, 1e4])
def test_decode_at_the_temperature_limits(api, tau):
    """Degenerate temperatures: tau -> 0 makes the soft assignment one-hot (the
    score counts hard collisions, many keys tie), tau -> infinity makes every
    table uniform (the score is the norm times a constant, ties wherever f16
    norms are equal). The selection must stay a valid top-k with ties to the
    lower index, and match the oracle's output where the sets agree."""
    w = wl.shrink(wl.LLAMA_8B, B=1, Hkv=2, Hq=8, N=5000, k=5000 // 33, tau=tau)
    inp = wl.make_inputs(w, DEV)
    ids, nrm, ids_nat, norms, _ = _cache(api, w, inp)
    _decode_and_compare(api, w, inp, ids, nrm, ids_nat, norms, pa.out_tol(w))


def test_hash_keys_empty_range_is_a_no_op(api):
    w = _w("g2_small_n")
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = torch.full((w.B, w.Hkv, Ncap, api.ids_bytes_per_key(w.L)), 7, dtype=torch.uint8, device=DEV)
    nrm = torch.full((w.B, w.Hkv, Ncap), 3.0, dtype=torch.float16, device=DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, nrm, 5, 0)
    api.check_status()
    assert (ids == 7).all() and (nrm == 3.0).all()
