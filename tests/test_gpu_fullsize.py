"""Full-size workloads, in the launch configuration the benchmark times,
checked on sampled (batch, KV-head) pairs that the oracle computes one by one.

The GPU hashes the whole cache; for the sampled pairs the oracle hashes the
keys itself (checking the GPU IDs and norms) and its cache replaces the GPU's
for those pairs, so the decode parity below uses no GPU-produced oracle input.
"""

import numpy as np
import pytest
import torch

from oracle import hata_ref as ho
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


def _sample_pairs(w, n):
    g = np.random.default_rng(w.seed + 7)
    allp = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    picks = g.choice(len(allp), size=min(n, len(allp)), replace=False)
    return sorted({allp[i] for i in picks} | {allp[0], allp[-1]})


@pytest.mark.parametrize("wname,nsample", [("llama3.2-1b_n32k", 8), ("llama3.1-8b_n100k", 3), ("qwen3-30b_n140k", 3)])
def test_socket_fullsize_sampled(api, wname, nsample):
    w = wl.WORKLOADS[wname]
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, DEV)
    norms = api.empty_norms(w.B, w.Hkv, Ncap, DEV)
    api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms)
    torch.cuda.synchronize()
    pairs = _sample_pairs(w, nsample)
    ref_nat, ref_norms, proj = pa.oracle_socket_cache(inp, w, pairs)
    R = inp["R"].double().cpu().numpy()
    nat = api.ids_to_natural(ids, w.L)
    for b, h in pairs:
        K = inp["K"][b, h, : w.N].double().cpu().numpy()
        robust = pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, w.L, w.P).all(axis=2)
        assert pa.check_ids(nat[b, h, : w.N].cpu().numpy(), ref_nat[b, h, : w.N], robust) == 0
        assert np.array_equal(norms[b, h, : w.N].cpu().numpy(), ref_norms[b, h, : w.N])
        nat[b, h] = torch.from_numpy(ref_nat[b, h]).to(DEV)
        norms[b, h] = torch.from_numpy(ref_norms[b, h]).to(DEV)
    ids = api.natural_to_ids(nat)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, norms, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
    api.check_status()
    compared = 0
    for b, h in pairs:
        Qg, K, V = pa.pair_arrays(inp, w, b, h)
        o_ref, idx_ref, s_ref = so.socket_decode_pair(Qg, K, V, R, ref_nat[b, h, : w.N], ref_norms[b, h, : w.N],
                                                      w.L, w.P, w.tau, w.k, w.scale)
        got = idx[b, h].cpu().numpy()
        assert pa.check_selection(s_ref, got, w.k) == [], (b, h)
        if w.needles:
            assert set(inp["needle_pos"][b, h].tolist()) <= set(got.tolist())
        if np.array_equal(got, idx_ref):
            compared += 1
            assert pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref) < pa.BF16_TOL
    assert compared >= len(pairs) - 1
    # every pair: ascending, in range, no repeats
    all_idx = idx.cpu().numpy()
    assert np.all(np.diff(all_idx, axis=-1) > 0) and all_idx.min() >= 0 and all_idx.max() < w.N


def test_hata_fullsize_sampled(api):
    w = wl.HATA_16
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    codes = api.empty_codes(w.B, w.Hkv, Ncap, DEV)
    api.hata_hash_keys(inp["K"], inp["R128"], codes)
    torch.cuda.synchronize()
    pairs = _sample_pairs(w, 3)
    ref, proj = pa.oracle_codes(inp, w, pairs)
    R = inp["R128"].double().cpu().numpy()
    nat = api.ids_to_natural(codes, 16)
    for b, h in pairs:
        K = inp["K"][b, h, : w.N].double().cpu().numpy()
        robust = pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, 16, 8).all(axis=2)
        assert pa.check_ids(nat[b, h, : w.N].cpu().numpy(), ref[b, h, : w.N], robust) == 0
        nat[b, h] = torch.from_numpy(ref[b, h]).to(DEV)
    codes = api.natural_to_ids(nat)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, idx)
    api.check_status()
    for b, h in pairs:
        Qg, K, V = pa.pair_arrays(inp, w, b, h)
        o_ref, idx_ref, _ = ho.hata_decode_pair(Qg, K, V, R, ref[b, h, : w.N], w.k, w.scale)
        assert np.array_equal(idx[b, h].cpu().numpy(), idx_ref)
        assert pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref) < pa.BF16_TOL
