"""GPU parity of the hard-hash (HATA-style) variant against the oracle."""

import numpy as np
import pytest
import torch

from oracle import hata_ref as ho
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
        "hata_small": wl.shrink(wl.HATA_16, B=2, Hkv=2, Hq=8, N=20000, k=500),
        "hata_ragged_g8": wl.shrink(wl.HATA_16, B=1, Hkv=2, Hq=16, N=3333, k=77),
        "hata_f32_g1": wl.shrink(wl.HATA_16, B=1, Hkv=1, Hq=1, N=4096, k=128, kv_dtype="f32"),
    }[name]


@pytest.mark.parametrize("name", ["hata_small", "hata_ragged_g8", "hata_f32_g1"])
def test_codes_match_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    Ncap = inp["K"].shape[2]
    codes = api.empty_codes(w.B, w.Hkv, Ncap, DEV)
    api.hata_hash_keys(inp["K"], inp["R128"], codes)
    torch.cuda.synchronize()
    got = api.ids_to_natural(codes, 16).cpu().numpy()
    ref, proj = pa.oracle_codes(inp, w)
    R = inp["R128"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            K = inp["K"][b, h, : w.N].double().cpu().numpy()
            robust = pa.sign_band(K, R, proj[(b, h)]).reshape(w.N, 16, 8).all(axis=2)
            assert pa.check_ids(got[b, h, : w.N], ref[b, h, : w.N], robust) == 0


@pytest.mark.parametrize("name", ["hata_small", "hata_ragged_g8", "hata_f32_g1"])
def test_hata_decode_matches_oracle(api, name):
    w = _w(name)
    inp = wl.make_inputs(w, DEV)
    codes_nat, _ = pa.oracle_codes(inp, w)
    codes = api.natural_to_ids(torch.from_numpy(codes_nat)).to(DEV)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, idx)
    api.check_status()
    R = inp["R128"].double().cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            o_ref, idx_ref, _ = ho.hata_decode_pair(Qg, K, V, R, codes_nat[b, h, : w.N], w.k, w.scale)
            assert np.array_equal(idx[b, h].cpu().numpy(), idx_ref), (b, h)     # integer scores: exact
            assert pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref) < pa.out_tol(w)


def test_hata_self_query_key_selected(api):
    """A key equal to a query head matches all 128 bits for that head and is selected."""
    w = _w("hata_small")
    inp = wl.make_inputs(w, DEV)
    pos = 12345
    for b in range(w.B):
        for h in range(w.Hkv):
            inp["K"][b, h, pos] = inp["Q"][b, h * w.G]
    codes = api.empty_codes(w.B, w.Hkv, inp["K"].shape[2], DEV)
    api.hata_hash_keys(inp["K"], inp["R128"], codes)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, idx)
    api.check_status()
    for b in range(w.B):
        for h in range(w.Hkv):
            assert pos in idx[b, h].cpu().tolist()


def test_hata_decode_large_n_runs_the_unfused_chain(api):
    """700K keys of one pair do not fit one cluster's shared memory: the hard-hash
    decode then runs the unfused chain (byte-tables, scores through HBM, radix
    top-k, attention) and still matches the oracle exactly on the index set."""
    w = wl.shrink(wl.HATA_16, B=1, Hkv=1, Hq=4, N=700_000, k=2048)
    inp = wl.make_inputs(w, DEV)
    codes_nat, _ = pa.oracle_codes(inp, w)
    codes = api.natural_to_ids(torch.from_numpy(codes_nat)).to(DEV)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, idx)
    api.check_status()
    R = inp["R128"].double().cpu().numpy()
    Qg, K, V = pa.pair_arrays(inp, w, 0, 0)
    o_ref, idx_ref, _ = ho.hata_decode_pair(Qg, K, V, R, codes_nat[0, 0, : w.N], w.k, w.scale)
    assert np.array_equal(idx[0, 0].cpu().numpy(), idx_ref)
    assert pa.row_rel_err(O[0].cpu().numpy(), o_ref) < pa.out_tol(w)


def test_hata_decode_over_several_waves(api):
    """128 pairs of 40K keys need 2-CTA clusters, 256 CTAs: more than one wave,
    so the decode builds the byte-tables once in a table kernel and the
    selection copies them. Sampled pairs carry the oracle's codes and are
    compared exactly on the index set."""
    w = wl.shrink(wl.HATA_16, B=16, Hkv=8, Hq=32, N=40000, k=1024)
    inp = wl.make_inputs(w, DEV)
    sample = [(0, 0), (5, 3), (11, 6), (15, 7)]
    codes_nat, _ = pa.oracle_codes(inp, w, sample)
    Ncap = inp["K"].shape[2]
    codes = api.empty_codes(w.B, w.Hkv, Ncap, DEV)
    api.hata_hash_keys(inp["K"], inp["R128"], codes)
    codes_o = api.natural_to_ids(torch.from_numpy(codes_nat)).to(DEV)
    for b, h in sample:
        codes[b, h] = codes_o[b, h]
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, idx)
    api.check_status()
    R = inp["R128"].double().cpu().numpy()
    for b, h in sample:
        Qg, K, V = pa.pair_arrays(inp, w, b, h)
        o_ref, idx_ref, _ = ho.hata_decode_pair(Qg, K, V, R, codes_nat[b, h, : w.N], w.k, w.scale)
        assert np.array_equal(idx[b, h].cpu().numpy(), idx_ref), (b, h)
        assert pa.row_rel_err(O[b, h * w.G:(h + 1) * w.G].cpu().numpy(), o_ref) < pa.out_tol(w)
