"""Helpers shared by the GPU parity tests: oracle caches and comparisons.

Tolerances (derived from the arithmetic):

* bucket IDs and hard-hash codes: bit-exact, except tables / code bytes with a
  projection |k . r| below max(1e-6, d * 2^-24 * sum_c |k_c r_c|) -- the f32
  accumulation error bound of a length-d dot product of exact bf16 products;
* value norms: bit-exact (both sides round the float64 norm once to f16);
* soft scores: relative error <= 6e-7 (f32 table entries, a depth-6 summation
  tree and one product: 9 roundings of 2^-24);
* top-k index set: exact, except keys within 1e-6 relative of the oracle's
  k-th score (near ties); exact for the integer hard-hash scores;
* attention output: per query row max_c |o - o_ref| / max_c |o_ref| below
  2e-3 for bf16 K/V and 1e-5 for f32 K/V.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import hata_ref as ho
from oracle import socket_ref as so

BF16_TOL = 2e-3
F32_TOL = 1e-5
SCORE_REL_TOL = 6e-7
TIE_REL = 1e-6


def out_tol(w) -> float:
    return F32_TOL if w.kv_dtype == "f32" else BF16_TOL


def pair_arrays(inp, w, b, h):
    G = w.G
    K = inp["K"][b, h, : w.N].double().cpu().numpy()
    V = inp["V"][b, h, : w.N].double().cpu().numpy()
    Qg = inp["Q"][b, h * G:(h + 1) * G].double().cpu().numpy()
    return Qg, K, V


def oracle_socket_cache(inp, w, pairs=None):
    """Oracle bucket IDs [B, Hkv, Ncap, L] uint8 (natural layout) and f16 norms for the pairs."""
    B, Hkv, Ncap = w.B, w.Hkv, inp["K"].shape[2]
    ids = np.zeros((B, Hkv, Ncap, w.L), dtype=np.uint8)
    norms = np.zeros((B, Hkv, Ncap), dtype=np.float16)
    proj = {}
    R = inp["R"].double().cpu().numpy()
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        K = inp["K"][b, h, : w.N].double().cpu().numpy()
        V = inp["V"][b, h, : w.N].double().cpu().numpy()
        i, pr = so.hash_key_ids(K, R, w.L, w.P)
        ids[b, h, : w.N] = i.astype(np.uint8)
        norms[b, h, : w.N] = so.value_norms_f16(V)
        proj[(b, h)] = pr
    return ids, norms, proj


def oracle_codes(inp, w, pairs=None):
    B, Hkv, Ncap = w.B, w.Hkv, inp["K"].shape[2]
    codes = np.zeros((B, Hkv, Ncap, 16), dtype=np.uint8)
    proj = {}
    R = inp["R128"].double().cpu().numpy()
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in todo:
        K = inp["K"][b, h, : w.N].double().cpu().numpy()
        c, pr = ho.binary_codes(K, R)
        codes[b, h, : w.N] = c
        proj[(b, h)] = pr
    return codes, proj


def sign_band(K, R, proj):
    """Per (key, projection): True where the sign is decided robustly in f32."""
    absdot = np.abs(K) @ np.abs(R).T
    d = K.shape[1]
    band = np.maximum(1e-6, d * 2.0 ** -24 * absdot)
    return np.abs(proj) > band


def check_ids(gpu_nat, ref_nat, robust_tables):
    """gpu_nat, ref_nat: [n, L] ids; robust_tables: [n, L] bool. Returns mismatches on robust entries."""
    bad = (gpu_nat != ref_nat) & robust_tables
    return int(bad.sum())


def check_selection(scores_ref, idx_gpu, k, rel=TIE_REL):
    """The GPU index set against the oracle's scores with the near-tie band.

    Returns a list of problems (empty when the set is valid)."""
    problems = []
    idx_gpu = np.asarray(idx_gpu, dtype=np.int64)
    if len(idx_gpu) != k:
        problems.append(f"size {len(idx_gpu)} != k {k}")
    if np.any(np.diff(idx_gpu) <= 0):
        problems.append("not strictly ascending")
    if len(idx_gpu) and (idx_gpu.min() < 0 or idx_gpu.max() >= len(scores_ref)):
        problems.append("index out of range")
        return problems
    t = np.sort(scores_ref)[::-1][k - 1]
    chosen = np.zeros(len(scores_ref), dtype=bool)
    chosen[idx_gpu] = True
    must = scores_ref > t * (1 + rel)
    must_not = scores_ref < t * (1 - rel)
    if np.any(must & ~chosen):
        problems.append(f"{int((must & ~chosen).sum())} keys above the band not chosen")
    if np.any(must_not & chosen):
        problems.append(f"{int((must_not & chosen).sum())} keys below the band chosen")
    return problems


def row_rel_err(o_gpu, o_ref):
    """max over rows of max_c |o - o_ref| / max_c |o_ref|."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    num = np.abs(o_gpu - o_ref).max(axis=-1)
    den = np.abs(o_ref).max(axis=-1)
    return float((num / den).max())


def to_device_cache(ids_nat, norms, device):
    from hash_scored_top_b200 import api
    ids = api.natural_to_ids(torch.from_numpy(ids_nat)).to(device)
    return ids, torch.from_numpy(norms).to(device)
