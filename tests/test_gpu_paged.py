"""GPU parity of the paged K/V gather (device pools and pinned host pools)
against the oracle, through the C ABI.

Pools are built from a contiguous cache by scattering its pages over a
shuffled set of physical pages (with unused pages in between). The device
pool runs the same attention kernel as socket_sparse_attend on translated row
indices, so its output must equal that call's bit for bit; the host pool
gathers the rows first and attends with a different split, so it is held to
the oracle tolerance.
"""

import numpy as np
import pytest
import torch

from oracle import paged_ref as pr
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


def _paged(K, V, page_size, seed, spare=7):
    """Scatter K, V [B, Hkv, Ncap, d] into pools [num_pages, page_size, d] and a page table."""
    B, Hkv, Ncap, d = K.shape
    per = (Ncap + page_size - 1) // page_size
    num_pages = B * Hkv * per + spare
    g = torch.Generator().manual_seed(seed)
    phys = torch.randperm(num_pages, generator=g)[: B * Hkv * per].view(B, Hkv, per)
    Kp = torch.zeros(num_pages, page_size, d, dtype=K.dtype)
    Vp = torch.zeros_like(Kp)
    pad = per * page_size - Ncap
    Kpad = torch.nn.functional.pad(K, (0, 0, 0, pad)).view(B, Hkv, per, page_size, d)
    Vpad = torch.nn.functional.pad(V, (0, 0, 0, pad)).view(B, Hkv, per, page_size, d)
    Kp[phys.flatten()] = Kpad.reshape(-1, page_size, d)
    Vp[phys.flatten()] = Vpad.reshape(-1, page_size, d)
    return Kp, Vp, phys.int().contiguous()


def _case(seed, dtype, B, Hkv, G, N, d, k):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Ncap = (N + 31) // 32 * 32
    Q = torch.randn(B, Hkv * G, d, generator=g).to(dt)
    K = torch.randn(B, Hkv, Ncap, d, generator=g).to(dt)
    V = torch.randn(B, Hkv, Ncap, d, generator=g).to(dt)
    idx = torch.stack([torch.stack([torch.randperm(N, generator=g)[:k].sort().values for _ in range(Hkv)])
                       for _ in range(B)]).int()
    return Q, K, V, idx


def _oracle_check(O, Q, Kp, Vp, table, idx, page_size, scale, tol):
    B, Hkv, _ = table.shape
    G = Q.shape[1] // Hkv
    Kn, Vn = Kp.double().numpy(), Vp.double().numpy()
    for b in range(B):
        for h in range(Hkv):
            ref = pr.attend_subset_paged(Q[b, h * G:(h + 1) * G].double().numpy(), Kn, Vn, table[b, h].numpy(),
                                         idx[b, h].numpy(), page_size, scale)
            err = pa.row_rel_err(O[b, h * G:(h + 1) * G].cpu().numpy(), ref)
            assert err < tol, (err, b, h)


@pytest.mark.parametrize("dtype,B,Hkv,G,N,d,k,page_size", [
    ("bf16", 2, 2, 4, 4096, 128, 300, 16),
    ("bf16", 1, 3, 8, 5000, 128, 1000, 128),
    ("bf16", 2, 1, 2, 3000, 64, 77, 1),
    ("f32", 1, 2, 3, 2000, 128, 129, 64),
    ("f32", 2, 2, 1, 1000, 64, 33, 32),
])
def test_paged_attend_device_and_host_pools(api, dtype, B, Hkv, G, N, d, k, page_size):
    Q, K, V, idx = _case(k + page_size, dtype, B, Hkv, G, N, d, k)
    Kp, Vp, table = _paged(K, V, page_size, seed=k)
    scale = d ** -0.5
    tol = pa.BF16_TOL if dtype == "bf16" else pa.F32_TOL
    Qd, idxd, tabd = Q.to(DEV), idx.to(DEV), table.to(DEV)
    # device pool: the same kernel as the contiguous call, on translated rows
    O_dev = torch.empty(B, Hkv * G, d, device=DEV)
    api.socket_sparse_attend_paged(Qd, Kp.to(DEV), Vp.to(DEV), tabd, idxd, scale, O_dev)
    O_ref = torch.empty_like(O_dev)
    api.socket_sparse_attend(Qd, K.to(DEV), V.to(DEV), idxd, scale, O_ref)
    api.check_status()
    assert torch.equal(O_dev, O_ref)
    _oracle_check(O_dev, Q, Kp, Vp, table, idx, page_size, scale, tol)
    # pinned host pool: gathered over the host link, then attended
    O_host = torch.empty_like(O_dev)
    api.socket_sparse_attend_paged(Qd, Kp.pin_memory(), Vp.pin_memory(), tabd, idxd, scale, O_host)
    api.check_status()
    _oracle_check(O_host, Q, Kp, Vp, table, idx, page_size, scale, tol)


@pytest.mark.parametrize("name,page_size", [("llama8b", 64), ("qwen_l48_g8", 256)])
def test_decode_paged_matches_decode(api, name, page_size):
    w = {"llama8b": wl.shrink(wl.LLAMA_8B, B=2, Hkv=2, Hq=8, N=12000, k=12000 // 33),
         "qwen_l48_g8": wl.shrink(wl.QWEN3_30B, B=1, Hkv=2, Hq=16, N=6000, k=6000 // 50)}[name]
    inp = wl.make_inputs(w, DEV)
    ids_nat, norms, _ = pa.oracle_socket_cache(inp, w)
    ids, nrm = pa.to_device_cache(ids_nat, norms, DEV)
    Kp, Vp, table = _paged(inp["K"].cpu(), inp["V"].cpu(), page_size, seed=page_size)
    O = torch.empty(w.B, w.Hq, w.d, device=DEV)
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=DEV)
    api.socket_decode(inp["Q"], inp["K"], inp["V"], inp["R"], ids, nrm, w.N, w.L, w.P, w.tau, w.k, w.scale, O, idx)
    O_p = torch.empty_like(O)
    idx_p = torch.empty_like(idx)
    api.socket_decode_paged(inp["Q"], Kp.to(DEV), Vp.to(DEV), table.to(DEV), inp["R"], ids, nrm, w.N, w.L, w.P, w.tau,
                            w.k, w.scale, O_p, idx_p)
    api.check_status()
    assert torch.equal(idx, idx_p)
    assert torch.equal(O, O_p)
    O_h = torch.empty_like(O)
    api.socket_decode_paged(inp["Q"], Kp.pin_memory(), Vp.pin_memory(), table.to(DEV), inp["R"], ids, nrm, w.N, w.L,
                            w.P, w.tau, w.k, w.scale, O_h)
    api.check_status()
    _oracle_check(O_h, inp["Q"].cpu(), Kp, Vp, table, idx.cpu(), page_size, w.scale, pa.out_tol(w))


def test_page_table_entry_out_of_range_is_reported(api):
    Q, K, V, idx = _case(3, "bf16", 1, 2, 4, 512, 128, 64)
    Kp, Vp, table = _paged(K, V, 16, seed=3)
    bad = table.clone()
    bad[0, 1, 5] = Kp.shape[0] + 3            # past the pool
    idx[0, 1, 0] = 5 * 16 + 2                  # a selected key on that page
    O = torch.empty(1, 8, 128, device=DEV)
    for pool in [(Kp.to(DEV), Vp.to(DEV)), (Kp.pin_memory(), Vp.pin_memory())]:
        api.socket_sparse_attend_paged(Q.to(DEV), pool[0], pool[1], bad.to(DEV), idx.to(DEV), 0.1, O)
        with pytest.raises(RuntimeError, match="page-table entry"):
            api.check_status()
        assert torch.isfinite(O).all()
        # the next call with a good table is correct again
        api.socket_sparse_attend_paged(Q.to(DEV), pool[0], pool[1], table.to(DEV), idx.to(DEV), 0.1, O)
        api.check_status()
        _oracle_check(O, Q, Kp, Vp, table, idx, 16, 0.1, pa.BF16_TOL)


def test_pageable_host_pool_is_rejected(api):
    Q, K, V, idx = _case(4, "bf16", 1, 1, 1, 256, 64, 8)
    Kp, Vp, table = _paged(K, V, 32, seed=4)
    O = torch.empty(1, 1, 64, device=DEV)
    ws = torch.empty(1 << 22, dtype=torch.uint8, device=DEV)
    # the binding refuses unpinned host memory before the library sees it
    with pytest.raises(ValueError, match="pinned"):
        api.socket_sparse_attend_paged(Q.to(DEV), Kp, Vp, table.to(DEV), idx.to(DEV), 0.1, O, ws)
