"""GPU parity of the soft-count attention estimator against the oracle.

The estimator (SOCKET technical summary, section 主要な貢献 item 4) weights
the selected keys' values by their soft collision counts. Both sides read the
same bf16 / f32 values exactly. The GPU rounds the float64 factors of the soft
assignment to f32 and sums each count in f32, so every count is off by a
relative eps_i with |eps_i| <= (L + 2) u (u = 2^-24: two factor roundings,
one product, L - 1 additions); the weighted sums are f32 as well. For one
output element this gives |o - o_ref| <= 2 (n + 4) u sum_i c_i |v_i| / S +
2 (L + 3) u (sum_i c_i |v_i| / S + |o_ref|), S = sum_i c_i, with n the number
of terms on the longest summation path (at most k); the test evaluates the
bound from the oracle's counts.
"""

import numpy as np
import pytest
import torch

from oracle import estimator_ref as eo

pytestmark = pytest.mark.gpu

DEV = "cuda"
U = 2.0 ** -24


@pytest.fixture(scope="module")
def api():
    from hash_scored_top_b200 import build
    build.build()
    from hash_scored_top_b200 import api as _api
    return _api


def _inputs(seed, dtype, B, Hkv, G, N, d, L, P, k, ncap=None):
    g = torch.Generator().manual_seed(seed)
    ncap = ncap or (N + 31) // 32 * 32
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    Q = torch.randn(B, Hkv * G, d, generator=g).to(dt)
    V = torch.randn(B, Hkv, ncap, d, generator=g).to(dt)
    R = torch.randn(L * P, d, generator=g).to(torch.bfloat16)
    ids_nat = torch.randint(0, 1 << P, (B, Hkv, ncap, L), generator=g, dtype=torch.int64).to(torch.uint8)
    idx = torch.stack([torch.stack([torch.randperm(N, generator=g)[:k] for _ in range(Hkv)]) for _ in range(B)])
    return Q, V, R, ids_nat, idx.int()


def _run(api, Q, V, R, ids_nat, idx, L, P, tau):
    ids = api.natural_to_ids(ids_nat).to(DEV)
    O = torch.empty(Q.shape, dtype=torch.float32, device=DEV)
    api.socket_soft_count_attend(Q.to(DEV), V.to(DEV), R.to(DEV), ids, idx.to(DEV), L, P, tau, O)
    torch.cuda.synchronize()
    return O.cpu().numpy()


def _check(O, Q, V, R, ids_nat, idx, L, P, tau):
    B, Hkv = idx.shape[:2]
    G = Q.shape[1] // Hkv
    k = idx.shape[-1]
    Rn = R.double().numpy()
    worst = 0.0
    for b in range(B):
        for h in range(Hkv):
            Qg = Q[b, h * G:(h + 1) * G].double().numpy()
            Vp = V[b, h].double().numpy()
            ids_p = ids_nat[b, h].numpy()
            sel = idx[b, h].numpy()
            ref = eo.soft_count_attention(Qg, Vp, Rn, ids_p, sel, L, P, tau)
            for g_ in range(G):
                c = eo.soft_counts(Qg[g_], Rn, ids_p[sel], L, P, tau)
                wabs = (c @ np.abs(Vp[sel])) / c.sum()
                bound = 2 * (k + 4) * U * wabs + 2 * (L + 3) * U * (wabs + np.abs(ref[g_])) + 1e-30
                err = np.abs(O[b, h * G + g_] - ref[g_])
                assert (err <= bound).all(), (b, h, g_, float((err / bound).max()))
                worst = max(worst, float((err / bound).max()))
    return worst


@pytest.mark.parametrize("dtype,B,Hkv,G,N,d,L,P,k,tau", [
    ("bf16", 2, 2, 4, 8192, 128, 32, 8, 1000, 0.5),     # Llama-style group, one table chunk
    ("bf16", 1, 2, 8, 6000, 128, 48, 8, 300, 0.5),      # 48 tables, G = 8
    ("bf16", 1, 2, 8, 3000, 128, 64, 8, 777, 0.3),      # 64 tables: two factor chunks
    ("bf16", 4, 8, 4, 12000, 128, 32, 8, 9000, 0.5),    # many keys per CTA
    ("f32", 1, 2, 8, 3000, 128, 64, 8, 1000, 0.3),      # f32 rows, 64 tables: one CTA per SM, several splits
    ("bf16", 2, 1, 2, 2000, 64, 20, 6, 129, 0.4),       # d = 64
    ("f32", 1, 3, 3, 100, 128, 5, 3, 9, 0.7),           # small k, odd group
    ("f32", 2, 2, 1, 500, 64, 16, 4, 1, 1.0),           # one key
])
def test_soft_count_attend_matches_oracle(api, dtype, B, Hkv, G, N, d, L, P, k, tau):
    Q, V, R, ids_nat, idx = _inputs(k + L + d, dtype, B, Hkv, G, N, d, L, P, k)
    O = _run(api, Q, V, R, ids_nat, idx, L, P, tau)
    _check(O, Q, V, R, ids_nat, idx, L, P, tau)
    if k == 1:
        # one key: the output is its value, up to the two f32 roundings of
        # (c v) / c
        for b in range(B):
            for h in range(Hkv):
                want = V[b, h, int(idx[b, h, 0])].float().numpy()
                for g_ in range(G):
                    np.testing.assert_allclose(O[b, h * G + g_], want, rtol=2.5 * U, atol=0)


def test_soft_count_attend_is_deterministic(api):
    Q, V, R, ids_nat, idx = _inputs(5, "bf16", 2, 2, 4, 4096, 128, 32, 8, 700)
    a = _run(api, Q, V, R, ids_nat, idx, 32, 8, 0.5)
    b = _run(api, Q, V, R, ids_nat, idx, 32, 8, 0.5)
    assert np.array_equal(a, b)


def test_soft_count_attend_rejects_bad_arguments(api):
    Q, V, R, ids_nat, idx = _inputs(1, "bf16", 1, 1, 9, 64, 128, 4, 4, 8)
    # G = 9 > 8: the workspace query refuses the shapes, and so does the
    # entry point itself when handed a workspace
    with pytest.raises(ValueError):
        _run(api, Q, V, R, ids_nat, idx, 4, 4, 0.5)
    ids = api.natural_to_ids(ids_nat).to(DEV)
    O = torch.empty(Q.shape, dtype=torch.float32, device=DEV)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    with pytest.raises(RuntimeError, match="group size"):
        api.socket_soft_count_attend(Q.to(DEV), V.to(DEV), R.to(DEV), ids, idx.to(DEV), 4, 4, 0.5, O, ws=ws)
