"""socket_sparse_attend_noalloc: the sparse attention for callers that cannot
allocate device memory (a host whose memory manager has already reserved the
free HBM, or a latency-critical path where cudaMalloc / cudaFree and their
device synchronisation are not allowed). It keeps its partials in a fixed
static device array inside the library instead of a caller workspace.

The GPU test calls the new entry point through the C ABI twice in a row, on
different shapes, and checks each output against socket_sparse_attend with a
caller workspace and against the oracle's attention over the same keys, at
the tolerance the other attention tests use. It must pass
in a fresh process (the first call looks up the scratch address) and after
every other test (the scratch keeps the previous call's contents). The file
name makes pytest collect it last.
"""

import ctypes

import numpy as np
import pytest

from oracle import attention_ref as ao
from tests import parity as pa

DEV = "cuda"


@pytest.fixture(scope="module")
def lib():
    from hash_scored_top_b200 import build
    build.build()
    from hash_scored_top_b200 import _lib
    return _lib


def _noalloc_call(lib, Q, K, V, idx, scale, O):
    import torch
    from hash_scored_top_b200 import api
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    rc = lib.lib.socket_sparse_attend_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), api._dtype_code(K),
                                              idx.data_ptr(), B, Hq, Hkv, Ncap, d, idx.shape[-1],
                                              ctypes.c_float(scale), O.data_ptr(),
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.last_error()


def _case(w, seed):
    import torch
    from hash_scored_top_b200 import workloads as wl
    inp = wl.make_inputs(w, DEV)
    g = np.random.default_rng(seed)
    idx = np.stack([np.sort(g.choice(w.N, size=w.k, replace=False)) for _ in range(w.B * w.Hkv)])
    idx = torch.from_numpy(idx.reshape(w.B, w.Hkv, w.k).astype(np.int32)).to(DEV)
    return inp, idx


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    import torch
    from hash_scored_top_b200 import api
    from hash_scored_top_b200 import workloads as wl
    shapes = [wl.shrink(wl.LLAMA_8B, B=2, Hkv=4, Hq=16, N=20000, k=777),
              wl.shrink(wl.LLAMA_1B, B=3, Hkv=2, Hq=16, N=9000, k=300)]
    for call, w in enumerate(shapes):
        inp, idx = _case(w, 9100 + call)
        O_new = torch.full((w.B, w.Hq, w.d), float("nan"), device=DEV)
        _noalloc_call(lib, inp["Q"], inp["K"], inp["V"], idx, w.scale, O_new)
        api.check_status()
        O_ws = torch.empty(w.B, w.Hq, w.d, device=DEV)
        api.socket_sparse_attend(inp["Q"], inp["K"], inp["V"], idx, w.scale, O_ws)
        api.check_status()
        got, ref = O_new.cpu().numpy(), O_ws.cpu().numpy()
        assert np.isfinite(got).all(), call
        idx_h = idx.cpu().numpy()
        for p in range(w.B * w.Hkv):
            b, h = divmod(p, w.Hkv)
            rows = slice(h * w.G, (h + 1) * w.G)
            assert pa.row_rel_err(got[b, rows], ref[b, rows]) < pa.out_tol(w), (call, b, h)
            # and against the oracle's attention over the same subset
            Qg, K, V = pa.pair_arrays(inp, w, b, h)
            o_ref = ao.attend_subset(Qg, K, V, idx_h[b, h], w.scale)
            assert pa.row_rel_err(got[b, rows], o_ref) < pa.out_tol(w), (call, b, h)


def test_noalloc_rejects_shapes_beyond_the_static_scratch(lib):
    """Too many pairs for the fixed scratch: a workspace error, nothing launched
    (the pointers are never dereferenced, so this runs without a GPU)."""
    assert lib.lib.sk_noalloc_scratch_bytes() == 4 << 20
    p = ctypes.c_void_p(256)
    rc = lib.lib.socket_sparse_attend_noalloc(p, p, p, 1, p, 2048, 8, 1, 32, 128, 1, ctypes.c_float(0.1), p, None)
    msg = lib.last_error()
    assert rc == 5 and "static scratch" in msg and "4194304" in msg
