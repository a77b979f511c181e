"""The C-ABI library loads, exports every entry point its header declares, and
validates arguments on the host (no GPU needed: these paths launch nothing)."""

import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "hash_scored_top.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from hash_scored_top_b200 import build
    build.build()
    from hash_scored_top_b200 import _lib
    return _lib


def test_header_lists_the_path_entry_points():
    names = _declared_functions()
    for want in ("socket_hash_keys", "socket_score", "socket_topk", "socket_sparse_attend", "socket_decode",
                 "socket_decode_append", "socket_decode_step_host", "socket_select",
                 "hata_hash_keys", "hata_decode", "dense_decode", "sk_workspace_bytes", "sk_check_status",
                 "sk_last_error", "sk_version"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib.lib, name), f"{name} declared in the header but not exported"
        assert name in lib.SIGNATURES, f"{name} has no ctypes signature in the binding"
    assert "sm_100a" in lib.version()


def test_workspace_sizes(lib):
    from hash_scored_top_b200 import api
    # decode at the 100K-token Llama-8B-like shape: index list + attention partials + counters
    # + room for the pairs' table images (one 64 KB chunk each, used when the
    # selection takes more than one wave)
    idx_bytes = 397312                       # 32 pairs x 3103 int32, rounded up to 256 bytes
    part_bytes = 32 * 9 * 4 * 130 * 4        # 9 splits x 4 heads x (m, l, o[128]) per pair
    tables = 32 * 65536
    assert (api.workspace_bytes(api.OP_DECODE, 4, 32, 8, 102400, 102400, 128, 32, 8, 3103)
            == idx_bytes + part_bytes + 256 + tables)
    assert api.workspace_bytes(api.OP_SCORE, 4, 32, 8, 102400, 102400, 128, 32, 8, 0) == 32 * 65536
    assert api.workspace_bytes(api.OP_SCORE, 8, 32, 4, 143360, 143360, 128, 48, 8, 0) == 32 * 2 * 65536
    n = api.workspace_bytes(api.OP_SPARSE_ATTEND, 4, 32, 8, 102400, 102400, 128, 0, 0, 3103)
    assert n == part_bytes + 256
    assert api.workspace_bytes(api.OP_DENSE_DECODE, 1, 8, 8, 4096, 4096, 64) > 0
    with pytest.raises(ValueError):
        api.workspace_bytes(api.OP_DECODE, 1, 3, 2, 64, 64, 128, 8, 4, 8)     # Hq % Hkv != 0


def _rc_and_msg(lib, fn, *args):
    rc = fn(*args)
    return rc, lib.last_error()


def test_host_validation_rejects_without_launching(lib):
    L = lib.lib
    p = ctypes.c_void_p(256)         # never dereferenced: validation fails first
    null = None
    # socket_decode: NULL query
    rc, msg = _rc_and_msg(lib, L.socket_decode, null, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4, 0.5, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 1 and "Q is NULL" in msg
    # Hq not a multiple of Hkv
    rc, msg = _rc_and_msg(lib, L.socket_decode, p, p, p, 1, p, p, p, 1, 3, 2, 64, 64, 128, 8, 4, 0.5, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 1 and "multiple" in msg
    # unsupported head dim
    rc, msg = _rc_and_msg(lib, L.socket_decode, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 96, 8, 4, 0.5, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 2
    # k > N
    rc, msg = _rc_and_msg(lib, L.socket_decode, p, p, p, 1, p, p, p, 1, 4, 1, 64, 32, 128, 8, 4, 0.5, 33, 0.1, p,
                          null, null, 0, null)
    assert rc == 1 and "k=33" in msg
    # P too large for byte IDs
    rc, msg = _rc_and_msg(lib, L.socket_decode, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 9, 0.5, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 2 and "P=9" in msg
    # tau must be positive
    rc, msg = _rc_and_msg(lib, L.socket_decode, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4, 0.0, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 1 and "tau" in msg
    # Ncap not a multiple of 32
    rc, msg = _rc_and_msg(lib, L.socket_hash_keys, p, p, 1, p, 1, 1, 40, 0, 40, 128, 8, 4, p, p, null)
    assert rc == 1 and "Ncap" in msg
    # key range outside the cache
    rc, msg = _rc_and_msg(lib, L.socket_hash_keys, p, p, 1, p, 1, 1, 64, 60, 8, 128, 8, 4, p, p, null)
    assert rc == 1 and "range" in msg
    # score without a workspace
    rc, msg = _rc_and_msg(lib, L.socket_score, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4, 0.5, p, null, 0, null)
    assert rc == 5 and "workspace" in msg
    # sparse attention with too small a workspace
    rc, msg = _rc_and_msg(lib, L.socket_sparse_attend, p, p, p, 1, p, 1, 4, 1, 64, 128, 8, 0.1, p, p, 16, null)
    assert rc == 5
    # top-k with k = 0
    rc, msg = _rc_and_msg(lib, L.socket_topk, p, 1, 1, 64, 64, 0, p, null, 0, null)
    assert rc == 1
    # hard-hash decode with a group of 16 heads
    rc, msg = _rc_and_msg(lib, L.hata_decode, p, p, p, 1, p, p, 1, 16, 1, 64, 64, 128, 8, 0.1, p, null, null, 0, null)
    assert rc == 2 and "G=16" in msg
    # bucket IDs must allow 32-byte loads
    rc, msg = _rc_and_msg(lib, L.socket_select, p, 1, p, ctypes.c_void_p(272), p, 1, 4, 1, 64, 64, 128, 8, 4, 0.5, 8,
                          p, null, 0, null)
    assert rc == 1 and "ids must be 32-byte aligned" in msg
    # K rows are bulk-copied: 16-byte alignment
    rc, msg = _rc_and_msg(lib, L.socket_sparse_attend, p, ctypes.c_void_p(264), p, 1, p, 1, 4, 1, 64, 128, 8, 0.1, p,
                          p, 1 << 20, null)
    assert rc == 1 and "K must be 16-byte aligned" in msg
    # decode_append: workspace checked before anything is launched
    rc, msg = _rc_and_msg(lib, L.socket_decode_append, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4, 0.5, 8, 0.1, p,
                          null, null, 0, null)
    assert rc == 5 and "workspace" in msg
    # unknown dtype
    rc, msg = _rc_and_msg(lib, L.dense_decode, p, p, p, 7, 1, 4, 1, 64, 64, 128, 0.1, p, p, 1 << 20, null)
    assert rc == 1 and "dtype" in msg
    # decode step from host buffers: a missing host buffer, then a missing
    # workspace, both reported before any copy or launch
    rc, msg = _rc_and_msg(lib, L.socket_decode_step_host, null, p, p, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4,
                          0.5, 8, 0.1, p, p, p, 1 << 20, null)
    assert rc == 1 and "Q_host" in msg
    rc, msg = _rc_and_msg(lib, L.socket_decode_step_host, p, p, p, p, p, p, 1, p, p, p, 1, 4, 1, 64, 64, 128, 8, 4, 0.5,
                          8, 0.1, p, p, null, 0, null)
    assert rc == 5 and "workspace" in msg


def test_host_validation_of_the_later_entry_points(lib):
    """The per-head, adaptive, estimator and paged entry points reject bad
    arguments on the host, before any launch or device query."""
    L = lib.lib
    p = ctypes.c_void_p(256)
    null = None
    # per-head decode: k > N
    rc, msg = _rc_and_msg(lib, L.socket_decode_heads, p, p, p, 1, p, p, p, 1, 8, 2, 64, 32, 128, 8, 4, 0.5, 40,
                          0.1, p, null, null, 0, null)
    assert rc == 1 and "k=40" in msg
    # adaptive decode: mass outside (0, 1], k_min > k_max, k_max > N, per_head not 0/1
    for mass, kmin, kmax, ph, want in [(0.0, 1, 8, 0, "mass"), (1.5, 1, 8, 0, "mass"), (0.5, 9, 8, 0, "k_min"),
                                       (0.5, 1, 65, 0, "k_min"), (0.5, 1, 8, 2, "per_head")]:
        rc, msg = _rc_and_msg(lib, L.socket_decode_adaptive, p, p, p, 1, p, p, p, 1, 8, 2, 64, 64, 128, 8, 4, 0.5, ph,
                              mass, kmin, kmax, 0.1, p, p, p, null, 0, null)
        assert rc == 1 and want in msg, (mass, kmin, kmax, ph, msg)
    # adaptive decode: the index list and counts are required
    rc, msg = _rc_and_msg(lib, L.socket_decode_adaptive, p, p, p, 1, p, p, p, 1, 8, 2, 64, 64, 128, 8, 4, 0.5, 0,
                          0.5, 1, 8, 0.1, p, null, p, null, 0, null)
    assert rc == 1 and "idx is NULL" in msg
    # estimator: group of 9 heads, k = 0, no workspace
    rc, msg = _rc_and_msg(lib, L.socket_soft_count_attend, p, p, 1, p, p, p, 1, 9, 1, 64, 128, 8, 4, 0.5, 8, p,
                          null, 0, null)
    assert rc == 2 and "G=9" in msg
    rc, msg = _rc_and_msg(lib, L.socket_soft_count_attend, p, p, 1, p, p, p, 1, 8, 2, 64, 128, 8, 4, 0.5, 0, p,
                          null, 0, null)
    assert rc == 1 and "k=0" in msg
    rc, msg = _rc_and_msg(lib, L.socket_soft_count_attend, p, p, 1, p, p, p, 1, 8, 2, 64, 128, 8, 4, 0.5, 8, p,
                          null, 0, null)
    assert rc == 5 and "workspace" in msg
    # paged attention: page parameters must be >= 1, the page table present
    rc, msg = _rc_and_msg(lib, L.socket_sparse_attend_paged, p, p, p, 1, p, 4, 0, 8, p, 1, 8, 2, 128, 16, 0.1, p,
                          null, 0, null)
    assert rc == 1 and "page_size=0" in msg
    rc, msg = _rc_and_msg(lib, L.socket_sparse_attend_paged, p, p, p, 1, null, 4, 16, 8, p, 1, 8, 2, 128, 16, 0.1,
                          p, null, 0, null)
    assert rc == 1 and "page_table is NULL" in msg
    # paged decode: the pages must cover N keys
    rc, msg = _rc_and_msg(lib, L.socket_decode_paged, p, p, p, 1, p, 2, 16, 8, p, p, p, 1, 8, 2, 64, 64, 128, 8, 4,
                          0.5, 8, 0.1, p, null, null, 0, null)
    assert rc == 1 and "< N" in msg


def test_workspace_queries_of_the_later_entry_points(lib):
    from hash_scored_top_b200 import api
    # per-query-head decode: 128 units of group size 1
    n_heads = api.workspace_bytes(api.OP_DECODE_HEADS, 4, 32, 8, 102400, 102400, 128, 32, 8, 3103)
    n_group = api.workspace_bytes(api.OP_DECODE, 4, 32, 8, 102400, 102400, 128, 32, 8, 3103)
    assert n_heads > n_group > 0
    # adaptive decode: tables, scores (4 B per key and unit) and attention for k_max
    n_ad = api.workspace_bytes(api.OP_DECODE_ADAPTIVE, 4, 32, 8, 102400, 102400, 128, 32, 8, 12412)
    assert n_ad > 32 * 65536 + 32 * 102400 * 4
    assert api.workspace_bytes(api.OP_DECODE_ADAPTIVE_HEADS, 4, 32, 8, 102400, 102400, 128, 32, 8, 12412) > n_ad
    # estimator: factor image (f32, 32 per head and table), partials, counters
    n_est = api.workspace_bytes(api.OP_SOFT_COUNT, 4, 32, 8, 102400, 3103, 128, 32, 8, 3103)
    assert n_est >= 32 * 4 * 32 * 32 * 4
    # paged: a host pool stages k rows of K and V per pair
    n_pg = api.workspace_bytes(api.OP_SPARSE_ATTEND_PAGED, 4, 32, 8, 32, 3103, 128, 1, 1, 3103)
    assert n_pg >= 2 * 32 * 3103 * 128 * 4
    with pytest.raises(ValueError):
        api.workspace_bytes(api.OP_SOFT_COUNT, 1, 9, 1, 64, 8, 128, 8, 4, 8)       # G = 9
