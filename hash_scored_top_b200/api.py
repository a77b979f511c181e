"""Python binding of libhash_scored_top.so (argument marshalling only).

Every function here checks tensor devices, dtypes and shapes, passes raw
pointers and sizes to the C entry point of the same name, and raises
``RuntimeError`` with the library's message on a non-zero status. All
compute happens in the library's CUDA kernels on the current torch stream;
torch only provides device memory (outputs and workspaces) and the stream.
Without a ``ws`` argument a workspace of the size sk_workspace_bytes gives is
allocated for the call; a ``ws`` that is passed goes to the library as it is
(no size query on the host), which rejects one that is too small.
There is no CPU fallback: if the library is missing the import of
``_lib`` fails loudly.
"""

from __future__ import annotations

import ctypes

import torch

from . import _lib

SK_F32, SK_BF16 = 0, 1
(OP_HASH_KEYS, OP_SCORE, OP_TOPK, OP_SPARSE_ATTEND, OP_DECODE, OP_HATA_HASH, OP_HATA_DECODE, OP_DENSE_DECODE,
 OP_SELECT, OP_SOFT_COUNT, OP_DECODE_HEADS, OP_DECODE_ADAPTIVE, OP_DECODE_ADAPTIVE_HEADS, OP_SPARSE_ATTEND_PAGED,
 OP_DECODE_PAGED) = range(15)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SK_F32
    if t.dtype == torch.bfloat16:
        return SK_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _pool_ptr(t):
    """A K/V pool: device memory, or pinned host memory that the device reads directly."""
    if t.is_cuda:
        return _ptr(t)
    if not (t.is_pinned() and t.is_contiguous()):
        raise ValueError("host pools must be pinned and contiguous (the device reads them directly)")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed (status {rc}): {_lib.last_error()}")


def _want(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return ws
    if ws is None or ws.numel() * ws.element_size() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws


def _ws_bytes(ws):
    return 0 if ws is None else ws.numel() * ws.element_size()


# ---------------------------------------------------------------- cache allocation / layout
def ids_bytes_per_key(L: int) -> int:
    """Bytes per key of the bucket-ID cache (see the C header)."""
    return 16 if L <= 16 else 32 if L <= 32 else 48 if L <= 48 else 64


def _chunk_size(L: int, chunk: int) -> int:
    if chunk == 0:
        return 16 if L <= 16 else 32
    return 16 if L <= 48 else 32


def _byte_positions(L: int, n: int, device) -> torch.Tensor:
    """pos[i, l]: byte of key i (i < n) that holds table l's ID (the rotated layout)."""
    r = torch.arange(n, device=device)[:, None] % 32
    ll = torch.arange(L, device=device)[None, :]
    c = (ll >= 32).long()
    S = torch.where(c == 1, _chunk_size(L, 1), _chunk_size(L, 0))
    return 32 * c + torch.remainder(ll - 32 * c - r, S)


def empty_ids(B: int, Hkv: int, Ncap: int, L: int, device="cuda") -> torch.Tensor:
    """Bucket-ID cache [B, Hkv, Ncap, ids_bytes_per_key(L)] uint8 (rotated key-major layout)."""
    return torch.zeros(B, Hkv, Ncap, ids_bytes_per_key(L), dtype=torch.uint8, device=device)


def empty_norms(B: int, Hkv: int, Ncap: int, device="cuda") -> torch.Tensor:
    return torch.zeros(B, Hkv, Ncap, dtype=torch.float16, device=device)


def empty_codes(B: int, Hkv: int, Ncap: int, device="cuda") -> torch.Tensor:
    """Hard-hash code cache [B, Hkv, Ncap, 16] uint8: byte j of key n holds code byte (j + n) mod 16."""
    return torch.zeros(B, Hkv, Ncap, 16, dtype=torch.uint8, device=device)


def ids_to_natural(ids: torch.Tensor, L: int) -> torch.Tensor:
    """Cache layout -> [B, Hkv, Ncap, L] with [.., n, l] the ID of table l (a byte gather, no arithmetic)."""
    B, H, n, _ = ids.shape
    pos = _byte_positions(L, n, ids.device).expand(B, H, n, L)
    return torch.gather(ids, -1, pos)


def natural_to_ids(nat: torch.Tensor) -> torch.Tensor:
    """[B, Hkv, Ncap, L] -> cache layout (inverse of ids_to_natural; padding bytes are 0)."""
    B, H, n, L = nat.shape
    out = torch.zeros(B, H, n, ids_bytes_per_key(L), dtype=nat.dtype, device=nat.device)
    pos = _byte_positions(L, n, nat.device).expand(B, H, n, L)
    return out.scatter_(-1, pos, nat)


# ---------------------------------------------------------------- entry points
def workspace_bytes(op: int, B, Hq, Hkv, Ncap, N, d, L=0, P=0, k=0) -> int:
    n = _lib.lib.sk_workspace_bytes(op, B, Hq, Hkv, Ncap, N, d, L, P, k)
    if n == ctypes.c_size_t(-1).value:
        raise ValueError("invalid shapes for workspace query")
    return n


def socket_hash_keys(K, V, R, L: int, P: int, ids, norms, n_begin: int = 0, n_count: int | None = None):
    """SOCKET step 1 for keys [n_begin, n_begin + n_count) of every pair (see the C header)."""
    B, Hkv, Ncap, d = K.shape
    n_count = Ncap - n_begin if n_count is None else n_count
    _want(V, K.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    rc = _lib.lib.socket_hash_keys(_ptr(K), _ptr(V), _dtype_code(K), _ptr(R), B, Hkv, Ncap, n_begin, n_count, d, L, P,
                                   _ptr(ids), _ptr(norms), _stream())
    _check(rc, "socket_hash_keys")


def socket_score(Q, R, ids, norms, N: int, L: int, P: int, tau: float, scores, ws=None):
    """SOCKET steps 2-3: scores [B, Hkv, Ncap] f32 for keys < N."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = ids.shape
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(scores, torch.float32, (B, Hkv, Ncap), "scores")
    _want(R, torch.bfloat16, (L * P, d), "R")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_SCORE, B, Hq, Hkv, Ncap, N, d, L, P, 0), Q.device, ws)
    rc = _lib.lib.socket_score(_ptr(Q), _dtype_code(Q), _ptr(R), _ptr(ids), _ptr(norms), B, Hq, Hkv, Ncap, N, d, L, P,
                               ctypes.c_float(tau), _ptr(scores), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_score")


def socket_topk(scores, N: int, k: int, idx):
    """SOCKET step 4 (selection): idx [B, Hkv, k] int32 ascending."""
    B, Hkv, Ncap = scores.shape
    _want(scores, torch.float32, scores.shape, "scores")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    rc = _lib.lib.socket_topk(_ptr(scores), B, Hkv, Ncap, N, k, _ptr(idx), None, 0, _stream())
    _check(rc, "socket_topk")


def socket_sparse_attend(Q, K, V, idx, scale: float, O, ws=None):
    """SOCKET step 4 (attention over idx): O [B, Hq, d] f32."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    k = idx.shape[-1]
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    _want(O, torch.float32, (B, Hq, d), "O")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_SPARSE_ATTEND, B, Hq, Hkv, Ncap, k, d, 0, 0, k), Q.device, ws)
    rc = _lib.lib.socket_sparse_attend(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(idx), B, Hq, Hkv, Ncap, d, k,
                                       ctypes.c_float(scale), _ptr(O), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_sparse_attend")


def socket_sparse_attend_noalloc(Q, K, V, idx, scale: float, O):
    """socket_sparse_attend for callers that cannot allocate device memory.

    The library keeps a fixed static device scratch (``noalloc_scratch_bytes()``
    bytes per GPU) for the attention partials, so this call allocates nothing;
    shapes that do not fit raise RuntimeError. All calls on a GPU share that
    scratch: calls that overlap on the GPU race. The first call on a device
    looks up the scratch address; make it before any stream capture.
    """
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    k = idx.shape[-1]
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    _want(O, torch.float32, (B, Hq, d), "O")
    rc = _lib.lib.socket_sparse_attend_noalloc(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(idx), B, Hq, Hkv,
                                               Ncap, d, k, ctypes.c_float(scale), _ptr(O), _stream())
    _check(rc, "socket_sparse_attend_noalloc")


def noalloc_scratch_bytes() -> int:
    """Bytes of the static scratch socket_sparse_attend_noalloc uses."""
    return int(_lib.lib.sk_noalloc_scratch_bytes())


def socket_decode(Q, K, V, R, ids, norms, N: int, L: int, P: int, tau: float, k: int, scale: float, O, idx_out=None,
                  ws=None):
    """The fused decode step (SOCKET steps 2-4)."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    if idx_out is not None:
        _want(idx_out, torch.int32, (B, Hkv, k), "idx_out")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DECODE, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_decode(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(R), _ptr(ids), _ptr(norms), B, Hq, Hkv,
                                Ncap, N, d, L, P, ctypes.c_float(tau), k, ctypes.c_float(scale), _ptr(O),
                                _ptr(idx_out), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_decode")


def socket_decode_heads(Q, K, V, R, ids, norms, N: int, L: int, P: int, tau: float, k: int, scale: float, O,
                        idx_out=None, ws=None):
    """The decode step with one index set per query head; idx_out: [B, Hq, k]."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    if idx_out is not None:
        _want(idx_out, torch.int32, (B, Hq, k), "idx_out")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DECODE_HEADS, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_decode_heads(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(R), _ptr(ids), _ptr(norms), B,
                                      Hq, Hkv, Ncap, N, d, L, P, ctypes.c_float(tau), k, ctypes.c_float(scale),
                                      _ptr(O), _ptr(idx_out), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_decode_heads")


def socket_decode_adaptive(Q, K, V, R, ids, norms, N: int, L: int, P: int, tau: float, mass: float, k_min: int,
                           k_max: int, scale: float, O, idx, kcount, per_head: bool = False, ws=None):
    """The decode step with the adaptive k; idx: [B, U, k_max], kcount: [B, U] (U = Hkv, or Hq per head)."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    U = Hq if per_head else Hkv
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    _want(idx, torch.int32, (B, U, k_max), "idx")
    _want(kcount, torch.int32, (B, U), "kcount")
    op = OP_DECODE_ADAPTIVE_HEADS if per_head else OP_DECODE_ADAPTIVE
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(op, B, Hq, Hkv, Ncap, N, d, L, P, k_max), Q.device, ws)
    rc = _lib.lib.socket_decode_adaptive(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(R), _ptr(ids), _ptr(norms),
                                         B, Hq, Hkv, Ncap, N, d, L, P, ctypes.c_float(tau), int(bool(per_head)),
                                         ctypes.c_float(mass), k_min, k_max, ctypes.c_float(scale), _ptr(O),
                                         _ptr(idx), _ptr(kcount), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_decode_adaptive")


def _want_pool(K_pool, V_pool, dtype, d):
    if K_pool.dtype != dtype or V_pool.dtype != dtype:
        raise TypeError(f"pools: dtypes {K_pool.dtype}, {V_pool.dtype}, expected {dtype}")
    if K_pool.dim() != 3 or tuple(K_pool.shape) != tuple(V_pool.shape) or K_pool.shape[2] != d:
        raise ValueError(f"pools: shapes {tuple(K_pool.shape)}, {tuple(V_pool.shape)}, expected [pages, page_size, {d}]")
    if not (K_pool.is_contiguous() and V_pool.is_contiguous()):
        raise ValueError("pools must be contiguous")
    if K_pool.device.type == "cpu" and not (K_pool.is_pinned() and V_pool.is_pinned()):
        raise ValueError("host pools must be pinned (the device reads them directly)")


def socket_sparse_attend_paged(Q, K_pool, V_pool, page_table, idx, scale: float, O, ws=None):
    """Sparse attention with K/V in a paged pool (device or pinned host memory).

    K_pool, V_pool: [num_pages, page_size, d]; page_table: [B, Hkv, max_pages] int32 (device);
    idx: [B, Hkv, k] int32 (device)."""
    B, Hq, d = Q.shape
    _, Hkv, max_pages = page_table.shape
    num_pages, page_size, _ = K_pool.shape
    k = idx.shape[-1]
    _want_pool(K_pool, V_pool, Q.dtype, d)
    _want(page_table, torch.int32, (B, Hkv, max_pages), "page_table")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    _want(O, torch.float32, (B, Hq, d), "O")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_SPARSE_ATTEND_PAGED, B, Hq, Hkv, 32, k, d, 1, 1, k), Q.device, ws)
    rc = _lib.lib.socket_sparse_attend_paged(_ptr(Q), _pool_ptr(K_pool), _pool_ptr(V_pool), _dtype_code(Q),
                                             _ptr(page_table), max_pages, page_size, num_pages, _ptr(idx), B, Hq,
                                             Hkv, d, k, ctypes.c_float(scale), _ptr(O), _ptr(ws), _ws_bytes(ws),
                                             _stream())
    _check(rc, "socket_sparse_attend_paged")


def socket_decode_paged(Q, K_pool, V_pool, page_table, R, ids, norms, N: int, L: int, P: int, tau: float, k: int,
                        scale: float, O, idx_out=None, ws=None):
    """The decode step with a paged K/V cache; ids and norms are the contiguous hashed-key cache."""
    B, Hq, d = Q.shape
    _, Hkv, max_pages = page_table.shape
    num_pages, page_size, _ = K_pool.shape
    Ncap = ids.shape[2]
    _want_pool(K_pool, V_pool, Q.dtype, d)
    _want(page_table, torch.int32, (B, Hkv, max_pages), "page_table")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    if idx_out is not None:
        _want(idx_out, torch.int32, (B, Hkv, k), "idx_out")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DECODE_PAGED, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_decode_paged(_ptr(Q), _pool_ptr(K_pool), _pool_ptr(V_pool), _dtype_code(Q),
                                      _ptr(page_table), max_pages, page_size, num_pages, _ptr(R), _ptr(ids),
                                      _ptr(norms), B, Hq, Hkv, Ncap, N, d, L, P, ctypes.c_float(tau), k,
                                      ctypes.c_float(scale), _ptr(O), _ptr(idx_out), _ptr(ws), _ws_bytes(ws),
                                      _stream())
    _check(rc, "socket_decode_paged")


def socket_decode_append(Q, K, V, R, ids, norms, N: int, L: int, P: int, tau: float, k: int, scale: float, O,
                         idx_out=None, ws=None):
    """One decoder step: hash key N - 1 into (ids, norms), then the decode over N keys."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    if idx_out is not None:
        _want(idx_out, torch.int32, (B, Hkv, k), "idx_out")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DECODE, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_decode_append(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(R), _ptr(ids), _ptr(norms), B,
                                       Hq, Hkv, Ncap, N, d, L, P, ctypes.c_float(tau), k, ctypes.c_float(scale),
                                       _ptr(O), _ptr(idx_out), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_decode_append")


def _host_ptr(t, name):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host tensor (pinned for asynchronous copies)")
    return ctypes.c_void_p(t.data_ptr())


def socket_decode_step_host(Q_host, K_new_host, V_new_host, Q, K, V, R, ids, norms, N: int, L: int, P: int,
                            tau: float, k: int, scale: float, O, O_host, ws=None):
    """One decode step from host buffers: Q_host [B, Hq, d] and the new token's rows K_new_host, V_new_host
    [B, Hkv, d] (pinned, K's dtype) are copied in (the rows to position N - 1 of K and V), the step runs as
    socket_decode_append, and O [B, Hq, d] float32 is copied to O_host (pinned). All on the current stream:
    O_host holds the result once the stream has synchronised."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(Q, K.dtype, (B, Hq, d), "Q")
    _want(V, K.dtype, K.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(O, torch.float32, (B, Hq, d), "O")
    _want(Q_host, K.dtype, (B, Hq, d), "Q_host")
    _want(K_new_host, K.dtype, (B, Hkv, d), "K_new_host")
    _want(V_new_host, K.dtype, (B, Hkv, d), "V_new_host")
    _want(O_host, torch.float32, (B, Hq, d), "O_host")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DECODE, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_decode_step_host(_host_ptr(Q_host, "Q_host"), _host_ptr(K_new_host, "K_new_host"),
                                          _host_ptr(V_new_host, "V_new_host"), _ptr(Q), _ptr(K), _ptr(V),
                                          _dtype_code(K), _ptr(R), _ptr(ids), _ptr(norms), B, Hq, Hkv, Ncap, N, d, L,
                                          P, ctypes.c_float(tau), k, ctypes.c_float(scale), _ptr(O),
                                          _host_ptr(O_host, "O_host"), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_decode_step_host")


def socket_select(Q, R, ids, norms, N: int, L: int, P: int, tau: float, k: int, idx, ws=None):
    """SOCKET steps 2-4 without the attention: idx [B, Hkv, k] int32 ascending."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = ids.shape
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(norms, torch.float16, (B, Hkv, Ncap), "norms")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_SELECT, B, Hq, Hkv, Ncap, N, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_select(_ptr(Q), _dtype_code(Q), _ptr(R), _ptr(ids), _ptr(norms), B, Hq, Hkv, Ncap, N, d, L,
                                P, ctypes.c_float(tau), k, _ptr(idx), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "socket_select")


def hata_hash_keys(K, R128, codes, n_begin: int = 0, n_count: int | None = None):
    """128-bit sign codes of keys [n_begin, n_begin + n_count) of every pair."""
    B, Hkv, Ncap, d = K.shape
    n_count = Ncap - n_begin if n_count is None else n_count
    _want(R128, torch.bfloat16, (128, d), "R128")
    _want(codes, torch.uint8, (B, Hkv, Ncap, 16), "codes")
    rc = _lib.lib.hata_hash_keys(_ptr(K), _dtype_code(K), _ptr(R128), B, Hkv, Ncap, n_begin, n_count, d, _ptr(codes),
                                 _stream())
    _check(rc, "hata_hash_keys")


def hata_decode(Q, K, V, R128, codes, N: int, k: int, scale: float, O, idx_out=None, ws=None):
    """Hard-hash decode step: Hamming scores, exact top-k, attention over the selection."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(R128, torch.bfloat16, (128, d), "R128")
    _want(codes, torch.uint8, (B, Hkv, Ncap, 16), "codes")
    _want(O, torch.float32, (B, Hq, d), "O")
    if idx_out is not None:
        _want(idx_out, torch.int32, (B, Hkv, k), "idx_out")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_HATA_DECODE, B, Hq, Hkv, Ncap, N, d, 16, 8, k), Q.device, ws)
    rc = _lib.lib.hata_decode(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), _ptr(R128), _ptr(codes), B, Hq, Hkv, Ncap, N,
                              d, k, ctypes.c_float(scale), _ptr(O), _ptr(idx_out), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "hata_decode")


def dense_decode(Q, K, V, N: int, scale: float, O, ws=None):
    """Dense decode attention over the first N cached keys."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = K.shape
    _want(K, Q.dtype, K.shape, "K")
    _want(V, Q.dtype, K.shape, "V")
    _want(O, torch.float32, (B, Hq, d), "O")
    if ws is None:                # a caller's workspace is passed as it is: the library checks its size
        ws = _workspace(workspace_bytes(OP_DENSE_DECODE, B, Hq, Hkv, Ncap, N, d), Q.device, ws)
    rc = _lib.lib.dense_decode(_ptr(Q), _ptr(K), _ptr(V), _dtype_code(K), B, Hq, Hkv, Ncap, N, d, ctypes.c_float(scale),
                               _ptr(O), _ptr(ws), _ws_bytes(ws), _stream())
    _check(rc, "dense_decode")


def socket_soft_count_attend(Q, V, R, ids, idx, L: int, P: int, tau: float, O, ws=None):
    """The soft-count attention estimator over the selected keys idx (see the C header)."""
    B, Hq, d = Q.shape
    _, Hkv, Ncap, _ = V.shape
    k = idx.shape[-1]
    _want(V, Q.dtype, V.shape, "V")
    _want(R, torch.bfloat16, (L * P, d), "R")
    _want(ids, torch.uint8, (B, Hkv, Ncap, ids_bytes_per_key(L)), "ids")
    _want(idx, torch.int32, (B, Hkv, k), "idx")
    _want(O, torch.float32, (B, Hq, d), "O")
    if ws is None:              # a caller's workspace is passed as it is: the library checks its size
        if ws is None:                # a caller's workspace is passed as it is: the library checks its size
            ws = _workspace(workspace_bytes(OP_SOFT_COUNT, B, Hq, Hkv, Ncap, k, d, L, P, k), Q.device, ws)
    rc = _lib.lib.socket_soft_count_attend(_ptr(Q), _ptr(V), _dtype_code(V), _ptr(R), _ptr(ids), _ptr(idx), B, Hq,
                                           Hkv, Ncap, d, L, P, ctypes.c_float(tau), k, _ptr(O), _ptr(ws),
                                           _ws_bytes(ws), _stream())
    _check(rc, "socket_soft_count_attend")


def check_status():
    """Synchronises the current stream and raises if a kernel flagged an error."""
    _check(_lib.lib.sk_check_status(_stream()), "sk_check_status")
