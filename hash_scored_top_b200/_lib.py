"""Loads libhash_scored_top.so (built in-tree) and declares its C signatures.

Importing this module fails loudly if the library has not been built
(``python -m hash_scored_top_b200.build``); nothing falls back to Python.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhash_scored_top.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m hash_scored_top_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_z = ctypes.c_size_t

# name -> (restype, argtypes); the order follows include/hash_scored_top.h
SIGNATURES = {
    "socket_hash_keys": (_i, [_p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "socket_score": (_i, [_p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _z, _p]),
    "socket_topk": (_i, [_p, _i, _i, _i, _i, _i, _p, _p, _z, _p]),
    "socket_sparse_attend": (_i, [_p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p, _z, _p]),
    "socket_sparse_attend_noalloc": (_i, [_p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p]),
    "sk_noalloc_scratch_bytes": (_z, []),
    "socket_decode": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _f, _p, _p, _p, _z,
                           _p]),
    "socket_decode_append": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _f, _p, _p, _p,
                                  _z, _p]),
    "socket_decode_step_host": (_i, [_p, _p, _p, _p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                                     _f, _p, _p, _p, _z, _p]),
    "socket_select": (_i, [_p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _p, _p, _z, _p]),
    "hata_hash_keys": (_i, [_p, _i, _p, _i, _i, _i, _i, _i, _i, _p, _p]),
    "hata_decode": (_i, [_p, _p, _p, _i, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _p, _z, _p]),
    "dense_decode": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _p, _p, _z, _p]),
    "socket_soft_count_attend": (_i, [_p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _f, _i, _p, _p, _z, _p]),
    "socket_decode_heads": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _f, _p, _p, _p,
                                 _z, _p]),
    "socket_decode_adaptive": (_i, [_p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _f, _i, _i,
                                    _f, _p, _p, _p, _p, _z, _p]),
    "socket_sparse_attend_paged": (_i, [_p, _p, _p, _i, _p, _i, _i, _i, _p, _i, _i, _i, _i, _i, _f, _p, _p, _z, _p]),
    "socket_decode_paged": (_i, [_p, _p, _p, _i, _p, _i, _i, _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                                 _f, _p, _p, _p, _z, _p]),
    "sk_workspace_bytes": (_z, [_i, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "sk_check_status": (_i, [_p]),
    "sk_profile_phases": (_i, [_p]),
    "sk_test_set_wait_limit": (_i, [ctypes.c_longlong]),
    "sk_last_error": (ctypes.c_char_p, []),
    "sk_version": (ctypes.c_char_p, []),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def last_error() -> str:
    return lib.sk_last_error().decode()


def version() -> str:
    return lib.sk_version().decode()
