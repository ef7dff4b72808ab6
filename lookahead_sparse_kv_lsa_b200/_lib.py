"""ctypes view of the C ABI in include/lsa.h (liblsa_b200.so, built in-tree).

Argument marshalling only. Loading fails loudly when the shared library is missing:
there is no fallback implementation of any step.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblsa_b200.so")

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_CAPACITY, LSA_ERR_CUDA, LSA_ERR_TIMEOUT, \
    LSA_ERR_UNIMPLEMENTED = range(6)

DEVERR_SEL_CAPACITY = 1
DEVERR_POOL_CAPACITY = 2
DEVERR_BAD_PAGE = 4
DEVERR_BAD_SIZE = 8
DEVERR_TIMEOUT = 16
DEVERR_NUMERIC = 32

BLOCK = 64
TAU = 64

_p = C.c_void_p
_i32 = C.c_int32
_i64 = C.c_int64
_sz = C.c_size_t


class LsaState(C.Structure):
    """Mirror of `lsa_state` (field order and types as declared in lsa.h)."""
    _fields_ = [
        ("B", _i32), ("L", _i32), ("D", _i32), ("d_i", _i32), ("H", _i32), ("d", _i32),
        ("W", _i32), ("cap", _i32), ("max_cand", _i32), ("scale", C.c_float),
        ("w_q", _p), ("k_idx", _p), ("kidx_off", _p), ("bias", _p),
        ("host_pool", _p), ("host_blocks", _i64), ("host_blk_off", _p), ("nb0", _p),
        ("hbm_pool", _p), ("n_pages", _i64),
        ("n_cand", _p), ("sel_ids", _p), ("sel_cnt", _p), ("res_pages", _p), ("n_res", _p),
        ("block_table", _p), ("bt_stride", _i32),
        ("n_entries", _p), ("tail_len", _p),
        ("index_ws", _p), ("index_ws_bytes", _sz),
        ("attn_ws", _p), ("attn_ws_bytes", _sz),
        ("err", _p),
        ("kidx_layer_stride", _i64),
        ("kept_ids", _p), ("kept_pages", _p), ("kept_cnt", _p),
        ("gather_ws", _p), ("gather_ws_bytes", _sz),
    ]


# name -> (restype, argtypes)
SIGNATURES = {
    "lsa_status_str": (C.c_char_p, [_i32]),
    "lsa_version": (_i32, []),
    "lsa_index": (_i32, [_p, _p, _p, _p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _i32,
                         _p, _p, _p, _sz, _p, _p]),
    "lsa_index_ex": (_i32, [_p, _p, _p, _p, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p,
                            _i32, _p, _p, _p, _sz, _p, _p]),
    "lsa_index_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "lsa_index_lowrank": (_i32, [_p, _p, _p, _i32, _p, _p, _i64, _p, _p, _i32, _i32, _i32, _i32,
                                 _i32, _p, _p, _i32, _p, _p, _p, _sz, _p, _p]),
    "lsa_index_lowrank_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "lsa_gather": (_i32, [_p, _i64, _p, _p, _p, _i32, _p, _p, _i32, _i32, _i32, _p, _i64, _i32,
                          _i32, _p, _i32, _p, _p, _p]),
    "lsa_gather_delta": (_i32, [_p, _i64, _p, _p, _p, _i32, _p, _p, _i32, _i32, _i32, _p, _i64,
                                _i32, _i32, _p, _i32, _p, _p, _p, _p, _p, _sz, _p, _p, _p]),
    "lsa_gather_delta_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "lsa_decode_attn": (_i32, [_p, _p, _i64, _p, _i32, _p, _p, _i32, _i32, _i32, C.c_float, _p,
                               _p, _sz, _p, _p]),
    "lsa_decode_attn_workspace_size": (_sz, [_i32, _i32, _i32, _i32]),
    "lsa_decode_attn_noalloc": (_i32, [_p, _p, _i64, _p, _i32, _p, _p, _i32, _i32, _i32,
                                       C.c_float, _p, _p, _p]),
    "lsa_state_check": (_i32, [C.POINTER(LsaState)]),
    "lsa_state_size": (_sz, []),
    "lsa_load_window": (_i32, [C.POINTER(LsaState), _i32, _p]),
    "lsa_step": (_i32, [C.POINTER(LsaState), _i64, _p, _p, _p, _p, _p, _p]),
    "lsa_pass_setup": (_i32, [C.POINTER(LsaState), _i32, _p]),
    "lsa_append": (_i32, [C.POINTER(LsaState), _i64, _p, _p, _p]),
    "lsa_decode_step": (_i32, [C.POINTER(LsaState), _i64, _p, _p, _p, _p, _p]),
    "lsa_denoise_labels": (_i32, [_p, _i32, _i32, _i32, C.c_double, _i32, _p, _p, _p, _p, _i32,
                                  _p, _p, _p]),
    "lsa_wait_selftest": (_i32, [_p, C.c_uint32, _i64, _p, _p]),
}

_lib = None


def lib() -> C.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "liblsa_b200.so is not built; run `python -m lookahead_sparse_kv_lsa_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class LsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().lsa_status_str(status).decode()
        super().__init__("%s failed: %s (status %d)" % (fn, msg, status))


def check(fn: str, status: int) -> None:
    if status != LSA_OK:
        raise LsaError(fn, status)
