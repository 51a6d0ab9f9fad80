"""ctypes declarations of libsplitkv.so (include/splitkv.h).

Argument marshalling only: no computation happens on the Python side.
Loading fails loudly when the shared library has not been built.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsplitkv.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE_TOO_SMALL = -3
ERR_CUDA = -4
ERR_TIMEOUT = -5
ERR_NOT_UPLOADED = -6
ERR_NO_MEMORY = -7

FLAG_EQUAL_COUNT = 1
FLAG_BLOCK_KEYS_IN_CONTEXT = 2
FLAG_PARTIAL_BF16 = 4
FLAG_TILE_COST = 8
FLAG_FWD_TILE_COST = 16
FLAG_DYNAMIC_CLAIM = 32
FLAG_CONTIGUOUS_SCHEDULE = 64
FLAG_CONTIGUOUS_RANKS = 128

STATIC_SCRATCH_BYTES = 16 << 20

DTYPE_F32 = 0
DTYPE_BF16 = 1

WS_FWD = 0
WS_BWD = 1
TIMES_DQ = 2

EXPORT_ENTRIES = 0
EXPORT_CHUNK_PAIRS = 1
EXPORT_FWD_SCHEDULE = 2
EXPORT_BWD_SCHEDULE = 3
EXPORT_FWD_LOADS = 4
EXPORT_BWD_LOADS = 5
EXPORT_CONTIG_LOADS = 6
EXPORT_FWD_LPT_ORDER = 7
EXPORT_BWD_LPT_ORDER = 8
EXPORT_CHUNK_OWNER = 9
EXPORT_QUERY_SHARD = 10
MAX_RANKS = 4096


class Problem(ctypes.Structure):
    _fields_ = [
        ("num_samples", ctypes.c_int32),
        ("sample_lens", ctypes.POINTER(ctypes.c_int32)),
        ("num_anchors", ctypes.c_int32),
        ("anchors", ctypes.POINTER(ctypes.c_int32)),
        ("block_size", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("kv_chunk", ctypes.c_int32),
        ("num_workers", ctypes.c_int32),
        ("num_bwd_workers", ctypes.c_int32),
        ("q_slice", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
    ]


class Stats(ctypes.Structure):
    _fields_ = [
        ("context_len", ctypes.c_int64),
        ("num_queries", ctypes.c_int64),
        ("num_chunks", ctypes.c_int32),
        ("num_entries", ctypes.c_int32),
        ("num_tiles", ctypes.c_int32),
        ("num_fwd_items", ctypes.c_int32),
        ("num_bwd_items", ctypes.c_int32),
        ("num_workers", ctypes.c_int32),
        ("num_bwd_workers", ctypes.c_int32),
        ("context_pairs", ctypes.c_uint64),
        ("block_pairs", ctypes.c_uint64),
        ("fwd_max_load", ctypes.c_uint64),
        ("bwd_max_load", ctypes.c_uint64),
        ("fwd_imbalance", ctypes.c_double),
        ("bwd_imbalance", ctypes.c_double),
        ("contig_imbalance", ctypes.c_double),
        ("plan_us", ctypes.c_double),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/splitkv.h
SIGNATURES = {
    "splitkv_error_string": (ctypes.c_char_p, [_I]),
    "splitkv_plan": (_I, [ctypes.POINTER(Problem), ctypes.POINTER(_P)]),
    "splitkv_plan_update": (_I, [_P, ctypes.POINTER(Problem)]),
    "splitkv_plan_shard": (_I, [ctypes.POINTER(Problem), ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(_P)]),
    "splitkv_combine_ranks": (_I, [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _P, _P, _P, _I, _P, _P]),
    "splitkv_merge_to_owners": (_I, [_P, _P, _P, _P, _F, _P, _SZ, ctypes.c_int32, ctypes.c_int32, _P, _P, _P]),
    "splitkv_bwd_reduce_to_owners": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _SZ, ctypes.c_int32,
                                          ctypes.c_int32, _P, _P]),
    "splitkv_sum_ranks": (_I, [ctypes.c_int32, ctypes.c_int64, _P, _P, _P]),
    "splitkv_cast_bf16": (_I, [ctypes.c_int64, _P, _P, _P]),
    "splitkv_enable_peer_access": (_I, [ctypes.c_int32]),
    "splitkv_plan_upload": (_I, [_P, _P]),
    "splitkv_plan_destroy": (_I, [_P]),
    "splitkv_plan_stats": (_I, [_P, ctypes.POINTER(Stats)]),
    "splitkv_plan_export": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64,
                                 ctypes.POINTER(ctypes.c_int64)]),
    "splitkv_workspace_size": (_I, [_P, _I, ctypes.POINTER(_SZ)]),
    "splitkv_attn_fwd": (_I, [_P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_merge": (_I, [_P, _P, _P, _P, _F, _P, _SZ, _P, _I, _P, _P]),
    "splitkv_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_bwd_delta": (_I, [_P, _P, _I, _P, _P, _SZ, _P]),
    "splitkv_bwd_partial": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_bwd_reduce": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_bwd_dkdv": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_bwd_dq": (_I, [_P, _P, _P, _P, _P, _P, _F, _P, _SZ, _P]),
    "splitkv_attn_fwd_static_scratch": (_I, [_P, _P, _P, _P, _P, _P, _F, _P, _I, _P, _P]),
    "splitkv_plan_status": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
    "splitkv_plan_set_wait_limit": (_I, [_P, ctypes.c_int64]),
    "splitkv_selftest_exp2": (_I, [_P, _P, ctypes.c_int64, _P]),
    "splitkv_selftest_wait_timeout": (_I, [ctypes.POINTER(ctypes.c_int32), _P]),
    "splitkv_read_cta_times": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, _P]),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: the CUDA library has not been built "
            "(run `python -m context_block_sparse_b200.build` or __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
