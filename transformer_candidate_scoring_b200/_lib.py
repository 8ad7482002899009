"""ctypes declarations of libtr's C ABI (include/tr.h)."""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtr.so")

TR_OK, TR_ERR_INVALID_ARG, TR_ERR_UNSUPPORTED, TR_ERR_CUDA, TR_ERR_KEY_RANGE, TR_ERR_TIMEOUT, TR_ERR_NOMEM = range(7)
TR_F32, TR_BF16 = 0, 1
TR_MAX_TABLES, TR_MAX_REQUESTS, TR_MAX_LU = 64, 64, 256
TR_NOALLOC_SCRATCH_BYTES = 1 << 20
TR_MAX_TOPK = 4096
TR_MAX_LT = 16

_fp = C.POINTER(C.c_float)


class ModelDesc(C.Structure):
    _fields_ = [("D", C.c_int), ("n_layer", C.c_int), ("n_head", C.c_int), ("ffn_hidden", C.c_int),
                ("n_target_fields", C.c_int), ("comp_dims", C.c_int * 4), ("n_domains", C.c_int),
                ("dtype", C.c_int)]


class LayerWeights(C.Structure):
    _fields_ = [(n, _fp) for n in ("ln1_g", "ln1_b", "Wq", "bq", "Wk", "bk", "Wv", "bv", "Wo", "bo",
                                   "ln2_g", "ln2_b", "W1", "b1", "W2", "b2")]


class ModelWeights(C.Structure):
    _fields_ = [("domain_emb", _fp), ("layers", C.POINTER(LayerWeights)), ("lnf_g", _fp), ("lnf_b", _fp),
                ("w_head", _fp), ("b_head", C.c_float), ("comp_W", _fp * 3), ("comp_b", _fp * 3),
                ("comp_prelu", _fp * 2), ("comp_ln_g", _fp * 2), ("comp_ln_b", _fp * 2)]


class Table(C.Structure):
    _fields_ = [("data", C.c_void_p), ("n_rows", C.c_int64), ("dtype", C.c_int)]


SIGNATURES = {
    "tr_last_error": (C.c_char_p, []),
    "tr_version": (C.c_char_p, []),
    "tr_kernel_launches": (C.c_ulonglong, []),
    "tr_model_create": (C.c_int, [C.POINTER(ModelDesc), C.POINTER(ModelWeights), C.POINTER(C.c_void_p)]),
    "tr_model_destroy": (None, [C.c_void_p]),
    "tr_aggregate": (C.c_int, [C.POINTER(Table), C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                               C.c_int64, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "tr_aggregate_ex": (C.c_int, [C.POINTER(Table), C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                               C.c_int64, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "tr_kv_cache_bytes": (C.c_size_t, [C.c_void_p, C.c_int]),
    "tr_prefill_user": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "tr_prefill_user_noalloc": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p]),
    "tr_prefill_users": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_void_p]),
    "tr_compress_targets": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p]),
    "tr_compress_target_bags": (C.c_int, [C.c_void_p, C.POINTER(Table), C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                                          C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p]),
    "tr_score_candidates": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.POINTER(C.c_int64),
                                      C.POINTER(C.c_void_p), C.POINTER(C.c_int32), C.POINTER(C.c_int32),
                                      C.c_int, C.c_void_p, C.c_void_p]),
    "tr_score_candidates_uncompressed": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_int, C.POINTER(C.c_int64),
                                                   C.POINTER(C.c_void_p), C.POINTER(C.c_int32), C.POINTER(C.c_int32),
                                                   C.c_int, C.c_void_p, C.c_void_p]),
    "tr_topk": (C.c_int, [C.c_void_p, C.c_int64, C.POINTER(C.c_int64), C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                          C.c_void_p]),
    "tr_sync_status": (C.c_int, [C.c_void_p, C.c_int]),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libtr.so; raises if it is missing (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libtr.so not found at {path}; run transformer_candidate_scoring_b200.build")
        lib = C.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib
