"""The C-ABI library loads, exports every symbol include/tr.h declares, and rejects bad
arguments on the host before touching a GPU (these calls launch nothing)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(tr_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from transformer_candidate_scoring_b200 import build, _lib
    build.build()
    return _lib.load()


def test_header_declares_the_four_calls():
    names = declared_functions()
    for f in ("tr_aggregate", "tr_prefill_user", "tr_compress_targets", "tr_score_candidates"):
        assert f in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_host_validation_without_gpu(lib):
    from transformer_candidate_scoring_b200 import _lib as L
    assert lib.tr_version().startswith(b"libtr")
    assert lib.tr_kv_cache_bytes(None, 5) == 0
    # n_bags == 0 is a no-op; bad table count is rejected before any launch
    assert lib.tr_aggregate(None, 0, None, None, None, None, 0, 128, 1, None, None) == L.TR_OK
    t = (L.Table * 1)(L.Table(0, 10, 1))
    assert lib.tr_aggregate(t, 0, None, None, None, None, 5, 128, 1, None, None) == L.TR_ERR_INVALID_ARG
    assert b"n_tables" in lib.tr_last_error()
    assert lib.tr_aggregate(t, 1, None, None, None, None, 5, 128, 1, None, None) == L.TR_ERR_INVALID_ARG
    # unsupported model sizes are refused before allocation
    d = L.ModelDesc(96, 2, 4, 192, 8, (C.c_int * 4)(768, 384, 192, 96), 2, 1)   # d_h = 24
    h = C.c_void_p()
    assert lib.tr_model_create(C.byref(d), None, C.byref(h)) == L.TR_ERR_UNSUPPORTED
    d = L.ModelDesc(64, 2, 4, 128, 8, (C.c_int * 4)(500, 256, 128, 64), 2, 1)    # comp_dims[0] != F*D
    assert lib.tr_model_create(C.byref(d), None, C.byref(h)) == L.TR_ERR_INVALID_ARG
    assert lib.tr_score_candidates(None, None, 0, None, None, None, None, 1, None, None) == L.TR_ERR_INVALID_ARG


def test_topk_host_validation_without_gpu(lib):
    from transformer_candidate_scoring_b200 import _lib as L
    off = (C.c_int64 * 3)(0, 5, 9)
    assert lib.tr_topk(None, 9, off, 2, 0, None, None, None) == L.TR_ERR_INVALID_ARG          # k = 0
    assert lib.tr_topk(None, 9, off, 2, L.TR_MAX_TOPK + 1, None, None, None) == L.TR_ERR_INVALID_ARG
    assert lib.tr_topk(None, 9, off, 0, 5, None, None, None) == L.TR_ERR_INVALID_ARG          # R = 0
    assert lib.tr_topk(None, 8, off, 2, 5, None, None, None) == L.TR_ERR_INVALID_ARG          # offsets != n
    bad = (C.c_int64 * 3)(0, 6, 5)
    assert lib.tr_topk(None, 5, bad, 2, 5, None, None, None) == L.TR_ERR_INVALID_ARG          # decreasing
    assert lib.tr_topk(None, 9, off, 2, 5, None, None, None) == L.TR_ERR_INVALID_ARG          # null outputs
    assert b"null" in lib.tr_last_error()


def test_aggregate_ex_mode_validation_without_gpu(lib):
    from transformer_candidate_scoring_b200 import _lib as L
    t = (L.Table * 1)(L.Table(16, 10, 1))
    # unknown modes are rejected before anything else is looked at; n_bags == 0 is a no-op
    for bad in (3, 7, -1, 0x200, 0x100 | 5):
        assert lib.tr_aggregate_ex(t, 1, None, None, None, None, 5, 128, 1, bad, None, None) == L.TR_ERR_INVALID_ARG
        assert b"mode" in lib.tr_last_error()
    for ok in (0, 1, 2, 0x100, 0x101, 0x102):
        assert lib.tr_aggregate_ex(t, 1, None, None, None, None, 0, 128, 1, ok, None, None) == L.TR_OK


def test_uncompressed_host_validation_without_gpu(lib):
    from transformer_candidate_scoring_b200 import _lib as L
    # a null model handle is refused before anything else
    assert lib.tr_score_candidates_uncompressed(None, None, 0, 8, None, None, None, None, 1, None,
                                                None) == L.TR_ERR_INVALID_ARG


def test_fused_target_side_host_validation_without_gpu(lib):
    from transformer_candidate_scoring_b200 import _lib as L
    t = (L.Table * 1)(L.Table(16, 10, 1))
    # a null model is refused before any device call; the model check comes first
    assert lib.tr_compress_target_bags(None, t, 1, None, None, None, None, 5, None, None) == L.TR_ERR_INVALID_ARG
    assert b"model is null" in lib.tr_last_error()
    assert lib.tr_compress_target_bags(None, None, 0, None, None, None, None, 0, None, None) == L.TR_ERR_INVALID_ARG
    assert "tr_compress_target_bags" in declared_functions()
