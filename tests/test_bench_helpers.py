"""bench.py's host-side arithmetic: the algorithmic work it divides by (pinned to the
TransRetrieval §3.3 count in tests/golden) and the profile-traffic lookup."""
import json
import os
import shutil

import numpy as np

import bench
import datagen

HERE = os.path.dirname(os.path.abspath(__file__))


def test_stack_flops_match_golden():
    rows = json.load(open(os.path.join(HERE, "golden", "flops_per_candidate.json")))["rows"]
    dims = {64: datagen.WORKLOADS["64d3l"].dims, 128: datagen.WORKLOADS["128d5l"].dims}
    for r in rows:
        if r["L_t"] != 1:
            continue
        assert bench.stack_flops_per_candidate(dims[r["D"]], r["L_u"]) == r["with_self_and_head"]


def test_compressor_flops():
    # 2 * (1024*512 + 512*256 + 256*128) for the 128D-5L compressor dims
    assert bench.compressor_flops_per_candidate(datagen.WORKLOADS["128d5l"].dims) == 1_376_256


def test_aggregate_bytes_counts_rows_keys_headers_output():
    b = datagen.Bags(offsets=np.array([0, 2, 5], np.int64), keys=np.zeros(5, np.int32),
                     weights=np.ones(5, np.float32), bag_table=np.zeros(2, np.int32))
    # 5 rows * 128 * 2 + 5 * 8 + 2 * 12 + 8 + 2 * 128 * 2
    assert bench.aggregate_bytes(b, 128, 2, 2) == 1280 + 40 + 24 + 8 + 512


def test_profiled_traffic_follows_source_hash(tmp_path, monkeypatch):
    # a copy of the repository's profile and sources: the lookup works, and returns None
    # once a profiled source changes
    root = tmp_path
    (root / "profiles").mkdir()
    src = "transformer_candidate_scoring_b200/csrc"
    (root / src).mkdir(parents=True)
    for f in ("stack_tc.cu", "tc_common.cuh"):
        shutil.copy(os.path.join(bench.ROOT, src, f), root / src / f)
    for f in os.listdir(os.path.join(bench.ROOT, "profiles")):
        shutil.copy(os.path.join(bench.ROOT, "profiles", f), root / "profiles" / f)
    monkeypatch.setattr(bench, "ROOT", str(root))
    got = bench.profiled_traffic("stack_kernel")
    assert got is None or got > 0
    if got is not None:
        with open(root / src / "tc_common.cuh", "a") as fh:
            fh.write("\n// changed\n")
        assert bench.profiled_traffic("stack_kernel") is None
    assert bench.profiled_traffic("no_such_kernel") is None
