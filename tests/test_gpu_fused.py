"""GPU parity of the fused target side, tr_compress_target_bags: the weighted-average
aggregation of TransRetrieval §3.2 building the compressor's input rows (§3.3) on chip.

Three checks on the same seeded tables and bags:
  - against the fp64 oracle (weighted average, concatenation in field order, compressor),
    at the intermediate bar of tests/common.py;
  - bit for bit against the two launches it replaces (tr_aggregate to bf16, then
    tr_compress_targets), whenever tr_aggregate takes its many-bags kernel, which sums in the
    same order;
  - empty bags, out-of-range keys and bad table ids behave as in tr_aggregate.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from common import check_close
from test_gpu_parity import _bags, _oracle_agg, _tables, dev, dims_of, tr

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _both(m, dims, tables, bags, n):
    """(fused tokens, two-launch tokens) for n candidates."""
    F, D = dims.n_target_fields, dims.D
    args = [dev(bags.bag_table), dev(bags.offsets), dev(bags.keys), dev(bags.weights)]
    fused = torch.empty(n, D, dtype=torch.float32, device="cuda")
    tr().compress_target_bags(m, tables, *args, fused)
    X = torch.empty(n * F, D, dtype=torch.bfloat16, device="cuda")
    tr().aggregate(tables, *args, X)
    two = torch.empty(n, D, dtype=torch.float32, device="cuda")
    tr().compress_targets(m, X.view(n, F * D), two)
    torch.cuda.synchronize()
    return fused, two


@pytest.mark.parametrize("name,n,init,max_nf", [
    ("128d5l", 300, "paper", 8),     # three tiles, a ragged one
    ("128d5l", 1000, "wide", 8),     # eight tiles
    ("128d5l", 130, "paper", 40),    # bags of several key chunks
    ("64d3l", 777, "wide", 8),       # one 64-column slice per field
    ("64d3l", 200, "paper", 30),     # ... with bags of several key chunks
    ("128d5l", 1, "wide", 8),        # one candidate
])
def test_fused_target_side_parity(name, n, init, max_nf):
    dims = dims_of(name)
    F, D = dims.n_target_fields, dims.D
    P = datagen.make_params(dims, 4, init)
    m = tr().Model(dims, P)
    rows, n_tables = 5000, 3
    tables = _tables(11, n_tables, rows, D, "bf16")
    bags = _bags(np.random.default_rng(n + D), n * F, max_nf, rows, n_tables)
    fused, two = _both(m, dims, tables, bags, n)
    assert tr().sync_status() == 0
    if n * F > 4 * _sms():
        assert torch.equal(fused, two)
    X = _oracle_agg(11, bags, rows, D, "bf16").reshape(n, F * D)
    ref = oracle.compress_targets(P, X)
    check_close(fused.double().cpu().numpy(), ref, "bf16", "tokens", kind="intermediate")


def test_fused_target_side_bad_keys_and_tables():
    """A key outside its table is skipped and reported; a bag naming no table gives a zero
    token; both exactly as the two launches handle them."""
    dims = dims_of("128d5l")
    F = dims.n_target_fields
    n = 200
    m = tr().Model(dims, datagen.make_params(dims, 4, "paper"))
    tables = _tables(11, 2, 3000, dims.D, "bf16")
    bags = _bags(np.random.default_rng(3), n * F, 8, 3000, 2, empty_frac=0.2)
    keys = bags.keys.copy()
    keys[5] = 3000
    keys[len(keys) // 2] = -1
    tab = bags.bag_table.copy()
    tab[17] = 2
    tab[40] = -3
    bad = datagen.Bags(bags.offsets, keys, bags.weights, tab)
    fused, two = _both(m, dims, tables, bad, n)
    assert tr().sync_status() == 4
    assert tr().sync_status() == 0
    assert torch.equal(fused, two)


def test_fused_target_side_refuses_unsupported_models():
    dims = dims_of("tiny")     # fp32 model: no tensor-core compressor
    m = tr().Model(dims, datagen.make_params(dims, 4, "paper"))
    tables = _tables(11, 1, 100, dims.D, "f32")
    z = torch.zeros(2, dtype=torch.int64, device="cuda")
    out = torch.empty(1, dims.D, dtype=torch.float32, device="cuda")
    with pytest.raises(Exception):
        tr().compress_target_bags(m, tables, z.int(), z, z.int(), z.float(), out)


@pytest.mark.parametrize("name,n_sample", [("128d5l", 64), ("large", 48)])
def test_fused_target_side_full_size(name, n_sample):
    """The full target sides of the 128D-5L request (40,000 candidates over eight 4M-row
    tables) and of the large one (520,000 candidates, one 52M-row table): bit-identical to
    the two launches, and the oracle on sampled candidates (the first and last included)."""
    from oracle.pipeline import _select_candidates, aggregate_bags
    from transformer_candidate_scoring_b200.pipeline import DeviceBags
    w = datagen.WORKLOADS[name]
    dims = w.dims
    F, D = dims.n_target_fields, dims.D
    P = datagen.workload_params(w)
    m = tr().Model(dims, P)
    tables = []
    for t, rows in enumerate(w.target_rows):   # the workload's target tables (the ids the oracle reads)
        x = torch.empty(rows, D, dtype=torch.bfloat16, device="cuda")
        datagen.fill_table_device(x, w.seed, datagen.target_table_id(w, t))
        tables.append(x)
    req = datagen.make_requests(w)[0]
    bags = DeviceBags.of(req.target, "cuda")
    n = req.n_cand
    args = [bags.bag_table, bags.offsets, bags.keys, bags.weights]
    fused = torch.empty(n, D, dtype=torch.float32, device="cuda")
    tr().compress_target_bags(m, tables, *args, fused)
    X = torch.empty(n * F, D, dtype=torch.bfloat16, device="cuda")
    tr().aggregate(tables, *args, X)
    two = torch.empty_like(fused)
    tr().compress_targets(m, X.view(n, F * D), two)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    assert torch.equal(fused, two)
    rng = np.random.default_rng(1)
    cand = np.unique(np.concatenate([rng.choice(n, size=n_sample, replace=False), [0, n - 1]]))
    ref = oracle.compress_targets(P, aggregate_bags(w, _select_candidates(req, cand, F), "target").reshape(-1, F * D))
    check_close(fused[torch.from_numpy(cand).cuda()].double().cpu().numpy(), ref, "bf16", "tokens",
                kind="intermediate")
    del tables, X, fused, two
    torch.cuda.empty_cache()


def test_fused_target_side_empty_call():
    """n = 0 launches nothing and leaves the output alone."""
    dims = dims_of("128d5l")
    m = tr().Model(dims, datagen.make_params(dims, 4, "paper"))
    tables = _tables(11, 1, 100, dims.D, "bf16")
    z = torch.zeros(1, dtype=torch.int64, device="cuda")
    out = torch.full((1, dims.D), 7.0, dtype=torch.float32, device="cuda")
    before = tr().api.kernel_launches()
    tr().compress_target_bags(m, tables, z.int(), z, z.int(), z.float(), out[:0])
    torch.cuda.synchronize()
    assert tr().api.kernel_launches() == before
    assert torch.all(out == 7.0)
