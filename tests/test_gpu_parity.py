"""GPU parity: every stage of libtr against the fp64 oracle on the same seeded inputs.

Inputs come from ``datagen`` only (tables, bags, stand-alone tokens); the oracle never
reads anything the CUDA path produced.  Tolerances (tests/common.py, check_close): scores
within 1e-4 (fp32 models) or 2e-2 (bf16 models), both element by element (relative error
floored at the scores' rms) and in max-norm; intermediate bf16 outputs (K/V images,
compressed tokens) are held to the same max-norm bar and to a separate, named elementwise
bound.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from common import check_close, normwise_err, rel_err, score_topk_tol, topk_agrees
from kvdecode import decode_kv

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def lib():
    from transformer_candidate_scoring_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.init()
    yield


def tr():
    import transformer_candidate_scoring_b200 as t
    return t


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def dims_of(name):
    return datagen.WORKLOADS[name].dims


# ---------------------------------------------------------------- aggregation (§3.2)

def _bags(rng, n_bags, max_nf, n_rows, n_tables, empty_frac=0.1):
    counts = rng.integers(1, max_nf + 1, size=n_bags)
    counts[rng.random(n_bags) < empty_frac] = 0
    off = np.zeros(n_bags + 1, np.int64)
    np.cumsum(counts, out=off[1:])
    keys = rng.integers(0, n_rows, size=int(off[-1])).astype(np.int32)
    w = rng.uniform(0.1, 1.0, size=len(keys)).astype(np.float32)
    tab = rng.integers(0, n_tables, size=n_bags).astype(np.int32)
    return datagen.Bags(off, keys, w, tab)


def _tables(seed, n_tables, rows, D, dt):
    ts = []
    for t in range(n_tables):
        x = torch.empty(rows, D, dtype=tdt(dt), device="cuda")
        datagen.fill_table_device(x, seed, t)
        ts.append(x)
    return ts


def _oracle_agg(seed, bags, rows, D, dt):
    tab_of_key = np.repeat(bags.bag_table.astype(np.int64), np.diff(bags.offsets))
    out_rows = np.zeros((len(bags.keys), D))
    for t in np.unique(tab_of_key):
        sel = tab_of_key == t
        out_rows[sel] = datagen.table_rows_host(seed, int(t), bags.keys[sel], D, dt)
    return oracle.weighted_average(out_rows, bags.offsets, np.arange(len(bags.keys)), bags.weights)


def _run_agg(tables, bags, D, out_dtype):
    out = torch.empty(bags.n_bags, D, dtype=out_dtype, device="cuda")
    tr().aggregate(tables, dev(bags.bag_table), dev(bags.offsets), dev(bags.keys), dev(bags.weights), out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dt,D", [("f32", 32), ("bf16", 64), ("bf16", 128), ("f32", 128), ("bf16", 32)])
@pytest.mark.parametrize("out_dt", ["f32", "bf16"])
@pytest.mark.parametrize("n_bags,max_nf", [(1237, 100), (9001, 8), (6007, 70), (300, 400), (37, 3000), (500, 8)])
def test_aggregate_parity(dt, D, out_dt, n_bags, max_nf):
    """Few long bags and many short ones: bags longer than the rows a lane group keeps in
    flight and than one key chunk, empty bags, and 1 to 8 bags per warp (D and dtype set
    the lanes per row).  Calls of at most 4 bags per SM take the block-per-bag kernel
    (300, 37 and 500 bags here), bags of up to 3000 rows spanning several key chunks of
    every lane group."""
    rng = np.random.default_rng(D + n_bags)
    rows = 5000
    tables = _tables(11, 3, rows, D, dt)
    bags = _bags(rng, n_bags, max_nf, rows, 3)
    got = _run_agg(tables, bags, D, tdt(out_dt)).double().cpu().numpy()
    ref = _oracle_agg(11, bags, rows, D, dt)
    # fp32 accumulation error scales with the summands (table values), not with the
    # possibly cancelling result; bf16 output adds one rounding of the result.
    scale = float(np.abs(ref).max())
    err = np.abs(got - ref)
    if out_dt == "f32":
        assert np.all(err <= 1e-6 * scale), float(err.max() / scale)
    else:
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6 * scale), rel_err(got, ref)
    empty = np.diff(bags.offsets) == 0
    assert np.all(got[empty] == 0)
    assert tr().sync_status() == 0


def _oracle_agg_mode(seed, bags, rows, D, dt, mode, post_ln):
    tab_of_key = np.repeat(bags.bag_table.astype(np.int64), np.diff(bags.offsets))
    out_rows = np.zeros((len(bags.keys), D))
    for t in np.unique(tab_of_key):
        sel = tab_of_key == t
        out_rows[sel] = datagen.table_rows_host(seed, int(t), bags.keys[sel], D, dt)
    return oracle.aggregate(out_rows, bags.offsets, np.arange(len(bags.keys)), bags.weights, mode, post_ln)


@pytest.mark.parametrize("mode", ["mean", "sum", "max"])
@pytest.mark.parametrize("post_ln", [False, True])
@pytest.mark.parametrize("dt,D", [("bf16", 128), ("f32", 64), ("bf16", 32)])
@pytest.mark.parametrize("n_bags,max_nf", [(2500, 40), (200, 600)])
def test_aggregate_variants_parity(mode, post_ln, dt, D, n_bags, max_nf):
    """The §3.2 alternatives (weighted sum, max pooling, post-aggregation LayerNorm) against
    the oracle, through both kernels (200 bags: block per bag); max pooling without
    LayerNorm is exact."""
    rng = np.random.default_rng(D + len(mode) + post_ln + n_bags)
    rows = 3000
    tables = _tables(12, 2, rows, D, dt)
    bags = _bags(rng, n_bags, max_nf, rows, 2)
    out = torch.empty(bags.n_bags, D, dtype=torch.float32, device="cuda")
    tr().aggregate(tables, dev(bags.bag_table), dev(bags.offsets), dev(bags.keys), dev(bags.weights), out,
                   mode=mode, post_ln=post_ln)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    ref = _oracle_agg_mode(12, bags, rows, D, dt, mode, post_ln)
    empty = np.diff(bags.offsets) == 0
    assert np.all(got[empty] == 0)
    if mode == "max" and not post_ln:
        assert np.array_equal(got, ref)
    elif post_ln:
        # LayerNorm output is O(1); fp32 accumulation and normalisation
        np.testing.assert_allclose(got, ref, rtol=0, atol=2e-4)
    else:
        scale = float(np.abs(ref).max())
        assert np.all(np.abs(got - ref) <= 2e-6 * scale), float(np.abs(got - ref).max() / scale)
    assert tr().sync_status() == 0


def test_aggregate_variants_skip_and_report_out_of_range_keys():
    rng = np.random.default_rng(17)
    tables = _tables(5, 1, 1000, 64, "bf16")
    bags = _bags(rng, 300, 10, 1000, 1, empty_frac=0.0)
    bad = bags.keys.copy()
    bad[[2, 50]] = [1000, -3]
    keep = np.ones(len(bad), bool)
    keep[[2, 50]] = False
    cnt = np.array([keep[bags.offsets[b]:bags.offsets[b + 1]].sum() for b in range(300)])
    off = np.zeros(301, np.int64)
    np.cumsum(cnt, out=off[1:])
    clean = datagen.Bags(off, bags.keys[keep], bags.weights[keep], bags.bag_table)
    for mode in ("sum", "max"):
        out = torch.empty(300, 64, dtype=torch.float32, device="cuda")
        tr().aggregate(tables, dev(bags.bag_table), dev(bags.offsets), dev(bad), dev(bags.weights), out, mode=mode)
        torch.cuda.synchronize()
        assert tr().sync_status() == 4, mode
        ref = _oracle_agg_mode(5, clean, 1000, 64, "bf16", mode, False)
        np.testing.assert_allclose(out.double().cpu().numpy(), ref, rtol=1e-5, atol=1e-7)


def test_aggregate_scale_invariance_is_bitexact():
    rng = np.random.default_rng(5)
    tables = _tables(3, 2, 3000, 128, "bf16")
    bags = _bags(rng, 500, 40, 3000, 2)
    a = _run_agg(tables, bags, 128, torch.float32)
    for c in (4.0, 0.125, 1024.0):
        b = _run_agg(tables, datagen.scale_weights(bags, c), 128, torch.float32)
        assert torch.equal(a, b)


def test_aggregate_single_key_returns_row_exactly():
    rng = np.random.default_rng(6)
    tables = _tables(4, 1, 2000, 128, "bf16")
    keys = rng.integers(0, 2000, size=300).astype(np.int32)
    # (v * h) * (1 / v) is exact in binary floating point when v is a power of two
    w = (2.0 ** rng.integers(-6, 6, size=300)).astype(np.float32)
    bags = datagen.Bags(np.arange(301, dtype=np.int64), keys, w, np.zeros(300, np.int32))
    got = _run_agg(tables, bags, 128, torch.float32)
    want = tables[0][torch.from_numpy(keys).long().cuda()].float()
    assert torch.equal(got, want)
    # any other weight: within the roundings of v * h, of 1 / v and of their product (3 half-ulps)
    bags = datagen.Bags(bags.offsets, keys, rng.uniform(0.1, 1, 300).astype(np.float32), bags.bag_table)
    got = _run_agg(tables, bags, 128, torch.float32)
    assert torch.all(torch.abs(got - want) <= 2.0 ** -22 * torch.abs(want))


@pytest.mark.parametrize("n_bags", [50, 5000])
def test_aggregate_out_of_range_key_is_skipped_and_reported(n_bags):
    rng = np.random.default_rng(7)
    tables = _tables(5, 1, 1000, 64, "bf16")
    bags = _bags(rng, n_bags, 10, 1000, 1, empty_frac=0.0)
    bad = bags.keys.copy()
    bad[3] = 1000           # one past the end
    bad[7] = -5
    bad[len(bad) - 2] = 2 ** 30
    got = _run_agg(tables, datagen.Bags(bags.offsets, bad, bags.weights, bags.bag_table), 64, torch.float32)
    assert tr().sync_status() == 4
    assert tr().sync_status() == 0          # the word is cleared by the read
    keep = np.ones(len(bad), bool)
    keep[[3, 7, len(bad) - 2]] = False
    cnt = np.array([keep[bags.offsets[b]:bags.offsets[b + 1]].sum() for b in range(n_bags)])
    off = np.zeros(n_bags + 1, np.int64)
    np.cumsum(cnt, out=off[1:])
    ref = _oracle_agg(5, datagen.Bags(off, bags.keys[keep], bags.weights[keep], bags.bag_table), 1000, 64, "bf16")
    np.testing.assert_allclose(got.double().cpu().numpy(), ref, rtol=1e-5, atol=1e-7)


# ---------------------------------------------------------------- prefill (§3.1, §3.4)

@pytest.mark.parametrize("name,L_u,init", [("tiny", 8, "paper"), ("tiny", 1, "wide"), ("64d3l", 32, "wide"),
                                           ("128d5l", 64, "paper"), ("128d5l", 64, "wide"),
                                           ("128d5l", 128, "wide"), ("128d5l", 37, "wide"),
                                           ("128d5l", 256, "wide")])
def test_prefill_parity(name, L_u, init):
    dims = dims_of(name)
    P = datagen.make_params(dims, 3, init)
    m = tr().Model(dims, P)
    U = datagen.rand_matrix(21, (L_u, dims.D), 0.3 if init == "wide" else 0.01, "f32")
    kv = torch.zeros(tr().kv_cache_bytes(m, L_u), dtype=torch.uint8, device="cuda")
    tr().prefill_user(m, dev(U), L_u, 1, kv)
    torch.cuda.synchronize()
    dec = decode_kv(kv.cpu().numpy(), dims.dtype, dims.n_layer, L_u, dims.D)
    K, V = oracle.prefill_user(P, dims.n_head, U, 1)
    for l in range(dims.n_layer):
        check_close(dec[0][l], K[l], dims.dtype, f"K layer {l}", kind="intermediate")
        check_close(dec[1][l], V[l], dims.dtype, f"V layer {l}", kind="intermediate")
    if dims.dtype == "bf16":
        assert np.all(dec[2] == 0) and np.all(dec[3] == 0)     # zero padding rows


# ---------------------------------------------------------------- compressor (§3.3)

@pytest.mark.parametrize("name,n,init", [("tiny", 300, "paper"), ("64d3l", 300, "wide"), ("128d5l", 257, "paper"),
                                         ("128d5l", 1000, "wide"), ("128d5l", 1, "wide")])
def test_compress_parity(name, n, init):
    dims = dims_of(name)
    P = datagen.make_params(dims, 4, init)
    m = tr().Model(dims, P)
    X = datagen.rand_matrix(22, (n, dims.comp_dims[0]), 0.3 if init == "wide" else 0.01, dims.dtype)
    out = torch.empty(n, dims.D, dtype=torch.float32, device="cuda")
    tr().compress_targets(m, dev(X, tdt(dims.dtype)), out)
    torch.cuda.synchronize()
    ref = oracle.compress_targets(P, X)
    got = out.double().cpu().numpy()
    check_close(got, ref, dims.dtype, "tokens", kind="intermediate")


# ---------------------------------------------------------------- candidate stack (§3.3)

def _score_setup(name, init, L_us, n_per, seed=5, token_std=None):
    dims = dims_of(name)
    P = datagen.make_params(dims, seed, init)
    m = tr().Model(dims, P)
    std_u = 0.3 if init == "wide" else 0.01
    std_t = token_std or (0.5 if init == "wide" else 0.3)
    users = [datagen.rand_matrix(100 + r, (L, dims.D), std_u, "f32") for r, L in enumerate(L_us)]
    toks = [datagen.rand_matrix(200 + r, (n, dims.D), std_t, dims.dtype) for r, n in enumerate(n_per)]
    doms = [r % dims.n_domains for r in range(len(L_us))]
    kvs = []
    for r, L in enumerate(L_us):
        kv = torch.zeros(max(tr().kv_cache_bytes(m, L), 16), dtype=torch.uint8, device="cuda")
        if L:
            tr().prefill_user(m, dev(users[r]), L, doms[r], kv)
        kvs.append(kv)
    return dims, P, m, users, toks, doms, kvs


def _gpu_scores(m, dims, toks, kvs, L_us, doms):
    T = dev(np.concatenate(toks), torch.float32)
    off = np.concatenate([[0], np.cumsum([len(t) for t in toks])])
    s = torch.empty(int(off[-1]), dtype=torch.float32, device="cuda")
    tr().score_candidates(m, T, off.tolist(), kvs, L_us, doms, s)
    torch.cuda.synchronize()
    return s.cpu().numpy().astype(np.float64), off


def _oracle_scores(P, dims, users, toks, doms):
    out = []
    for U, t, d in zip(users, toks, doms):
        K, V = oracle.prefill_user(P, dims.n_head, U, d)
        out.append(oracle.score_candidates(P, dims.n_head, t, K, V, d))
    return np.concatenate(out)


@pytest.mark.parametrize("name,init,L_u,n", [("tiny", "paper", 8, 256), ("tiny", "wide", 8, 300),
                                             ("64d3l", "wide", 32, 300), ("64d3l", "paper", 32, 129),
                                             ("128d5l", "paper", 64, 300), ("128d5l", "wide", 64, 300),
                                             ("128d5l", "wide", 128, 130), ("128d5l", "wide", 1, 64),
                                             ("128d5l", "wide", 0, 50), ("128d5l", "wide", 256, 40),
                                             ("128d5l", "wide", 64, 1)])
def test_score_parity(name, init, L_u, n):
    dims, P, m, users, toks, doms, kvs = _score_setup(name, init, [L_u], [n])
    got, _ = _gpu_scores(m, dims, toks, kvs, [L_u], doms)
    ref = _oracle_scores(P, dims, users, toks, doms)
    print(check_close(got, ref, dims.dtype, "scores"))
    # the candidate-dependent part alone, relative to its own spread
    if n > 1:
        ec = np.max(np.abs((got - got.mean()) - (ref - ref.mean()))) / ref.std()
        assert ec < (5e-4 if dims.dtype == "f32" else 6e-2), ec


def test_packed_requests_are_isolated_and_match_single_runs():
    L_us = [16, 128, 0, 77, 1, 64]
    n_per = [130, 40, 17, 256, 3, 200]
    dims, P, m, users, toks, doms, kvs = _score_setup("128d5l", "wide", L_us, n_per)
    packed, off = _gpu_scores(m, dims, toks, kvs, L_us, doms)
    for r in range(len(L_us)):
        single, _ = _gpu_scores(m, dims, [toks[r]], [kvs[r]], [L_us[r]], [doms[r]])
        assert np.array_equal(single, packed[off[r]:off[r + 1]]), r
    ref = _oracle_scores(P, dims, users, toks, doms)
    for r in range(len(L_us)):
        check_close(packed[off[r]:off[r + 1]], ref[off[r]:off[r + 1]], "bf16", f"request {r}")


def test_scores_independent_of_batch_mates_bitexact():
    dims, P, m, users, toks, doms, kvs = _score_setup("128d5l", "wide", [64], [700])
    full, _ = _gpu_scores(m, dims, toks, kvs, [64], doms)
    rng = np.random.default_rng(1)
    for idx in (np.arange(0, 700, 3), rng.permutation(700)[:129], np.array([699])):
        sub, _ = _gpu_scores(m, dims, [toks[0][idx]], kvs, [64], doms)
        assert np.array_equal(sub, full[idx])


# ---------------------------------------------------------------- whole request

def _pipeline(name, n_cand, rows, init="paper", seed=None):
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    w = datagen.scaled(datagen.WORKLOADS[name], n_cand_per_request=n_cand, rows=rows, seed=seed)
    P = datagen.make_params(w.dims, w.seed, init)
    dw = DeviceWorkload(w, params=P)
    dw.step()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    return w, P, dw


@pytest.mark.parametrize("name,n,rows,init", [("tiny", 256, None, "paper"), ("64d3l", 1500, 20000, "paper"),
                                              ("128d5l", 1000, 20000, "wide"), ("packed", 70, 20000, "paper")])
def test_pipeline_end_to_end(name, n, rows, init):
    w, P, dw = _pipeline(name, n, rows, init)
    got = dw.scores.double().cpu().numpy()
    for r, req in enumerate(dw.reqs):
        ref = oracle.score_request(w, P, req).scores
        g = got[dw.req_offsets[r]:dw.req_offsets[r + 1]]
        print(r, check_close(g, ref, w.dims.dtype, f"request {r}"))
        tol_abs = score_topk_tol(ref, w.dims.dtype)
        k = min(100, len(ref))
        idx = np.lexsort((np.arange(len(g)), -g))[:k]
        ok, why = topk_agrees(idx, ref, k, tol_abs)
        assert ok, why


@pytest.mark.parametrize("name,n_sample", [("128d5l", 96), ("packed", 48), ("large", 64)])
def test_full_size_sampled(name, n_sample):
    """The full workload sizes (tables, candidate counts), oracle on sampled candidates."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    w = datagen.WORKLOADS[name]
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    got = dw.scores.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    P = dw.params
    rng = np.random.default_rng(0)
    for r in range(0, len(dw.reqs), max(1, len(dw.reqs) // 3)):
        req = dw.reqs[r]
        cand = np.sort(rng.choice(req.n_cand, size=min(n_sample, req.n_cand), replace=False))
        if r == 0:
            cand = np.unique(np.concatenate([cand, [0, req.n_cand - 1]]))
        ref = oracle.score_request(w, P, req, cand=cand).scores
        g = got[dw.req_offsets[r] + cand]
        print(r, check_close(g, ref, "bf16", f"request {r}"))
    del dw
    torch.cuda.empty_cache()


def test_host_feed_matches_device_resident_steps():
    """Bags fed from pinned host memory with the copy of batch i + 1 overlapping batch i
    (two device slots) give bit-identical scores to the device-resident steps."""
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, DeviceWorkload, HostFeed, pack_target_bags, pack_user_bags
    w = datagen.scaled(datagen.WORKLOADS["128d5l"], n_cand_per_request=500, rows=20000)
    sets = [datagen.make_requests(w, seed=900 + k) for k in range(3)]
    dw = DeviceWorkload(w, reqs=sets[0])
    ref = []
    for reqs in sets:
        dw.set_requests(reqs)
        dw.step()
        ref.append(dw.scores.clone())
    dw.set_requests(sets[0])

    def pinned(b):
        return DeviceBags(*(x.pin_memory() for x in (b.offsets, b.keys, b.weights, b.bag_table)))
    batches = [(pinned(DeviceBags.of(pack_user_bags(reqs), "cpu")), pinned(DeviceBags.of(pack_target_bags(reqs), "cpu")),
                reqs) for reqs in sets]
    feed = HostFeed(dw, batches)
    out = [torch.empty(dw.n_cand, dtype=torch.float32).pin_memory() for _ in range(7)]
    feed.run(0, 7, out)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(7):
        assert torch.equal(out[i], ref[i % 3].cpu()), i
    # the same through replayed graphs (one per device slot and host batch)
    feed.capture()
    for o in out:
        o.zero_()
    feed.run(0, 7, out)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(7):
        assert torch.equal(out[i], ref[i % 3].cpu()), ("graph", i)


def _serial_reference(w, sets):
    """Scores of each request set through DeviceWorkload.step, one after the other."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    dw = DeviceWorkload(w, reqs=sets[0])
    ref = []
    for reqs in sets:
        dw.set_requests(reqs)
        dw.step()
        ref.append(dw.scores.clone())
    torch.cuda.synchronize()
    dw.set_requests(sets[0])
    return dw, ref


@pytest.mark.parametrize("name,n_sms", [("128d5l", 6), ("128d5l", 148), ("64d3l", 6), ("tiny", 6)])
def test_overlapped_steps_match_serial_steps(name, n_sms):
    """Consecutive requests overlapped over two slots (compression and scoring split at
    their last partial wave, whose tail runs beside the next request's aggregation) give
    each request the scores of a serial step, bit for bit, eagerly and from one captured
    graph.  n_sms = 6 forces a split at this size (16 tiles = 8 units of two: 6 + 2); at 148
    there is a single round and no split.  The fp32 model runs every stage on the CUDA-core kernels,
    whose scratch is per stream: the user, main and tail streams run them concurrently."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload, Overlapped, score_split
    w = datagen.scaled(datagen.WORKLOADS[name], n_cand_per_request=2000, rows=20000)
    sets = [datagen.make_requests(w, seed=700 + k) for k in range(3)]
    dw, ref = _serial_reference(w, sets)
    dw2 = DeviceWorkload(w, reqs=sets[0], params=dw.params, tables=(dw.user_tables, dw.target_tables))
    ov = Overlapped([dw, dw2])
    ov.n_sms = n_sms
    assert (score_split(dw.req_offsets, n_sms) == 1536) == (n_sms == 6)
    n_batch = 7
    out = [torch.zeros(dw.n_cand, dtype=torch.float32, device="cuda") for _ in range(n_batch)]

    def bind(i, slot, main):
        slot.use_bags(*_set_bags(dw, sets, i))

    def scored(i, slot, back):
        with torch.cuda.stream(back):
            out[i].copy_(slot.scores)

    ov.run(0, n_batch, bind=bind, scored=scored)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(n_batch):
        assert torch.equal(out[i], ref[i % 3]), ("eager", i)
    for o in out:
        o.zero_()
    g = ov.capture(0, n_batch, bind=bind, scored=scored)
    if name == "128d5l":
        assert ov.launches_per_step == (7 if n_sms == 6 else 5)   # compress and score each in two parts
    for o in out:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(n_batch):
        assert torch.equal(out[i], ref[i % 3]), ("graph", i)


@pytest.mark.parametrize("name,n_cand,n_slots,comp_chunk,units", [
    ("128d5l", 2000, 3, 640, 3),         # launches of 5 tiles / 3 units, across batches and ring wraps
    ("128d5l", 40000, 4, None, None),    # the default launch sizes (launches every fourth batch: eight
                                         # compressor rounds, four score rounds) on a four-slot ring
    ("128d5l", 40000, None, None, None), # the configuration bench.py times (a 64-slot ring)
    ("packed", 300, 2, 1000, 5),         # 16 requests of mixed L_u per batch (one request set:
                                         # the slots' caches are sized by L_u); launches span many
    ("64d3l", 2000, 3, 768, 4),
    ("tiny", 500, 2, 256, 2),            # fp32: every stage on the CUDA-core kernels
])
def test_streamed_steps_match_serial_steps(name, n_cand, n_slots, comp_chunk, units):
    """Batches scored as one stream of candidate tiles (compress and score launches of fixed
    size across batch boundaries, over a ring of activation slots) give each batch the
    scores of a serial step, bit for bit, eagerly and from one captured graph."""
    from transformer_candidate_scoring_b200.pipeline import Streamed
    w = datagen.scaled(datagen.WORKLOADS[name], n_cand_per_request=n_cand, rows=20000)
    sets = [datagen.make_requests(w, seed=800 + k) for k in range(3)]
    dw, ref = _serial_reference(w, sets)
    one_set = name == "packed"
    if one_set:
        sets, ref = sets[:1], ref[:1]
    st = Streamed(dw, n_slots=n_slots, comp_chunk=comp_chunk, score_units=units)
    n_batch = 7
    out = [torch.zeros(dw.n_cand, dtype=torch.float32, device="cuda") for _ in range(n_batch)]

    def bind(i, slot, main):
        slot.use_bags(*_set_bags(dw, sets, i))

    def scored(i, slot, s):
        with torch.cuda.stream(s):
            out[i].copy_(slot.scores)

    st.run(0, n_batch, bind=bind, scored=scored)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(n_batch):
        bad = torch.nonzero(out[i] != ref[i % len(ref)]).flatten()
        if bad.numel():
            # which side is off: score the batch serially once more
            dw.use_bags(*_set_bags(dw, sets, i))
            dw.step()
            torch.cuda.synchronize()
            again = dw.scores.clone()
        assert bad.numel() == 0, ("eager", i, bad.numel(), sorted(set((bad // 128).tolist()))[:20],
                                  float((out[i] - ref[i % len(ref)]).abs().max()),
                                  "serial again == serial" if torch.equal(again, ref[i % len(ref)]) else
                                  "serial again == streamed" if torch.equal(again, out[i]) else "three ways")
    g = st.capture(0, n_batch, bind=bind, scored=scored)
    for o in out:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(n_batch):
        assert torch.equal(out[i], ref[i % len(ref)]), ("graph", i)


def test_full_request_scores_repeat_bit_identical():
    """A 40,000-candidate request: 148 two-tile units on every SM at once, then 17 single
    tiles on 17 of the same CTAs.  Scored 20 times (every other time after the gather and the
    compressor have cycled the caches), it gives the same bits each time, and the same bits
    as two launches that hold no single tile behind a pair (one round of 148 units, then the
    rest).  A CTA that moves from a pair to a single tile must not reload the K/V images
    while the pair's second tile still reads them."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    w = datagen.scaled(datagen.WORKLOADS["128d5l"], n_cand_per_request=40000, rows=20000)
    dw = DeviceWorkload(w)
    dw.step()
    dw.score_range(0, 37888)
    dw.score_range(37888, 40000)
    torch.cuda.synchronize()
    ref = dw.scores.clone()
    for k in range(20):
        if k % 2:
            dw.target_aggregate()
            dw.compress()
        dw.score()
        torch.cuda.synchronize()
        bad = torch.nonzero(dw.scores != ref).flatten()
        assert bad.numel() == 0, (k, sorted(set((bad // 128).tolist()))[:20])
    assert tr().sync_status() == 0


_SET_BAGS = {}


def _set_bags(dw, sets, i):
    """Device bags of request set i % len(sets) (uploaded once per set)."""
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, pack_target_bags, pack_user_bags
    reqs = sets[i % len(sets)]
    key = (id(dw), i % len(sets))
    if key not in _SET_BAGS or _SET_BAGS[key][2] is not reqs:      # (ids of freed objects recur)
        _SET_BAGS[key] = (DeviceBags.of(pack_user_bags(reqs), dw.device),
                          DeviceBags.of(pack_target_bags(reqs), dw.device), reqs)
    return _SET_BAGS[key]


def test_overlapped_packed_requests_split_inside_a_request():
    """Packed batches of 16 requests with different L_u: the score split falls inside a
    request (score_range gives each piece the request's cache), scores match serial steps."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload, Overlapped, score_split
    w = datagen.scaled(datagen.WORKLOADS["packed"], n_cand_per_request=300, rows=20000)
    sets = [datagen.make_requests(w, seed=800 + k) for k in range(2)]
    dw, ref = _serial_reference(w, sets)
    dw.set_requests(sets[0])
    dw2 = DeviceWorkload(w, reqs=sets[1], params=dw.params, tables=(dw.user_tables, dw.target_tables))
    ov = Overlapped([dw, dw2])
    ov.n_sms = 9                                   # 32 units -> 27 + 5, cut one unit into request 13
    cut = score_split(dw.req_offsets, ov.n_sms)
    assert cut is not None and cut not in dw.req_offsets
    out = [torch.zeros(dw.n_cand, dtype=torch.float32, device="cuda") for _ in range(5)]

    def scored(i, slot, back):
        with torch.cuda.stream(back):
            out[i].copy_(slot.scores)

    ov.run(0, 5, scored=scored)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(5):
        assert torch.equal(out[i], ref[i % 2]), i


def test_host_feed_overlapped_matches_serial_steps():
    """Host-fed batches through the overlapped slots (bags copied during the previous batch,
    scores copied back after the last score launch), eager and as one captured graph."""
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, DeviceWorkload, HostFeed, Overlapped, pack_target_bags, pack_user_bags
    w = datagen.scaled(datagen.WORKLOADS["128d5l"], n_cand_per_request=1000, rows=20000)
    sets = [datagen.make_requests(w, seed=950 + k) for k in range(3)]
    dw, ref = _serial_reference(w, sets)
    dw2 = DeviceWorkload(w, reqs=sets[0], params=dw.params, tables=(dw.user_tables, dw.target_tables))
    ov = Overlapped([dw, dw2])
    ov.n_sms = 3                                   # 4 units -> 3 + 1

    def pinned(b):
        return DeviceBags(*(x.pin_memory() for x in (b.offsets, b.keys, b.weights, b.bag_table)))
    batches = [(pinned(DeviceBags.of(pack_user_bags(reqs), "cpu")), pinned(DeviceBags.of(pack_target_bags(reqs), "cpu")),
                reqs) for reqs in sets]
    feed = HostFeed(dw, batches)
    out = [torch.empty(dw.n_cand, dtype=torch.float32).pin_memory() for _ in range(7)]
    feed.run_overlapped(ov, 0, 7, out)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(7):
        assert torch.equal(out[i], ref[i % 3].cpu()), ("eager", i)
    g = feed.capture_overlapped(ov, 0, 7, out)
    for o in out:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    for i in range(7):
        assert torch.equal(out[i], ref[i % 3].cpu()), ("graph", i)


def test_compress_corpus_chunked_equals_one_pass_and_oracle():
    """Near-line bulk compression in chunks (with a ragged last chunk) gives the same bits
    as one aggregate + compress pass over all items, and matches the oracle on a sample."""
    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, DeviceWorkload, compress_corpus
    w = datagen.scaled(datagen.WORKLOADS["128d5l"], n_cand_per_request=64, rows=20000)
    dw = DeviceWorkload(w)
    n_items = 5000
    bags = datagen.make_target_bags(np.random.default_rng(4), w, n_items)
    db = DeviceBags.of(bags, "cuda")
    F, D = w.dims.n_target_fields, w.dims.D
    out = torch.empty(n_items, D, dtype=torch.float32, device="cuda")
    compress_corpus(dw.model, dw.target_tables, db, n_items, F, out, chunk=1536)
    X = torch.empty(n_items, F * D, dtype=torch.bfloat16, device="cuda")
    api.aggregate(dw.target_tables, db.bag_table, db.offsets, db.keys, db.weights, X.view(-1, D))
    ref_gpu = torch.empty(n_items, D, dtype=torch.float32, device="cuda")
    api.compress_targets(dw.model, X, ref_gpu)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    assert torch.equal(out, ref_gpu)
    # oracle on a sample of items (including the last, ragged chunk)
    idx = np.array([0, 1, 1535, 1536, 3071, 4607, 4999])
    rows = []
    for i in idx:
        sub = datagen.Bags(bags.offsets[i * F:(i + 1) * F + 1] - bags.offsets[i * F],
                           bags.keys[bags.offsets[i * F]:bags.offsets[(i + 1) * F]],
                           bags.weights[bags.offsets[i * F]:bags.offsets[(i + 1) * F]], bags.bag_table[i * F:(i + 1) * F])
        toks = []
        for f in range(F):
            k = sub.keys[sub.offsets[f]:sub.offsets[f + 1]]
            r = datagen.table_rows_host(w.seed, datagen.target_table_id(w, int(sub.bag_table[f])), k, D, "bf16")
            toks.append(oracle.weighted_average(r, np.array([0, len(k)]), np.arange(len(k)),
                                                sub.weights[sub.offsets[f]:sub.offsets[f + 1]])[0])
        rows.append(np.concatenate(toks))
    ref = oracle.compress_targets(dw.params, np.stack(rows))
    check_close(out[torch.from_numpy(idx).cuda()].double().cpu().numpy(), ref, "bf16", "corpus sample",
                kind="intermediate")


def test_captured_step_replays_bit_identical():
    """A step captured into a CUDA graph and replayed gives the eager step's scores bit for
    bit (same kernels, same inputs)."""
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    w = datagen.scaled(datagen.WORKLOADS["packed"], n_cand_per_request=300, rows=20000)
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    ref = dw.scores.clone()
    g = dw.capture_step()
    dw.scores.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    assert torch.equal(dw.scores, ref)


@pytest.mark.parametrize("name,init,L_t,L_us,n_per", [
    ("tiny", "wide", 4, [8, 3], [37, 20]),
    ("tiny", "paper", 8, [8], [50]),
    ("64d3l", "wide", 8, [32, 0], [40, 9]),
    ("64d3l", "paper", 4, [32, 5], [70, 9]),
    ("128d5l", "wide", 8, [64], [60]),
    ("128d5l", "paper", 8, [64, 17], [60, 33]),     # two requests, ragged last tiles
    ("128d5l", "wide", 8, [0, 64], [20, 30]),       # a request without user keys
    ("128d5l", "wide", 2, [64], [100]),
    ("128d5l", "paper", 16, [32], [20]),
    ("128d5l", "wide", 16, [64, 40, 0], [9, 0, 5]),  # a request without candidates, one without users
    ("128d5l", "wide", 3, [64], [30]),              # not a power of two: CUDA-core kernels
])
def test_uncompressed_targets_parity(name, init, L_t, L_us, n_per):
    """Candidates of L_t target tokens (the variant target compression replaces) against the
    oracle, packed requests included.  bf16 models with L_t a power of two up to 16 run the
    tensor-core stack (own-candidate attention by warp shuffles), the rest the CUDA-core
    kernels."""
    dims, P, m, users, _, doms, kvs = _score_setup(name, init, L_us, n_per)
    std = 0.5 if init == "wide" else 0.3
    toks = [datagen.rand_matrix(300 + r, (n, L_t, dims.D), std, dims.dtype) for r, n in enumerate(n_per)]
    T = dev(np.concatenate(toks), tdt(dims.dtype))
    off = np.concatenate([[0], np.cumsum(n_per)]).tolist()
    s = torch.empty(off[-1], dtype=torch.float32, device="cuda")
    tr().api.score_candidates_uncompressed(m, T, L_t, off, kvs, L_us, doms, s)
    torch.cuda.synchronize()
    assert tr().sync_status() == 0
    got = s.cpu().numpy().astype(np.float64)
    for r, (U, t, d) in enumerate(zip(users, toks, doms)):
        if len(t) == 0:
            continue
        K, V = oracle.prefill_user(P, dims.n_head, U, d)
        ref = oracle.score_candidates_uncompressed(P, dims.n_head, t, K, V, d)
        check_close(got[off[r]:off[r + 1]], ref, dims.dtype, f"request {r}")


def test_uncompressed_with_one_token_equals_single_token_path_tensor_cores():
    """L_t = 1 on the bf16 model: the tensor-core variant with bf16 tokens equals
    tr_score_candidates on the same values in fp32 bit for bit (one own key, numerator sum 1,
    the mean value is the own value)."""
    dims, P, m, users, toks, doms, kvs = _score_setup("128d5l", "wide", [64, 20], [300, 45])
    a, off = _gpu_scores(m, dims, toks, kvs, [64, 20], doms)
    T = dev(np.concatenate(toks), torch.bfloat16)
    assert torch.equal(T.float().cpu(), torch.from_numpy(np.concatenate(toks)).float())
    s = torch.empty(int(off[-1]), dtype=torch.float32, device="cuda")
    tr().api.score_candidates_uncompressed(m, T, 1, off.tolist(), kvs, [64, 20], doms, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().astype(np.float64), a)


def test_uncompressed_with_one_token_equals_single_token_path_fp32():
    """L_t = 1 on the fp32 model runs the same CUDA-core code as tr_score_candidates: bit-equal."""
    dims, P, m, users, toks, doms, kvs = _score_setup("tiny", "wide", [8, 5], [40, 17])
    a, off = _gpu_scores(m, dims, toks, kvs, [8, 5], doms)
    T = dev(np.concatenate(toks), tdt(dims.dtype))
    s = torch.empty(int(off[-1]), dtype=torch.float32, device="cuda")
    tr().api.score_candidates_uncompressed(m, T, 1, off.tolist(), kvs, [8, 5], doms, s)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy().astype(np.float64), a)
