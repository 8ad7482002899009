"""Pins of the whole-request oracle (oracle/pipeline.py) against a brute force built here.

TransRetrieval §3.1 ("Architecture Overview") lists the stages of one request: (1) weighted-
average aggregation of every user field and every target field, (2) target compression of
the concatenated target-field tokens into one token (§3.3), (3) the domain embedding added
to every token (§3.4), (4) the N-layer Transformer, then the score head.  The brute force
below restates those stages with nothing from the oracle:

* every weighted average is a plain-Python loop over the bag's (key, weight) pairs, each
  row read from the data generator's table by the field -> table reading (user field f reads
  user table f mod T_u, target field f reads target table f mod T_t);
* the compressor input is the field tokens concatenated in field order, the compressor a
  ``torch.nn.Sequential(Linear, PReLU, LayerNorm, Linear, PReLU, LayerNorm, Linear)``;
* the score is the full-sequence forward of [user tokens..., candidate] through PyTorch's
  ``TransformerEncoderLayer`` stack with the candidate masked from the users.

A mistake planted in the oracle on the CPU (a wrong field -> table map, a permuted
concatenation order, an off-by-one candidate selection) must fail these comparisons.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
import oracle.pipeline as OP
from test_oracle_pins import _lin, _ln, _torch_full_sequence_scores


def _workloads():
    """A single-request fp32 workload (the tiny model) and a three-request one with mixed
    L_u, three target tables for four fields (field 3 wraps to table 0), two layers."""
    tiny = datagen.scaled(datagen.WORKLOADS["tiny"], n_cand_per_request=12, seed=5)
    dims = datagen.ModelDims(D=32, n_layer=2, n_head=2, ffn_hidden=64, n_target_fields=4,
                             comp_dims=(128, 64, 32, 32), n_domains=3, dtype="f32")
    packed = datagen.Workload("packed_small", dims, n_requests=3, L_u=(2, 9), user_nf=(1, 6), user_tables=3,
                              user_rows=400, target_nf=(1, 4), target_rows=(500, 700, 900),
                              n_cand_per_request=7, seed=9)
    return {"tiny": tiny, "packed_small": packed}


def _row_lookup(w, table_id, keys):
    keys = np.asarray(sorted(set(int(k) for k in keys)), dtype=np.int64)
    rows = datagen.table_rows_host(w.seed, table_id, keys, w.dims.D, w.dims.dtype) if len(keys) else []
    return {int(k): np.asarray(r, np.float64) for k, r in zip(keys, rows)}


def _brute_wavg(offsets, keys, weights, bag, lookup, D):
    num = np.zeros(D)
    den = 0.0
    for i in range(int(offsets[bag]), int(offsets[bag + 1])):
        v = float(weights[i])
        num = num + v * lookup[int(keys[i])]
        den += v
    return num / den if den != 0.0 else np.zeros(D)


def _brute_user_tokens(w, req):
    D, T_u = w.dims.D, w.user_tables
    b = req.user
    out = np.zeros((req.L_u, D))
    for f in range(req.L_u):
        t = f % T_u
        lookup = _row_lookup(w, t, b.keys[b.offsets[f]:b.offsets[f + 1]])
        out[f] = _brute_wavg(b.offsets, b.keys, b.weights, f, lookup, D)
    return out


def _brute_concat(w, req, cand):
    D, F, T_t = w.dims.D, w.dims.n_target_fields, len(w.target_rows)
    b = req.target
    X = np.zeros((len(cand), F * D))
    for i, c in enumerate(cand):
        for f in range(F):
            bag = int(c) * F + f
            table_id = w.user_tables + f % T_t     # target tables follow the user tables
            lookup = _row_lookup(w, table_id, b.keys[b.offsets[bag]:b.offsets[bag + 1]])
            X[i, f * D:(f + 1) * D] = _brute_wavg(b.offsets, b.keys, b.weights, bag, lookup, D)
    return X


def _torch_compressor(P, c):
    mods = []
    for i in range(3):
        mods.append(_lin(P[f"c{i}.W"], P[f"c{i}.b"]))
        if i < 2:
            pr = torch.nn.PReLU(c[i + 1], dtype=torch.float64)
            with torch.no_grad():
                pr.weight.copy_(torch.from_numpy(np.asarray(P[f"c{i}.prelu"], np.float64)))
            mods += [pr, _ln(P[f"c{i}.ln_g"], P[f"c{i}.ln_b"])]
    return torch.nn.Sequential(*mods)


def _brute_request(w, P, req, cand):
    user = _brute_user_tokens(w, req)
    X = _brute_concat(w, req, cand)
    with torch.no_grad():
        tokens = _torch_compressor(P, w.dims.comp_dims)(torch.from_numpy(X)).numpy()
    scores = _torch_full_sequence_scores(P, w.dims, user, tokens, req.domain)
    return user, X, tokens, scores


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return a.shape == b.shape and float(np.max(np.abs(a - b), initial=0.0)) <= tol * max(1.0, float(np.max(np.abs(b), initial=0.0)))


def _agrees(w, P, req, cand=None):
    cand_idx = np.arange(req.n_cand) if cand is None else np.asarray(cand)
    got = oracle.score_request(w, P, req, cand=cand)
    user, X, tokens, scores = _brute_request(w, P, req, cand_idx)
    return (_close(got.user_tokens, user) and _close(got.X, X) and _close(got.tokens, tokens)
            and _close(got.scores, scores))


@pytest.mark.parametrize("name", ["tiny", "packed_small"])
def test_score_request_equals_brute_force(name):
    w = _workloads()[name]
    P = datagen.make_params(w.dims, w.seed, "wide")
    reqs = datagen.make_requests(w)
    assert len(reqs) == w.n_requests and (w.n_requests == 1 or len({r.L_u for r in reqs}) > 1)
    for req in reqs:
        got = oracle.score_request(w, P, req)
        user, X, tokens, scores = _brute_request(w, P, req, np.arange(req.n_cand))
        np.testing.assert_allclose(got.user_tokens, user, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got.X, X, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got.tokens, tokens, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(got.scores, scores, rtol=1e-10, atol=1e-10)


def test_candidate_subset_equals_rows_of_the_full_request():
    w = _workloads()["packed_small"]
    P = datagen.make_params(w.dims, w.seed, "wide")
    for req in datagen.make_requests(w):
        full = oracle.score_request(w, P, req)
        for cand in (np.array([0]), np.array([req.n_cand - 1]), np.arange(1, req.n_cand, 2), np.array([4, 1, 6])):
            sub = oracle.score_request(w, P, req, cand=cand)
            np.testing.assert_array_equal(sub.X, full.X[cand])
            np.testing.assert_allclose(sub.scores, full.scores[cand], rtol=0, atol=1e-13)
        assert _agrees(w, P, req, cand=np.array([4, 1, 6]))


def test_planted_field_to_table_map_fails(monkeypatch):
    w = _workloads()["packed_small"]
    P = datagen.make_params(w.dims, w.seed, "wide")
    req = datagen.make_requests(w)[0]
    assert _agrees(w, P, req)
    monkeypatch.setattr(datagen, "target_table_id", lambda w_, t: w_.user_tables + (t + 1) % len(w_.target_rows))
    assert not _agrees(w, P, req)


def test_planted_concatenation_order_fails(monkeypatch):
    w = _workloads()["tiny"]
    P = datagen.make_params(w.dims, w.seed, "wide")
    req = datagen.make_requests(w)[0]
    assert _agrees(w, P, req)
    real = OP._select_candidates

    def swapped(req_, cand, F):
        b = real(req_, cand, F)
        # fields 0 and 1 of every candidate exchange places in the compressor input
        n = len(b.offsets) - 1
        order = np.arange(n).reshape(-1, F)
        order[:, [0, 1]] = order[:, [1, 0]]
        order = order.reshape(-1)
        counts = np.diff(b.offsets)[order]
        off = np.zeros(n + 1, np.int64)
        np.cumsum(counts, out=off[1:])
        idx = np.concatenate([np.arange(b.offsets[i], b.offsets[i + 1]) for i in order]).astype(np.int64)
        return datagen.Bags(off, b.keys[idx], b.weights[idx], b.bag_table[order])
    monkeypatch.setattr(OP, "_select_candidates", swapped)
    assert not _agrees(w, P, req)


def test_planted_off_by_one_selection_fails(monkeypatch):
    w = _workloads()["packed_small"]
    P = datagen.make_params(w.dims, w.seed, "wide")
    req = datagen.make_requests(w)[1]
    cand = np.array([0, 3, 5])
    assert _agrees(w, P, req, cand=cand)
    real = OP._select_candidates
    monkeypatch.setattr(OP, "_select_candidates",
                        lambda req_, c, F: real(req_, np.minimum(np.asarray(c) + 1, req_.n_cand - 1), F))
    assert not _agrees(w, P, req, cand=cand)
