"""Pins of the fp64 oracle against things other than itself.

* Aggregation (TransRetrieval §3.2): the properties the paper states for the weighted
  average -- division by the weight sum cancels weight magnitudes (scale invariance) and
  bounds the output by the table's values (convex combination for v >= 0) -- plus the
  special cases that reduce to a plain mean or to one row, and the algebraic relation to
  the weighted sum it replaces.
* LayerNorm, the compressor (§3.3) and every Transformer layer (§3.1 stage (4)) are
  compared with PyTorch's own fp64 modules (LayerNorm, PReLU, Linear,
  TransformerEncoderLayer with norm_first=True and ReLU), which share no code with the
  oracle.
* The KV-cached candidate score (§3.3, deployment "Hardware-aware inference
  optimization") equals a brute-force full-sequence forward [user tokens..., candidate]
  with a mask that hides the candidate from the user tokens.
* The FLOP count meets the closed form 16*L_t*D^2 + 4*L_t*L_u*D per layer (§3.3).
"""
import json
import os

import numpy as np
import pytest
import torch

import datagen
import oracle
from oracle import transretrieval as T

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _rand_bags(rng, n_bags, max_nf, n_rows, allow_empty=False):
    lo = 0 if allow_empty else 1
    counts = rng.integers(lo, max_nf + 1, size=n_bags)
    off = np.zeros(n_bags + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    keys = rng.integers(0, n_rows, size=int(off[-1]))
    w = rng.uniform(0.1, 1.0, size=int(off[-1]))
    return off, keys, w


# ------------------------------------------------------------------ aggregation

def test_wavg_single_key_returns_its_row():
    rng = _rng(1)
    rows = rng.normal(size=(50, 16))
    keys = rng.integers(0, 50, size=20)
    off = np.arange(21)
    w = 2.0 ** rng.integers(-4, 4, size=20)          # exact in binary: v*h/v == h
    out = T.weighted_average(rows, off, keys, w)
    assert np.array_equal(out, rows[keys])
    w2 = rng.uniform(0.1, 1.0, size=20)
    np.testing.assert_allclose(T.weighted_average(rows, off, keys, w2), rows[keys], rtol=1e-15, atol=0)


@pytest.mark.parametrize("c", [3.7, 1e-3, 1e3, 0.25, 8.0])
def test_wavg_scale_invariance(c):
    rng = _rng(2)
    rows = rng.normal(size=(100, 8))
    off, keys, w = _rand_bags(rng, 30, 12, 100)
    a = T.weighted_average(rows, off, keys, w)
    b = T.weighted_average(rows, off, keys, w * c)
    if np.log2(c) == int(np.log2(c)):
        assert np.array_equal(a, b)
    else:
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_wavg_is_a_convex_combination():
    rng = _rng(3)
    rows = rng.normal(size=(200, 8)) * rng.uniform(0.1, 10, size=(200, 1))
    off, keys, w = _rand_bags(rng, 60, 40, 200)
    out = T.weighted_average(rows, off, keys, w)
    for b in range(60):
        r = rows[keys[off[b]:off[b + 1]]]
        assert np.all(out[b] >= r.min(0) - 1e-12) and np.all(out[b] <= r.max(0) + 1e-12)
        assert np.linalg.norm(out[b]) <= np.linalg.norm(r, axis=1).max() + 1e-12
    # the norm does not grow with cardinality, unlike the weighted sum (§3.2 profiling)
    big = np.zeros(2, dtype=np.int64)
    big[1] = 5000
    k = rng.integers(0, 200, size=5000)
    v = rng.uniform(0.1, 1, size=5000)
    assert np.linalg.norm(T.weighted_average(rows, big, k, v)) <= np.abs(rows).max() * np.sqrt(8)
    assert np.linalg.norm(T.weighted_sum(rows, big, k, v)) > 10 * np.linalg.norm(T.weighted_average(rows, big, k, v))


def test_wavg_equal_weights_is_the_plain_mean():
    rng = _rng(4)
    rows = rng.normal(size=(64, 12))
    off, keys, _ = _rand_bags(rng, 25, 9, 64)
    out = T.weighted_average(rows, off, keys, np.full(len(keys), 0.37))
    ref = np.stack([rows[keys[off[b]:off[b + 1]]].mean(0) for b in range(25)])
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_wavg_times_weight_sum_is_the_weighted_sum():
    rng = _rng(5)
    rows = rng.normal(size=(64, 12))
    off, keys, w = _rand_bags(rng, 25, 9, 64)
    den = np.add.reduceat(w, off[:-1])
    np.testing.assert_allclose(T.weighted_average(rows, off, keys, w) * den[:, None],
                               T.weighted_sum(rows, off, keys, w), rtol=1e-12, atol=1e-14)


def test_wavg_edge_cases():
    rows = np.arange(12, dtype=np.float64).reshape(4, 3) + 1.0
    # empty bag, zero-sum weights, duplicate keys, negative weight
    off = np.array([0, 0, 2, 4, 6])
    keys = np.array([1, 2, 3, 3, 0, 1])
    w = np.array([1.0, -1.0, 0.3, 0.7, 2.0, -1.0])
    out = T.weighted_average(rows, off, keys, w)
    assert np.array_equal(out[0], np.zeros(3))
    assert np.array_equal(out[1], np.zeros(3))
    np.testing.assert_allclose(out[2], rows[3], rtol=1e-15)
    np.testing.assert_allclose(out[3], 2 * rows[0] - rows[1], rtol=1e-15)


def test_wavg_brute_force_tiny():
    rng = _rng(6)
    rows = rng.normal(size=(10, 4))
    off, keys, w = _rand_bags(rng, 7, 5, 10, allow_empty=True)
    out = T.weighted_average(rows, off, keys, w)
    for b in range(7):
        num = [0.0] * 4
        den = 0.0
        for i in range(off[b], off[b + 1]):
            den += w[i]
            for d in range(4):
                num[d] += w[i] * rows[keys[i], d]
        want = [x / den for x in num] if den else [0.0] * 4
        np.testing.assert_allclose(out[b], want, rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------------ torch modules

def _lin(W, b):
    m = torch.nn.Linear(W.shape[0], W.shape[1], dtype=torch.float64)
    with torch.no_grad():
        m.weight.copy_(torch.from_numpy(np.asarray(W, np.float64).T))
        m.bias.copy_(torch.from_numpy(np.asarray(b, np.float64)))
    return m


def _ln(g, b):
    m = torch.nn.LayerNorm(len(g), eps=1e-5, dtype=torch.float64)
    with torch.no_grad():
        m.weight.copy_(torch.from_numpy(np.asarray(g, np.float64)))
        m.bias.copy_(torch.from_numpy(np.asarray(b, np.float64)))
    return m


def torch_layer(P, l, D, H):
    L = torch.nn.TransformerEncoderLayer(D, H, dim_feedforward=2 * D, dropout=0.0, activation="relu",
                                         layer_norm_eps=1e-5, batch_first=True, norm_first=True,
                                         dtype=torch.float64)
    f = lambda k: torch.from_numpy(np.asarray(P[f"l{l}.{k}"], np.float64))
    with torch.no_grad():
        L.self_attn.in_proj_weight.copy_(torch.cat([f("Wq").T, f("Wk").T, f("Wv").T]))
        L.self_attn.in_proj_bias.copy_(torch.cat([f("bq"), f("bk"), f("bv")]))
        L.self_attn.out_proj.weight.copy_(f("Wo").T)
        L.self_attn.out_proj.bias.copy_(f("bo"))
        L.linear1.weight.copy_(f("W1").T)
        L.linear1.bias.copy_(f("b1"))
        L.linear2.weight.copy_(f("W2").T)
        L.linear2.bias.copy_(f("b2"))
        L.norm1.weight.copy_(f("ln1_g"))
        L.norm1.bias.copy_(f("ln1_b"))
        L.norm2.weight.copy_(f("ln2_g"))
        L.norm2.bias.copy_(f("ln2_b"))
    return L.eval()


def _dims(D=32, N=2, H=4, dtype="f32"):
    return datagen.ModelDims(D=D, n_layer=N, n_head=H, ffn_hidden=2 * D, n_target_fields=4,
                             comp_dims=(4 * D, 2 * D, D, D), n_domains=3, dtype=dtype)


def _wide_params(dims, seed=0):
    """Parameters with larger weights than the N(0, 0.02) init, so that attention is far
    from uniform and every term of the layer matters in the comparison."""
    P = datagen.make_params(dims, seed)
    rng = _rng(seed + 100)
    out = {}
    for k, v in P.items():
        if k.endswith((".Wq", ".Wk", ".Wv", ".Wo", ".W1", ".W2", ".W")):
            out[k] = rng.normal(0, 1.0 / np.sqrt(v.shape[0]), size=v.shape)
        elif k.endswith(("_g",)):
            out[k] = rng.uniform(0.5, 1.5, size=v.shape)
        elif k.endswith("prelu"):
            out[k] = rng.uniform(-0.5, 0.5, size=v.shape)
        else:
            out[k] = rng.normal(0, 0.3, size=v.shape)
    return out


def test_layer_norm_matches_torch():
    rng = _rng(7)
    x = rng.normal(size=(9, 40)) * 3 + 1
    g, b = rng.normal(size=40), rng.normal(size=40)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (40,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-5).numpy()
    np.testing.assert_allclose(T.layer_norm(x, g, b), ref, rtol=1e-12, atol=1e-12)


def test_compressor_matches_torch_mlp():
    dims = _dims()
    P = _wide_params(dims, 1)
    c = dims.comp_dims
    mods = []
    for i in range(3):
        mods.append(_lin(P[f"c{i}.W"], P[f"c{i}.b"]))
        if i < 2:
            pr = torch.nn.PReLU(c[i + 1], dtype=torch.float64)
            with torch.no_grad():
                pr.weight.copy_(torch.from_numpy(np.asarray(P[f"c{i}.prelu"], np.float64)))
            mods += [pr, _ln(P[f"c{i}.ln_g"], P[f"c{i}.ln_b"])]
    mlp = torch.nn.Sequential(*mods)
    X = _rng(8).normal(size=(33, c[0]))
    with torch.no_grad():
        ref = mlp(torch.from_numpy(X)).numpy()
    np.testing.assert_allclose(T.compress_targets(P, X), ref, rtol=1e-10, atol=1e-12)


def _torch_full_sequence_scores(P, dims, user_tokens, tokens, domain):
    """Brute force: every candidate runs as the last token of [users..., candidate]
    through PyTorch's encoder layers; user positions may not attend to the candidate."""
    D, H, N = dims.D, dims.n_head, dims.n_layer
    s = np.asarray(P["domain_emb"], np.float64)[domain]
    n, L_u = len(tokens), len(user_tokens)
    seq = np.concatenate([np.broadcast_to(user_tokens + s, (n, L_u, D)), (tokens + s)[:, None, :]], axis=1)
    x = torch.from_numpy(np.ascontiguousarray(seq))
    mask = torch.zeros(L_u + 1, L_u + 1, dtype=torch.bool)
    mask[:L_u, L_u] = True
    with torch.no_grad():
        for l in range(N):
            x = torch_layer(P, l, D, H)(x, src_mask=mask)
        z = _ln(P["lnf_g"], P["lnf_b"])(x[:, -1])
        return (z @ torch.from_numpy(np.asarray(P["w_head"], np.float64)) + float(P["b_head"][0])).numpy()


@pytest.mark.parametrize("L_u", [0, 1, 7, 20])
def test_cached_scores_equal_masked_full_sequence(L_u):
    dims = _dims(D=32, N=3, H=4)
    P = _wide_params(dims, 2)
    rng = _rng(9)
    U = rng.normal(size=(L_u, 32))
    t = rng.normal(size=(11, 32))
    K, V = T.prefill_user(P, dims.n_head, U, 1)
    got = T.score_candidates(P, dims.n_head, t, K, V, 1)
    ref = _torch_full_sequence_scores(P, dims, U, t, 1)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-11)


def test_prefill_kv_match_torch_layers():
    dims = _dims(D=32, N=3, H=2)
    P = _wide_params(dims, 3)
    U = _rng(10).normal(size=(13, 32))
    K, V = T.prefill_user(P, dims.n_head, U, 2)
    x = torch.from_numpy(U + np.asarray(P["domain_emb"], np.float64)[2])[None]
    with torch.no_grad():
        for l in range(3):
            L = torch_layer(P, l, 32, 2)
            kv = torch.nn.functional.linear(L.norm1(x), L.self_attn.in_proj_weight[32:],
                                            L.self_attn.in_proj_bias[32:])[0].numpy()
            np.testing.assert_allclose(K[l], kv[:, :32], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(V[l], kv[:, 32:], rtol=1e-11, atol=1e-12)
            x = L(x)


# ------------------------------------------------------------------ stated invariants

def _setup(seed=11, L_u=9, n=17):
    dims = _dims(D=32, N=2, H=4)
    P = _wide_params(dims, seed)
    rng = _rng(seed)
    return dims, P, rng.normal(size=(L_u, 32)), rng.normal(size=(n, 32))


def test_scores_independent_of_batch_mates():
    dims, P, U, t = _setup()
    K, V = T.prefill_user(P, 4, U, 0)
    full = T.score_candidates(P, 4, t, K, V, 0)
    for idx in ([3], [0, 5, 16], list(range(16, -1, -2))):
        np.testing.assert_allclose(T.score_candidates(P, 4, t[idx], K, V, 0), full[idx], rtol=1e-13, atol=1e-14)


def test_scores_invariant_to_user_field_order():
    dims, P, U, t = _setup(12)
    perm = _rng(13).permutation(len(U))
    a = T.score_candidates(P, 4, t, *T.prefill_user(P, 4, U, 0), 0)
    b = T.score_candidates(P, 4, t, *T.prefill_user(P, 4, U[perm], 0), 0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_zero_query_gives_uniform_attention():
    """With W_q = 0 and b_q = 0 every score is 0, so keys stop mattering."""
    dims, P, U, t = _setup(14)
    for l in range(2):
        P[f"l{l}.Wq"] = np.zeros_like(P[f"l{l}.Wq"])
        P[f"l{l}.bq"] = np.zeros_like(P[f"l{l}.bq"])
    K, V = T.prefill_user(P, 4, U, 0)
    a = T.score_candidates(P, 4, t, K, V, 0)
    b = T.score_candidates(P, 4, t, _rng(15).normal(size=K.shape), V, 0)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    c = T.score_candidates(P, 4, t, K, V * 0.5, 0)
    assert np.max(np.abs(a - c)) > 1e-6


def test_domain_embedding_is_an_elementwise_add():
    dims, P, U, t = _setup(16)
    d = 2
    s = np.asarray(P["domain_emb"][d], np.float64)
    a = T.score_candidates(P, 4, t, *T.prefill_user(P, 4, U, d), d)
    P0 = dict(P)
    P0["domain_emb"] = np.zeros_like(P["domain_emb"])
    b = T.score_candidates(P0, 4, t + s, *T.prefill_user(P0, 4, U + s, d), d)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_user_only_request_reduces_to_candidate_alone():
    """L_u = 0: a candidate attends only to itself; equals a one-token sequence."""
    dims, P, _, t = _setup(17, L_u=0)
    K, V = T.prefill_user(P, 4, np.zeros((0, 32)), 1)
    got = T.score_candidates(P, 4, t, K, V, 1)
    ref = _torch_full_sequence_scores(P, dims, np.zeros((0, 32)), t, 1)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-11)


# ------------------------------------------------------------------ FLOPs (§3.3)

@pytest.mark.parametrize("D,N,L_u", [(32, 1, 8), (64, 3, 32), (128, 5, 64), (128, 5, 127)])
def test_flop_counter_meets_closed_form(D, N, L_u):
    dims = _dims(D=D, N=N, H=D // 16)
    P = datagen.make_params(dims, 0)
    rng = _rng(18)
    K = rng.normal(size=(N, L_u, D))
    V = rng.normal(size=(N, L_u, D))
    with T.FlopCounter() as fc:
        T.score_candidates(P, dims.n_head, rng.normal(size=(3, D)), K, V, 0)
    assert fc.flops == 3 * T.flops_per_candidate_closed_form(D, N, L_u)
    # the paper's count (no self term, no head) is the dominant part
    paper = T.flops_per_candidate_closed_form(D, N, L_u, self_term=False, head=False)
    assert fc.flops / 3 - paper == N * 4 * D + 2 * D


def test_flop_formula_golden_values():
    """Per-candidate FLOPs of the paper's formula for the two published backbones."""
    with open(os.path.join(GOLDEN, "flops_per_candidate.json")) as f:
        g = json.load(f)
    for row in g["rows"]:
        assert T.flops_per_candidate_closed_form(row["D"], row["n_layer"], row["L_u"], L_t=row["L_t"],
                                                 self_term=False, head=False) == row["paper_formula"]
        with T.FlopCounter() as fc:
            dims = _dims(D=row["D"], N=row["n_layer"], H=row["D"] // 16)
            P = datagen.make_params(dims, 0)
            rng = _rng(19)
            T.score_candidates(P, dims.n_head, rng.normal(size=(1, row["D"])),
                               rng.normal(size=(row["n_layer"], row["L_u"], row["D"])),
                               rng.normal(size=(row["n_layer"], row["L_u"], row["D"])), 0)
        if row["L_t"] == 1:
            assert fc.flops == row["with_self_and_head"]


def test_compressor_flops():
    dims = _dims(D=128)
    P = datagen.make_params(datagen.configs.DIMS_128D5L, 0)
    with T.FlopCounter() as fc:
        T.compress_targets(P, np.zeros((2, 1024)))
    assert fc.flops == 2 * 2 * (1024 * 512 + 512 * 256 + 256 * 128)


def test_topk_order_and_ties():
    s = np.array([0.5, 0.9, 0.5, -1.0, 0.9, 0.1])
    assert T.topk(s, 4).tolist() == [1, 4, 0, 2]


# ---------------------------------------------------------------- aggregator variants (§3.2)

def test_max_pool_pins():
    rng = np.random.default_rng(21)
    rows = rng.standard_normal((50, 6))
    off = np.array([0, 1, 4, 4, 9])
    keys = rng.integers(0, 50, 9)
    got = T.max_pool(rows, off, keys)
    # single-key bag returns its row; empty bag zeros; element-wise maximum by plain loops
    assert np.array_equal(got[0], rows[keys[0]])
    assert np.array_equal(got[2], np.zeros(6))
    for b, (s, e) in enumerate(zip(off[:-1], off[1:])):
        if e == s:
            continue
        for d in range(6):
            m = -np.inf
            for i in range(s, e):
                m = max(m, rows[keys[i], d])
            assert got[b, d] == m
    # permutation of a bag's keys does not matter; duplicating a key does not either
    perm = keys.copy()
    perm[1:4] = perm[1:4][::-1]
    assert np.array_equal(T.max_pool(rows, off, perm), got)
    # the extreme-value bias §3.2 names: the maximum is >= the weighted average (positive weights)
    w = rng.uniform(0.1, 1, 9)
    avg = T.weighted_average(rows, off, keys, w)
    ne = np.diff(off) > 0
    assert np.all(got[ne] >= avg[ne] - 1e-12)


def test_aggregate_modes_and_post_layernorm():
    import torch
    rng = np.random.default_rng(22)
    rows = rng.standard_normal((40, 8))
    off = np.array([0, 3, 7, 12])
    keys = rng.integers(0, 40, 12)
    w = rng.uniform(0.1, 1, 12)
    assert np.array_equal(T.aggregate(rows, off, keys, w, "mean"), T.weighted_average(rows, off, keys, w))
    assert np.array_equal(T.aggregate(rows, off, keys, w, "sum"), T.weighted_sum(rows, off, keys, w))
    assert np.array_equal(T.aggregate(rows, off, keys, w, "max"), T.max_pool(rows, off, keys))
    for mode in ("mean", "sum", "max"):
        base = T.aggregate(rows, off, keys, w, mode)
        ln = T.aggregate(rows, off, keys, w, mode, post_ln=True)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(base), (8,), eps=T.EPS).numpy()
        np.testing.assert_allclose(ln, ref, rtol=1e-12, atol=1e-12)
    # LayerNorm erases the per-field magnitude: scaling all weights of the weighted sum leaves
    # the normalised token unchanged up to the eps inside the square root
    s1 = T.aggregate(rows, off, keys, w, "sum", post_ln=True)
    s2 = T.aggregate(rows, off, keys, 7.0 * w, "sum", post_ln=True)
    np.testing.assert_allclose(s1, s2, rtol=0, atol=1e-4)
    assert np.abs(s1 - s2).max() > 0
    try:
        T.aggregate(rows, off, keys, w, "median")
        assert False
    except ValueError:
        pass


# ---------------------------------------------------------------- uncompressed targets (§3.3)

def _torch_full_sequence_scores_multi(P, dims, user_tokens, tokens, domain):
    """Brute force for candidates of L_t tokens: each candidate's tokens run as the tail of
    [users..., candidate tokens] through PyTorch's encoder layers, users masked from the
    candidate's tokens; score = mean over the candidate's tokens of the head."""
    D, H, N = dims.D, dims.n_head, dims.n_layer
    s = np.asarray(P["domain_emb"], np.float64)[domain]
    n, L_t, _ = tokens.shape
    L_u = len(user_tokens)
    seq = np.concatenate([np.broadcast_to(user_tokens + s, (n, L_u, D)), tokens + s], axis=1)
    x = torch.from_numpy(np.ascontiguousarray(seq))
    mask = torch.zeros(L_u + L_t, L_u + L_t, dtype=torch.bool)
    mask[:L_u, L_u:] = True
    with torch.no_grad():
        for l in range(N):
            x = torch_layer(P, l, D, H)(x, src_mask=mask)
        z = _ln(P["lnf_g"], P["lnf_b"])(x[:, L_u:])
    per = (z.numpy() @ np.asarray(P["w_head"], np.float64)) + float(np.asarray(P["b_head"]))
    return per.mean(axis=1)


@pytest.mark.parametrize("L_t", [1, 3, 8])
def test_uncompressed_scores_equal_full_sequence_forward(L_t):
    dims = _dims(D=32, N=2, H=2)
    P = _wide_params(dims, 5)
    rng = _rng(40 + L_t)
    users = rng.normal(size=(6, dims.D))
    K, V = T.prefill_user(P, dims.n_head, users, 1)
    toks = rng.normal(size=(5, L_t, dims.D))
    got = T.score_candidates_uncompressed(P, dims.n_head, toks, K, V, 1)
    ref = _torch_full_sequence_scores_multi(P, dims, users, toks, 1)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-10)


def test_uncompressed_reduces_to_single_token_and_is_permutation_invariant():
    dims = _dims(D=32, N=2, H=2)
    P = _wide_params(dims, 6)
    rng = _rng(50)
    users = rng.normal(size=(7, dims.D))
    K, V = T.prefill_user(P, dims.n_head, users, 0)
    one = rng.normal(size=(9, dims.D))
    np.testing.assert_allclose(T.score_candidates_uncompressed(P, dims.n_head, one[:, None, :], K, V, 0),
                               T.score_candidates(P, dims.n_head, one, K, V, 0), rtol=1e-12, atol=1e-12)
    toks = rng.normal(size=(4, 5, dims.D))
    a = T.score_candidates_uncompressed(P, dims.n_head, toks, K, V, 0)
    b = T.score_candidates_uncompressed(P, dims.n_head, toks[:, ::-1], K, V, 0)   # own tokens reversed
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    c = T.score_candidates_uncompressed(P, dims.n_head, toks[[2]], K, V, 0)        # batch-mates do not matter
    np.testing.assert_allclose(c, a[[2]], rtol=1e-12, atol=1e-12)


def test_uncompressed_flops_and_the_compression_saving():
    """Instrumented FLOPs of the L_t-token stack = N (16 L_t D^2 + 4 L_t (L_u + L_t) D) + 2 D L_t,
    and at the 128D-5L backbone (L_t = 8 fields, L_u = 64) compression to one token saves
    about 85 % of the per-candidate FLOPs (§3.3 and the summary's claim)."""
    D, N, L_u, L_t = 32, 2, 8, 4
    dims = _dims(D=D, N=N, H=2)
    P = datagen.make_params(dims, 0)
    rng = _rng(60)
    K = rng.normal(size=(N, L_u, D))
    V = rng.normal(size=(N, L_u, D))
    with T.FlopCounter() as fc:
        T.score_candidates_uncompressed(P, dims.n_head, rng.normal(size=(3, L_t, D)), K, V, 0)
    assert fc.flops == 3 * (N * (16 * L_t * D * D + 4 * L_t * (L_u + L_t) * D) + 2 * D * L_t)
    full = T.flops_per_candidate_closed_form(128, 5, 64, L_t=8, self_term=False, head=False)
    comp = T.flops_per_candidate_closed_form(128, 5, 64, L_t=1, self_term=False, head=False)
    assert 0.85 <= 1 - comp / full <= 0.90
