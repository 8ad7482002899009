"""fp64 CPU oracle of TransRetrieval candidate scoring.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the
tests, the smoke check and the bench's CPU-baseline / reference leg call it.  It is a
plain, slow restatement of what the method computes, written from the TransRetrieval
paper ("TransRetrieval: Scaling Up Transformer-Based Retrieval for Industrial
Recommendation"), in float64 throughout.  Library primitives (a matrix product, a
segmented sum) serve as single steps; there is no caching beyond what the paper itself
describes, no blocking and no fusion.

Readings of points the paper leaves open (each also listed in the design notes):
* weighted average of an empty bag, or of a bag whose weights sum to 0, is the zero
  vector; duplicate keys count once per occurrence;
* compressor order inside a hidden layer: Linear -> PReLU (one slope per channel) ->
  LayerNorm; the last layer is a plain Linear; LayerNorm eps = 1e-5 with affine gain/shift;
* attention: standard multi-head attention with biases on every projection, scale
  1/sqrt(d_h); user tokens attend to every user token; a candidate attends to every
  user token of its request and to itself;
* the domain embedding s_d is added to every user token before the first layer and to
  the compressed candidate token before the first layer;
* score head: final LayerNorm, then a linear map D -> 1 with bias; the raw value is the score.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-5


class FlopCounter:
    """Counts 2*m*k*n for every contraction the oracle performs while active."""
    active = None

    def __init__(self):
        self.flops = 0

    def __enter__(self):
        FlopCounter.active = self
        return self

    def __exit__(self, *a):
        FlopCounter.active = None


def _mm(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    if FlopCounter.active is not None:
        FlopCounter.active.flops += 2 * int(np.prod(a.shape[:-1])) * a.shape[-1] * b.shape[-1]
    return a @ b


def _count(n: int) -> None:
    if FlopCounter.active is not None:
        FlopCounter.active.flops += int(n)


# ------------------------------------------------------------------ §3.2 aggregation

def weighted_average(rows: np.ndarray, offsets: np.ndarray, keys: np.ndarray,
                     weights: np.ndarray) -> np.ndarray:
    """o_f = sum_i v_i h(k_i) / sum_i v_i for every bag (TransRetrieval §3.2, weighted
    average aggregation; the division by the weight sum is the step §3.2 adds to the
    weighted sum of §3.2's profiling paragraph).

    rows: [R, D] embedding rows h(.); keys index rows; offsets: CSR bag bounds.
    """
    rows = np.asarray(rows, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    n_bags = len(offsets) - 1
    D = rows.shape[1]
    v = np.asarray(weights, dtype=np.float64)
    out = np.zeros((n_bags, D), dtype=np.float64)
    counts = np.diff(offsets)
    nonempty = counts > 0
    if not nonempty.any():
        return out
    contrib = v[:, None] * rows[np.asarray(keys, dtype=np.int64)]
    starts = offsets[:-1][nonempty]
    num = np.add.reduceat(contrib, starts, axis=0)
    den = np.add.reduceat(v, starts)
    res = np.zeros_like(num)
    ok = den != 0
    res[ok] = num[ok] / den[ok, None]
    out[nonempty] = res
    return out


def weighted_sum(rows, offsets, keys, weights) -> np.ndarray:
    """The conventional aggregator §3.2 replaces: sum_i v_i h(k_i) (no normalisation)."""
    rows = np.asarray(rows, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    out = np.zeros((len(offsets) - 1, rows.shape[1]))
    for b in range(len(offsets) - 1):
        s, e = offsets[b], offsets[b + 1]
        for i in range(s, e):
            out[b] += float(weights[i]) * rows[int(keys[i])]
    return out


def max_pool(rows, offsets, keys) -> np.ndarray:
    """Element-wise maximum of a bag's embedding rows: the max-pooling aggregator §3.2
    rejects (extreme-value bias).  Weights do not enter; an empty bag gives zeros."""
    rows = np.asarray(rows, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    out = np.zeros((len(offsets) - 1, rows.shape[1]))
    for b in range(len(offsets) - 1):
        s, e = offsets[b], offsets[b + 1]
        if e > s:
            out[b] = rows[np.asarray(keys[s:e], dtype=np.int64)].max(axis=0)
    return out


def aggregate(rows, offsets, keys, weights, mode: str = "mean", post_ln: bool = False) -> np.ndarray:
    """One token per bag with the aggregator `mode` ("mean": weighted average, §3.2;
    "sum": weighted sum; "max": max pooling), optionally followed by the post-aggregation
    LayerNorm §3.2 compares against (no affine parameters, eps as everywhere else)."""
    if mode == "mean":
        o = weighted_average(rows, offsets, keys, weights)
    elif mode == "sum":
        o = weighted_sum(rows, offsets, keys, weights)
    elif mode == "max":
        o = max_pool(rows, offsets, keys)
    else:
        raise ValueError(mode)
    if post_ln:
        o = layer_norm(o, np.ones(o.shape[1]), np.zeros(o.shape[1]))
    return o


# ------------------------------------------------------------------ building blocks

def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray) -> np.ndarray:
    """LayerNorm over the last axis: biased variance, eps inside the square root."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + EPS) * g + b


def prelu(x: np.ndarray, a: np.ndarray) -> np.ndarray:
    return np.where(x >= 0, x, a * x)


def _p(P, k):
    return np.asarray(P[k], dtype=np.float64)


# ------------------------------------------------------------------ §3.3 target compressor

def compress_targets(P, X: np.ndarray) -> np.ndarray:
    """Target compressor (TransRetrieval §3.3): 3-layer MLP over the concatenation of a
    candidate's target-field tokens; PReLU and LayerNorm between layers; last layer a
    plain linear projection to one D-dim token.  X: [n, F*D] -> [n, D]."""
    h = np.asarray(X, dtype=np.float64)
    for i in range(3):
        h = _mm(h, _p(P, f"c{i}.W")) + _p(P, f"c{i}.b")
        if i < 2:
            h = layer_norm(prelu(h, _p(P, f"c{i}.prelu")), _p(P, f"c{i}.ln_g"), _p(P, f"c{i}.ln_b"))
    return h


# ------------------------------------------------------------------ §3.1/§3.3/§3.4 backbone

def _split_heads(x: np.ndarray, H: int) -> np.ndarray:
    return x.reshape(*x.shape[:-1], H, x.shape[-1] // H)


def _ffn(P, l: int, x: np.ndarray) -> np.ndarray:
    """Pre-LN ReLU FFN sub-block output (without the residual)."""
    a = layer_norm(x, _p(P, f"l{l}.ln2_g"), _p(P, f"l{l}.ln2_b"))
    h = np.maximum(_mm(a, _p(P, f"l{l}.W1")) + _p(P, f"l{l}.b1"), 0.0)
    return _mm(h, _p(P, f"l{l}.W2")) + _p(P, f"l{l}.b2")


def _qkv(P, l: int, x: np.ndarray):
    a = layer_norm(x, _p(P, f"l{l}.ln1_g"), _p(P, f"l{l}.ln1_b"))
    return tuple(_mm(a, _p(P, f"l{l}.W{m}")) + _p(P, f"l{l}.b{m}") for m in "qkv")


def prefill_user(P, n_head: int, user_tokens: np.ndarray, domain: int):
    """User side of a request (TransRetrieval §3.1 stages (3)-(4)): add s_d to every user
    token, run the N-layer Pre-LN Transformer with ReLU FFN over the user tokens alone
    (every user token attends to every user token), and return the per-layer keys and
    values that every candidate of the request reuses.

    user_tokens: [L_u, D] -> (K [N, L_u, D], V [N, L_u, D]).
    """
    x = np.asarray(user_tokens, dtype=np.float64) + _p(P, "domain_emb")[domain]
    n_layer = sum(1 for k in P if k.endswith(".Wq"))
    L_u, D = x.shape
    dh = D // n_head
    Ks, Vs = [], []
    for l in range(n_layer):
        q, k, v = _qkv(P, l, x)
        Ks.append(k)
        Vs.append(v)
        qh, kh, vh = (_split_heads(t, n_head) for t in (q, k, v))      # [L, H, dh]
        if L_u:
            s = np.einsum("ihd,jhd->hij", qh, kh) / np.sqrt(dh)
            _count(2 * L_u * L_u * D)
            s = s - s.max(axis=-1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=-1, keepdims=True)
            o = np.einsum("hij,jhd->ihd", p, vh).reshape(L_u, D)
            _count(2 * L_u * L_u * D)
        else:
            o = np.zeros((0, D))
        x = x + _mm(o, _p(P, f"l{l}.Wo")) + _p(P, f"l{l}.bo")
        x = x + _ffn(P, l, x)
    return np.stack(Ks) if Ks else np.zeros((0, L_u, D)), np.stack(Vs) if Vs else np.zeros((0, L_u, D))


def score_candidates(P, n_head: int, tokens: np.ndarray, K: np.ndarray, V: np.ndarray,
                     domain: int) -> np.ndarray:
    """Score single-token candidates against one request's cached user K/V.

    TransRetrieval §3.3: with the user K/V computed once per request, each candidate
    needs only its own Q/K/V/O projections, the FFN, and attention over the L_u user
    positions; here it also attends to its own key/value, as a token of the sequence
    [user tokens..., candidate] does when user tokens cannot see the candidate.
    §3.4: s_d is added to the candidate token.  Head: final LayerNorm, linear D -> 1.

    tokens: [n, D] compressed candidate tokens; K, V: [N, L_u, D].  Returns [n] scores.
    """
    y = np.asarray(tokens, dtype=np.float64) + _p(P, "domain_emb")[domain]
    n, D = y.shape
    dh = D // n_head
    n_layer = K.shape[0]
    L_u = K.shape[1]
    for l in range(n_layer):
        q, k, v = _qkv(P, l, y)
        qh, kh, vh = (_split_heads(t, n_head) for t in (q, k, v))      # [n, H, dh]
        Ku = _split_heads(np.asarray(K[l], dtype=np.float64), n_head)  # [L_u, H, dh]
        Vu = _split_heads(np.asarray(V[l], dtype=np.float64), n_head)
        s_user = np.einsum("nhd,lhd->nhl", qh, Ku)
        s_self = np.einsum("nhd,nhd->nh", qh, kh)[..., None]
        _count(2 * n * (L_u + 1) * D)
        s = np.concatenate([s_user, s_self], axis=-1) / np.sqrt(dh)   # [n, H, L_u + 1]
        s = s - s.max(axis=-1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=-1, keepdims=True)
        o = np.einsum("nhl,lhd->nhd", p[..., :L_u], Vu) + p[..., L_u:] * vh
        _count(2 * n * (L_u + 1) * D)
        y = y + _mm(o.reshape(n, D), _p(P, f"l{l}.Wo")) + _p(P, f"l{l}.bo")
        y = y + _ffn(P, l, y)
    z = layer_norm(y, _p(P, "lnf_g"), _p(P, "lnf_b"))
    return (_mm(z, _p(P, "w_head")[:, None]) + _p(P, "b_head"))[:, 0]


def score_candidates_uncompressed(P, n_head: int, tokens: np.ndarray, K: np.ndarray, V: np.ndarray,
                                  domain: int) -> np.ndarray:
    """The uncompressed-target alternative §3.3 measures compression against: a candidate is
    L_t target tokens (tokens: [n, L_t, D]).  Each token attends to the request's L_u cached
    user keys/values and to the keys/values of its own candidate's L_t tokens, as the tokens
    of [user tokens..., candidate tokens] do when user tokens cannot see the candidate;
    candidates never see each other.  The score is the mean over the candidate's tokens of
    w . LayerNorm_f(y_t) + b (the pages give no head for this variant; reading).  With
    L_t = 1 this is score_candidates.  Returns [n]."""
    t = np.asarray(tokens, dtype=np.float64)
    n, L_t, D = t.shape
    y = t.reshape(n * L_t, D) + _p(P, "domain_emb")[domain]
    dh = D // n_head
    L_u = K.shape[1]
    for l in range(K.shape[0]):
        q, k, v = _qkv(P, l, y)
        qh, kh, vh = (_split_heads(x, n_head).reshape(n, L_t, n_head, dh) for x in (q, k, v))
        Ku = _split_heads(np.asarray(K[l], dtype=np.float64), n_head)
        Vu = _split_heads(np.asarray(V[l], dtype=np.float64), n_head)
        s_user = np.einsum("cthd,lhd->cthl", qh, Ku)
        s_own = np.einsum("cthd,cshd->cths", qh, kh)                   # own candidate's tokens
        _count(2 * n * L_t * (L_u + L_t) * D)
        sc = np.concatenate([s_user, s_own], axis=-1) / np.sqrt(dh)     # [n, L_t, H, L_u + L_t]
        sc = sc - sc.max(axis=-1, keepdims=True)
        p = np.exp(sc)
        p = p / p.sum(axis=-1, keepdims=True)
        o = np.einsum("cthl,lhd->cthd", p[..., :L_u], Vu) + np.einsum("cths,cshd->cthd", p[..., L_u:], vh)
        _count(2 * n * L_t * (L_u + L_t) * D)
        y = y + _mm(o.reshape(n * L_t, D), _p(P, f"l{l}.Wo")) + _p(P, f"l{l}.bo")
        y = y + _ffn(P, l, y)
    z = layer_norm(y, _p(P, "lnf_g"), _p(P, "lnf_b"))
    per_token = (_mm(z, _p(P, "w_head")[:, None]) + _p(P, "b_head"))[:, 0]
    return per_token.reshape(n, L_t).mean(axis=1)


def topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, descending; equal scores by lower index first."""
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(len(s)), -s))
    return order[:k]


def flops_per_candidate_closed_form(D: int, n_layer: int, L_u: int, L_t: int = 1,
                                    self_term: bool = True, head: bool = True) -> int:
    """Per-candidate FLOPs of the scoring stack: per layer 16*L_t*D^2 + 4*L_t*L_u*D
    (TransRetrieval §3.3), plus 4*D per layer for the candidate's own key/value when
    ``self_term`` and 2*D for the head."""
    per_layer = 16 * L_t * D * D + 4 * L_t * (L_u + (1 if self_term else 0)) * D
    return n_layer * per_layer + (2 * D if head else 0)
