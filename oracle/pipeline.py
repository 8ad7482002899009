"""Whole-request oracle: the four stages of TransRetrieval §3.1 in order.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import datagen
from .transretrieval import compress_targets, prefill_user, score_candidates, weighted_average


def aggregate_bags(w: "datagen.Workload", bags: "datagen.Bags", side: str) -> np.ndarray:
    """Weighted average of every bag, reading only the touched table rows."""
    rows, keys = datagen.compact_rows(w, bags, side)
    return weighted_average(rows, bags.offsets, keys, bags.weights)


@dataclass
class RequestResult:
    user_tokens: np.ndarray     # [L_u, D]
    K: np.ndarray               # [N, L_u, D]
    V: np.ndarray               # [N, L_u, D]
    X: np.ndarray               # [n, F*D]  concatenated target-field tokens
    tokens: np.ndarray          # [n, D]    compressed candidate tokens
    scores: np.ndarray          # [n]


def _select_candidates(req: "datagen.Request", cand: np.ndarray, F: int) -> "datagen.Bags":
    tb = req.target
    cand = np.asarray(cand, dtype=np.int64)
    bag_ids = (cand[:, None] * F + np.arange(F)[None, :]).reshape(-1)
    counts = np.diff(tb.offsets)[bag_ids]
    off = np.zeros(len(bag_ids) + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    starts = tb.offsets[bag_ids]
    idx = (np.repeat(starts - off[:-1], counts) + np.arange(int(off[-1]))).astype(np.int64)
    return datagen.Bags(off, tb.keys[idx], tb.weights[idx], tb.bag_table[bag_ids])


def score_request_candidates(w: "datagen.Workload", P, req: "datagen.Request", cand: np.ndarray,
                             K: np.ndarray, V: np.ndarray):
    """Candidate side of one request given its user K/V: aggregate the selected
    candidates' target fields, compress, score.  Returns (X, tokens, scores)."""
    dims = w.dims
    F = dims.n_target_fields
    tb = _select_candidates(req, cand, F)
    X = aggregate_bags(w, tb, "target").reshape(-1, F * dims.D)
    tokens = compress_targets(P, X)
    return X, tokens, score_candidates(P, dims.n_head, tokens, K, V, req.domain)


def score_request(w: "datagen.Workload", P, req: "datagen.Request",
                  cand: np.ndarray | None = None) -> RequestResult:
    """(1) weighted-average aggregation of user and target fields, (2) target compression,
    (3) domain embedding, (4) N-layer Pre-LN Transformer with the user K/V computed once
    and reused by every candidate; then the linear head.  ``cand`` restricts the
    candidates scored (indices into the request's candidates)."""
    dims = w.dims
    user_tokens = aggregate_bags(w, req.user, "user")
    K, V = prefill_user(P, dims.n_head, user_tokens, req.domain)
    if cand is None:
        cand = np.arange(req.n_cand)
    X, tokens, scores = score_request_candidates(w, P, req, cand, K, V)
    return RequestResult(user_tokens, K, V, X, tokens, scores)
