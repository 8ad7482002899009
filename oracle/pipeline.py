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


def score_request(w: "datagen.Workload", P, req: "datagen.Request",
                  cand: np.ndarray | None = None) -> RequestResult:
    """(1) weighted-average aggregation of user and target fields, (2) target compression,
    (3) domain embedding, (4) N-layer Pre-LN Transformer with the user K/V computed once
    and reused by every candidate; then the linear head.  ``cand`` restricts the
    candidates scored (indices into the request's candidates)."""
    dims = w.dims
    F = dims.n_target_fields
    user_tokens = aggregate_bags(w, req.user, "user")
    K, V = prefill_user(P, dims.n_head, user_tokens, req.domain)
    tb = req.target
    if cand is not None:
        cand = np.asarray(cand, dtype=np.int64)
        bag_ids = (cand[:, None] * F + np.arange(F)[None, :]).reshape(-1)
        counts = np.diff(tb.offsets)[bag_ids]
        off = np.zeros(len(bag_ids) + 1, dtype=np.int64)
        np.cumsum(counts, out=off[1:])
        idx = np.concatenate([np.arange(tb.offsets[b], tb.offsets[b + 1]) for b in bag_ids]) \
            if len(bag_ids) else np.zeros(0, dtype=np.int64)
        tb = datagen.Bags(off, tb.keys[idx], tb.weights[idx], tb.bag_table[bag_ids])
    X = aggregate_bags(w, tb, "target").reshape(-1, F * dims.D)
    tokens = compress_targets(P, X)
    scores = score_candidates(P, dims.n_head, tokens, K, V, req.domain)
    return RequestResult(user_tokens, K, V, X, tokens, scores)
