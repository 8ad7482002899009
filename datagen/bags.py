"""Seeded (key, weight) bags shaped like TransRetrieval's feature fields.

A field is a set of (key, weight) pairs (TransRetrieval §3.1, "Feature Representation").
Bags are stored CSR-style: ``offsets`` (int64, n_bags+1), ``keys`` (int32 row indices) and
``weights`` (fp32).  ``bag_table`` (int32, n_bags) names the table each bag reads.

Recipe (the pages publish no data; these stand in for the shapes of the Industrial and
KuaiRand workloads):
* user fields: n_f ~ Uniform{lo..hi}; keys ~ Zipf(s) over the table's rows, rank -> row
  through a seeded affine permutation ``row = (a * rank + b) mod rows``;
* target fields: n_f ~ Uniform{lo..hi}; keys uniform over the table's rows;
* weights ~ Uniform(0.1, 1).
No arithmetic of the method lives here.
"""
from __future__ import annotations

from dataclasses import dataclass
from functools import lru_cache
from math import gcd
from typing import List

import numpy as np

from .configs import Workload


@dataclass
class Bags:
    offsets: np.ndarray    # int64 [n_bags + 1]
    keys: np.ndarray       # int32 [nnz]
    weights: np.ndarray    # fp32  [nnz]
    bag_table: np.ndarray  # int32 [n_bags]

    @property
    def n_bags(self) -> int:
        return len(self.offsets) - 1

    @property
    def nnz(self) -> int:
        return int(self.offsets[-1])


@dataclass
class Request:
    L_u: int
    domain: int
    user: Bags             # L_u bags, bag f -> user table f mod user_tables
    target: Bags           # n_cand * F bags, bag c*F + f -> target table f mod len(target_rows)
    n_cand: int


@lru_cache(maxsize=8)
def _zipf_cdf(n: int, s: float) -> np.ndarray:
    p = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(p)
    return c / c[-1]


def _zipf_rows(rng: np.random.Generator, n: int, rows: int, s: float, a: int, b: int) -> np.ndarray:
    rank = np.searchsorted(_zipf_cdf(rows, s), rng.random(n), side="right")
    rank = np.minimum(rank, rows - 1).astype(np.int64)
    return ((a * rank + b) % rows).astype(np.int32)


def _affine_perm(rng: np.random.Generator, rows: int):
    while True:
        a = int(rng.integers(1, rows))
        if gcd(a, rows) == 1:
            return a, int(rng.integers(0, rows))


def _offsets(counts: np.ndarray) -> np.ndarray:
    off = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    return off


def make_user_bags(rng: np.random.Generator, w: Workload, L_u: int) -> Bags:
    counts = rng.integers(w.user_nf[0], w.user_nf[1] + 1, size=L_u)
    table = (np.arange(L_u) % w.user_tables).astype(np.int32)
    keys = np.empty(int(counts.sum()), dtype=np.int32)
    off = _offsets(counts)
    perms = [_affine_perm(rng, w.user_rows) for _ in range(w.user_tables)]
    for f in range(L_u):
        a, b = perms[table[f]]
        keys[off[f]:off[f + 1]] = _zipf_rows(rng, int(counts[f]), w.user_rows, w.zipf_s, a, b)
    weights = rng.uniform(0.1, 1.0, size=len(keys)).astype(np.float32)
    return Bags(off, keys, weights, table)


def make_target_bags(rng: np.random.Generator, w: Workload, n_cand: int) -> Bags:
    F = w.dims.n_target_fields
    n_bags = n_cand * F
    counts = rng.integers(w.target_nf[0], w.target_nf[1] + 1, size=n_bags)
    table = np.tile((np.arange(F) % len(w.target_rows)).astype(np.int32), n_cand)
    off = _offsets(counts)
    rows_per_key = np.repeat(np.asarray(w.target_rows, dtype=np.int64)[table], counts)
    keys = np.floor(rng.random(len(rows_per_key)) * rows_per_key).astype(np.int64)
    keys = np.minimum(keys, rows_per_key - 1).astype(np.int32)
    weights = rng.uniform(0.1, 1.0, size=len(keys)).astype(np.float32)
    return Bags(off, keys, weights, table)


def make_requests(w: Workload, seed: int | None = None) -> List[Request]:
    """All requests of a workload.  Streams: [params, user bags, target bags, domains]."""
    ss = np.random.SeedSequence(w.seed if seed is None else seed)
    _, s_user, s_target, s_dom = ss.spawn(4)
    r_user = np.random.default_rng(s_user)
    r_target = np.random.default_rng(s_target)
    r_dom = np.random.default_rng(s_dom)
    lu = r_user.integers(w.L_u[0], w.L_u[1] + 1, size=w.n_requests)
    reqs = []
    for r in range(w.n_requests):
        user = make_user_bags(r_user, w, int(lu[r]))
        target = make_target_bags(r_target, w, w.n_cand_per_request)
        dom = int(r_dom.integers(0, w.dims.n_domains))
        reqs.append(Request(int(lu[r]), dom, user, target, w.n_cand_per_request))
    return reqs


def scale_weights(b: Bags, c: float) -> Bags:
    return Bags(b.offsets, b.keys, (b.weights * np.float32(c)).astype(np.float32), b.bag_table)
