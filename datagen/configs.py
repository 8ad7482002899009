"""Workload definitions: model sizes and the synthetic-input recipe.

The five workloads mirror the shapes TransRetrieval reports (TransRetrieval,
"Model-based Retrieval" and Table 2: ~4x10^4 candidates per request over a 52M
corpus, the 64D-3L and 128D-5L backbones).  This module holds sizes only; no
arithmetic of the method lives here.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Tuple


@dataclass(frozen=True)
class ModelDims:
    """Backbone and compressor sizes (xD-yL notation of TransRetrieval §4.1)."""
    D: int                      # token width
    n_layer: int                # Transformer layers
    n_head: int                 # attention heads, d_h = D / n_head
    ffn_hidden: int             # FFN hidden width (2D: forced by the 16*D^2 per-layer count, §3.3)
    n_target_fields: int        # F, target-side fields concatenated into the compressor input
    comp_dims: Tuple[int, int, int, int]  # compressor F*D -> c1 -> c2 -> D (§3.3)
    n_domains: int              # learned domain embeddings s_d (§3.4)
    dtype: str                  # "f32" or "bf16": storage/operand type of tables and weights

    @property
    def d_head(self) -> int:
        return self.D // self.n_head


@dataclass(frozen=True)
class Workload:
    name: str
    dims: ModelDims
    n_requests: int
    L_u: Tuple[int, int]            # user field count, inclusive range (fixed when lo == hi)
    user_nf: Tuple[int, int]        # keys per user field, Uniform{lo..hi}
    user_tables: int                # number of user tables; field f uses table f mod user_tables
    user_rows: int
    target_nf: Tuple[int, int]      # keys per target field, Uniform{lo..hi}
    target_rows: Tuple[int, ...]    # rows of each target table; field f uses table f mod len
    n_cand_per_request: int
    zipf_s: float = 1.1             # user keys ~ Zipf(s) over table rows
    seed: int = 0

    @property
    def n_cand(self) -> int:
        return self.n_cand_per_request * self.n_requests

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY_DIMS = ModelDims(D=32, n_layer=1, n_head=2, ffn_hidden=64, n_target_fields=4,
                      comp_dims=(128, 64, 32, 32), n_domains=2, dtype="f32")
DIMS_64D3L = ModelDims(D=64, n_layer=3, n_head=4, ffn_hidden=128, n_target_fields=8,
                       comp_dims=(512, 256, 128, 64), n_domains=4, dtype="bf16")
DIMS_128D5L = ModelDims(D=128, n_layer=5, n_head=8, ffn_hidden=256, n_target_fields=8,
                        comp_dims=(1024, 512, 256, 128), n_domains=4, dtype="bf16")

WORKLOADS = {
    # 1 request, 8 user fields of 1..20 Zipf keys over one 10k-row table, 4 target fields
    # of 1..5 keys over one 10k-row table, 256 candidates, fp32.
    "tiny": Workload("tiny", TINY_DIMS, 1, (8, 8), (1, 20), 1, 10_000, (1, 5), (10_000,), 256),
    "64d3l": Workload("64d3l", DIMS_64D3L, 1, (32, 32), (1, 50), 8, 1_000_000, (1, 8),
                      (1_000_000,) * 8, 40_000, seed=1),
    "128d5l": Workload("128d5l", DIMS_128D5L, 1, (64, 64), (1, 100), 16, 4_000_000, (1, 8),
                       (4_000_000,) * 8, 40_000, seed=2),
    # 16 requests of 4096 candidates, L_u ~ Uniform{16..128}, packed into one 65,536 batch.
    "packed": Workload("packed", DIMS_128D5L, 16, (16, 128), (1, 100), 16, 4_000_000, (1, 8),
                       (4_000_000,) * 8, 4096, seed=3),
    # One 52M-row target table for field 0 (plus 7 tables of 4M), 520k candidates, uniform keys.
    "large": Workload("large", DIMS_128D5L, 1, (64, 64), (1, 100), 16, 4_000_000, (1, 8),
                      (52_000_000,) + (4_000_000,) * 7, 520_000, seed=4),
}


def scaled(w: Workload, n_cand_per_request: int | None = None, rows: int | None = None,
           seed: int | None = None) -> Workload:
    """Same model and recipe, fewer candidates and/or smaller tables (parity-test sizes)."""
    kw = {}
    if n_cand_per_request is not None:
        kw["n_cand_per_request"] = n_cand_per_request
    if rows is not None:
        kw["user_rows"] = min(w.user_rows, rows)
        kw["target_rows"] = tuple(min(r, rows) for r in w.target_rows)
    if seed is not None:
        kw["seed"] = seed
    return w.with_(**kw)
