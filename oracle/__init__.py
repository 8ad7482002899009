"""Oracle for TransRetrieval candidate scoring -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU restatement of the method, used to check the CUDA path.  Only the
tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline / reference leg may
import it; the product package never does, and shares no code with it.  The only
module both sides use is ``datagen`` (seeded inputs, none of the method's arithmetic).
"""
from .transretrieval import (EPS, FlopCounter, compress_targets, flops_per_candidate_closed_form,
                             layer_norm, prefill_user, prelu, score_candidates, score_candidates_uncompressed, topk,
                             weighted_average, weighted_sum, max_pool, aggregate)
from .pipeline import aggregate_bags, score_request, score_request_candidates

__all__ = [
    "EPS", "FlopCounter", "compress_targets", "flops_per_candidate_closed_form", "layer_norm",
    "prefill_user", "prelu", "score_candidates", "score_candidates_uncompressed", "topk", "weighted_average", "weighted_sum", "max_pool", "aggregate",
    "score_request", "score_request_candidates", "aggregate_bags",
]
