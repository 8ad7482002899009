"""B200-native TransRetrieval candidate scoring.

The compute lives in libtr.so (hand-written CUDA for sm_100a behind the C ABI in
include/tr.h); this package is its Python binding plus the device-resident workload
driver.  There is no CPU fallback: every call raises if libtr.so is missing.
"""
from . import api
from .api import (Model, TrError, aggregate, compress_target_bags, compress_targets, kv_cache_bytes,
                  prefill_user, prefill_user_noalloc, score_candidates, sync_status, topk)

__all__ = ["api", "Model", "TrError", "aggregate", "compress_target_bags", "compress_targets", "kv_cache_bytes",
           "prefill_user", "prefill_user_noalloc", "score_candidates", "sync_status", "topk"]
