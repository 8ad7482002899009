"""Data-parallel sharding of the scoring step over ranks (one process per GPU).

Requests are independent in TransRetrieval candidate scoring (§3.1): each request's
candidates attend only to that request's own user K/V cache, and the score of a candidate
depends on nothing else in the batch.  So ranks take disjoint, contiguous groups of
requests and exchange nothing on the data path; the only collective is the max of the
timed region over ranks.  Host logic only: no CUDA is touched here.
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np


def shard_bounds(n_cand: Sequence[int], world: int) -> List[int]:
    """Boundaries b[0] = 0 <= b[1] <= ... <= b[world] = len(n_cand): rank r takes requests
    [b[r], b[r+1]).  Contiguous split at the quantiles of the cumulative candidate count, so
    every rank's candidate count is within one request of total / world."""
    if world < 1:
        raise ValueError("world must be >= 1")
    n = np.asarray(n_cand, dtype=np.int64)
    if (n < 0).any():
        raise ValueError("candidate counts must be >= 0")
    cum = np.concatenate([[0], np.cumsum(n)])
    total = int(cum[-1])
    bounds = [0]
    for r in range(1, world):
        target = total * r / world
        # first request boundary whose prefix reaches the target
        b = int(np.searchsorted(cum, target, side="left"))
        bounds.append(min(max(b, bounds[-1]), len(n)))
    bounds.append(len(n))
    return bounds


def local_requests(reqs: Sequence, rank: int, world: int) -> list:
    """The requests rank ``rank`` of ``world`` scores."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world {world}")
    b = shard_bounds([r.n_cand for r in reqs], world)
    return list(reqs[b[rank]:b[rank + 1]])


def rank_seed(base_seed: int, rank: int, set_index: int) -> int:
    """Seed of request set ``set_index`` on rank ``rank`` when every rank draws its own
    requests (weak scaling): distinct for every (rank, set) pair below 2**16 each."""
    if not (0 <= rank < 1 << 16 and 0 <= set_index < 1 << 16):
        raise ValueError("rank and set_index must be in [0, 65536)")
    return (int(base_seed) << 32) | (rank << 16) | set_index


def max_over_ranks(x: float, group=None) -> float:
    """Max of a host scalar over the ranks of ``group`` (the default group if None); the
    value itself when torch.distributed is not initialised.  Used for timings only."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(x)
    if dist.get_backend(group) == "nccl":
        dev = torch.device("cuda", torch.cuda.current_device())
    else:
        dev = torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
