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


# ------------------------------------------------------------------ one request over ranks
#
# A request too large for one GPU's time budget can be split: every rank recomputes the
# request's user side (cheaper than sending the K/V cache) and scores a contiguous slice of
# its candidates, then the ranks exchange their local top-k in one all-gather and each
# selects the request's top-k from the world x k gathered pairs.  The local top-k of each
# slice holds every candidate of that slice that can reach the global top-k, so the merge
# is exact.


def split_request(n_cand: int, world: int, tile: int = 128) -> List[int]:
    """Boundaries c[0] = 0 <= c[1] <= ... <= c[world] = n_cand: rank r scores candidates
    [c[r], c[r+1]) of one request.  Cuts fall on multiples of ``tile`` (the score kernel's
    tile), and the ranks' tile counts differ by at most one."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if n_cand < 0 or tile < 1:
        raise ValueError("n_cand must be >= 0 and tile >= 1")
    T = -(-n_cand // tile)
    return [min(n_cand, tile * (T * r // world)) for r in range(world)] + [n_cand]


def pack_topk(local_idx, local_scores, k: int):
    """One rank's top-k as the all-gather sends it: [2k] int64, the k indices then the k
    scores' fp32 bits, padding (index -1) turned into NaN scores so it ranks last."""
    import torch

    if local_idx.numel() != k or local_scores.numel() != k:
        raise ValueError("local_idx and local_scores must hold k entries")
    s = torch.where(local_idx >= 0, local_scores, torch.full_like(local_scores, float("nan")))
    return torch.cat([local_idx.to(torch.int64), s.contiguous().view(torch.int32).to(torch.int64)])


def merge_gathered(parts, k: int, select=None):
    """The request's top-k from every rank's packed list, in rank order: (idx [k] int64,
    scores [k] fp32), padded with -1 / -inf.  ``select(scores, k)`` returns the positions
    of the k best gathered scores (default: tr_topk on the device)."""
    import torch

    if select is None:
        from . import api

        def select(sc, kk):
            pos, _ = api.topk(sc, [0, sc.numel()], kk)
            return pos[0]
    world = len(parts)
    allp = torch.stack(parts).view(world, 2, k)
    all_idx = allp[:, 0, :].reshape(-1)
    all_scores = allp[:, 1, :].reshape(-1).to(torch.int32).view(torch.float32)
    pos = select(all_scores, k)
    idx = all_idx[pos]
    sc = all_scores[pos]
    return idx, torch.where(idx >= 0, sc, torch.full_like(sc, float("-inf")))


def merge_topk(local_idx, local_scores, k: int, group=None, select=None):
    """The top-k of one request whose candidates are split over the ranks of ``group``.

    local_idx [k] int64 / local_scores [k] fp32: this rank's top-k over its slice as
    tr_topk gives it (descending, equal scores by lower index, padded with -1 / -inf), the
    indices already offset to the whole request.  One collective gathers every rank's
    pairs (pack_topk: one int64 tensor of 2k entries); then every rank selects the k best
    of the world * k gathered pairs (merge_gathered).  Rank r's slice precedes rank
    r + 1's and each list is ordered, so equal scores resolve to the lower candidate index
    as in a single tr_topk over the request.  Padding competes as NaN (below every other
    score): only a request with NaN scores and fewer than k other candidates can see
    padding win a tie.  Returns (idx [k] int64, scores [k] fp32), identical on every rank."""
    import torch
    import torch.distributed as dist

    packed = pack_topk(local_idx, local_scores, k)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    parts = [packed]
    if world > 1:
        parts = [torch.empty_like(packed) for _ in range(world)]
        dist.all_gather(parts, packed, group=group)
    return merge_gathered(parts, k, select)
