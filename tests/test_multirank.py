"""Multi-rank host logic on CPU: request sharding, per-rank seeds and the max-over-ranks
timing reduction, with two gloo ranks.  The end-to-end check scores each rank's shard
with the oracle and compares the gathered result with one process scoring everything:
requests are independent, so sharding must not change a single bit."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import datagen
from transformer_candidate_scoring_b200.shard import (local_requests, max_over_ranks, merge_topk, rank_seed,
                                                      shard_bounds, split_request)


class _R:
    def __init__(self, n):
        self.n_cand = n


@pytest.mark.parametrize("n_cand,world", [
    ([40000], 1), ([40000], 2), ([4096] * 16, 2), ([4096] * 16, 3), ([4096] * 16, 8),
    ([1, 100, 5, 5000, 0, 7, 3000, 12], 4), ([0, 0, 0], 2), ([], 3), ([10, 20], 5),
])
def test_shard_bounds_partition(n_cand, world):
    b = shard_bounds(n_cand, world)
    assert len(b) == world + 1 and b[0] == 0 and b[-1] == len(n_cand)
    assert all(b[i] <= b[i + 1] for i in range(world))
    cum = np.concatenate([[0], np.cumsum(np.asarray(n_cand, np.int64))])
    total = int(cum[-1])
    biggest = max(n_cand) if n_cand else 0
    for r in range(world):
        got = int(cum[b[r + 1]] - cum[b[r]])
        assert abs(got - total / world) <= biggest, (r, got, total / world)
    # every request on exactly one rank
    reqs = [_R(n) for n in n_cand]
    seen = [id(x) for r in range(world) for x in local_requests(reqs, r, world)]
    assert sorted(seen) == sorted(id(x) for x in reqs)


def test_shard_bounds_rejects():
    with pytest.raises(ValueError):
        shard_bounds([1, 2], 0)
    with pytest.raises(ValueError):
        shard_bounds([1, -2], 2)
    with pytest.raises(ValueError):
        local_requests([_R(1)], 2, 2)


def test_rank_seed_distinct():
    seeds = {rank_seed(2, r, s) for r in range(8) for s in range(16)}
    assert len(seeds) == 8 * 16
    assert rank_seed(2, 0, 0) != rank_seed(3, 0, 0)
    with pytest.raises(ValueError):
        rank_seed(2, 1 << 16, 0)


def test_max_over_ranks_single_process():
    assert max_over_ranks(3.5) == 3.5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import oracle

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = datagen.scaled(datagen.WORKLOADS["tiny"], n_cand_per_request=24).with_(n_requests=5, L_u=(0, 9))
        P = datagen.workload_params(w)
        reqs = datagen.make_requests(w)
        mine = local_requests(reqs, rank, world)
        first = shard_bounds([r.n_cand for r in reqs], world)[rank]
        scores = {first + i: oracle.score_request(w, P, r).scores for i, r in enumerate(mine)}
        gathered = [None] * world
        dist.all_gather_object(gathered, scores)
        # each rank draws its own requests for the weak-scaling bench: they must differ
        own = datagen.make_requests(w, seed=rank_seed(w.seed, rank, 0))[0].target.keys
        keys = [None] * world
        dist.all_gather_object(keys, own)
        t = max_over_ranks(1.5 + rank)
        if rank == 0:
            merged = {}
            for g in gathered:
                assert not set(g) & set(merged)
                merged.update(g)
            ref = [oracle.score_request(w, P, r).scores for r in reqs]
            ok_scores = sorted(merged) == list(range(len(reqs))) and all(
                np.array_equal(merged[i], ref[i]) for i in range(len(reqs)))
            ok_keys = not np.array_equal(keys[0], keys[1])
            q.put((ok_scores, ok_keys, t))
        else:
            q.put(("rank", rank, t))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_shard_equals_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    out = [q.get(timeout=5) for _ in range(2)]
    main = [o for o in out if o[0] != "rank"][0]
    other = [o for o in out if o[0] == "rank"][0]
    assert main[0], "sharded oracle scores differ from the single-process scores"
    assert main[1], "ranks drew identical requests"
    assert main[2] == 2.5 and other[2] == 2.5


@pytest.mark.parametrize("n,world,tile", [(40000, 8, 128), (40000, 1, 128), (100, 4, 128), (0, 2, 128),
                                          (1000, 3, 7), (129, 2, 128)])
def test_split_request_partition(n, world, tile):
    c = split_request(n, world, tile)
    assert len(c) == world + 1 and c[0] == 0 and c[-1] == n
    assert all(c[i] <= c[i + 1] for i in range(world))
    assert all(x % tile == 0 for x in c[:-1])
    tiles = [-(-(c[i + 1] - c[i]) // tile) for i in range(world)]
    assert max(tiles) - min(tiles) <= 1


def _local_topk(scores, lo, hi, k):
    """This rank's top-k over candidates [lo, hi) as tr_topk returns it: descending, equal
    scores by lower index, padded with -1 / -inf; indices offset to the whole request."""
    import torch

    import oracle
    sel = oracle.topk(scores[lo:hi], k) if hi > lo else np.zeros(0, np.int64)
    idx = np.full(k, -1, np.int64)
    sc = np.full(k, -np.inf, np.float32)
    idx[:len(sel)] = sel + lo
    sc[:len(sel)] = scores[lo:hi][sel]
    return torch.from_numpy(idx), torch.from_numpy(sc)


def _topk_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        def select(s, kk):          # the oracle's top-k on the gathered scores (test stand-in for tr_topk)
            return torch.from_numpy(oracle.topk(s.numpy(), kk))
        results = []
        rng = np.random.default_rng(5)
        for n, k, levels in [(1000, 100, 7), (1000, 37, 0), (150, 200, 5), (3, 5, 0), (257, 256, 2)]:
            # few distinct values make ties, many across the ranks' boundary
            raw = rng.integers(0, levels, size=n) if levels else rng.normal(size=n)
            scores = raw.astype(np.float32)
            c = split_request(n, world)
            li, ls = _local_topk(scores, c[rank], c[rank + 1], k)
            idx, sc = merge_topk(li, ls, k, select=select)
            want = oracle.topk(scores, k)
            ok = (np.array_equal(idx.numpy()[:len(want)], want)
                  and np.array_equal(sc.numpy()[:len(want)], scores[want])
                  and np.all(idx.numpy()[len(want):] == -1) and np.all(sc.numpy()[len(want):] == -np.inf))
            results.append((n, k, bool(ok)))
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_merged_topk_equals_whole_request():
    """One request split over two ranks: the merged local top-k lists equal the top-k of
    the whole request, ties (by lower index) and padding included."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_topk_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    out = dict(q.get(timeout=5) for _ in range(2))
    for rank in (0, 1):
        assert all(ok for _, _, ok in out[rank]), out[rank]
