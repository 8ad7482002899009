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
from transformer_candidate_scoring_b200.shard import local_requests, max_over_ranks, rank_seed, shard_bounds


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
