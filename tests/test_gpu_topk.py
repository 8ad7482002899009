"""GPU per-request top-k (tr_topk) against the oracle's top-k on the same fp32 scores:
the selected indices must match exactly (equal scores ordered by lower index), including
ties, short requests, empty requests and NaN scores."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def tr():
    import transformer_candidate_scoring_b200 as m
    return m


def _expected(scores, off, k):
    idx = np.full((len(off) - 1, k), -1, np.int64)
    val = np.full((len(off) - 1, k), -np.inf, np.float32)
    for r in range(len(off) - 1):
        s = scores[off[r]:off[r + 1]]
        t = oracle.topk(s, k)
        idx[r, :len(t)] = t
        val[r, :len(t)] = s[t]
    return idx, val


def _run(scores, off, k):
    d = torch.from_numpy(scores).cuda()
    i, v = tr().topk(d, off, k)
    torch.cuda.synchronize()
    return i.cpu().numpy(), v.cpu().numpy()


@pytest.mark.parametrize("k", [1, 7, 100, 1000, 4096])
def test_topk_matches_oracle_with_ties_and_short_requests(k):
    rng = np.random.default_rng(k)
    sizes = [0, 1, 5, max(k - 1, 0), k, k + 1, 3000, 40000]
    off = np.concatenate([[0], np.cumsum(sizes)]).tolist()
    # coarse values: many exact ties, across the whole fp32 sign range
    scores = (rng.integers(-300, 300, size=off[-1]) * 0.125).astype(np.float32)
    scores[scores == 0] = 0.0625
    got_i, got_v = _run(scores, off, k)
    ref_i, ref_v = _expected(scores, off, k)
    assert np.array_equal(got_i, ref_i)
    assert np.array_equal(got_v, ref_v)


def test_topk_continuous_scores_and_nan():
    rng = np.random.default_rng(3)
    off = [0, 20000, 20001, 60000]
    scores = rng.standard_normal(off[-1]).astype(np.float32)
    scores[[5, 100, 20000, 30000]] = np.nan
    scores[[6, 7]] = np.inf
    scores[[8, 40000]] = -np.inf
    for k in (3, 500, 4096):
        got_i, got_v = _run(scores, off, k)
        ref_i, _ = _expected(scores, off, k)
        assert np.array_equal(got_i, ref_i), k
    # a request whose only candidate is NaN still returns it
    got_i, _ = _run(scores, off, 2)
    assert got_i[1].tolist() == [0, -1]


def test_topk_of_pipeline_scores_full_size():
    """The 128D-5L request (40,000 candidates) scored on the GPU, top 2000 on the GPU vs
    the oracle's ranking of the same scores, and the scores' top-k against the fp64 oracle
    within the scoring tolerance."""
    import datagen
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    w = datagen.scaled(datagen.WORKLOADS["128d5l"], rows=200_000)
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    s = dw.scores.cpu().numpy()
    k = 2000
    got_i, _ = _run(s, dw.req_offsets, k)
    ref_i, _ = _expected(s, dw.req_offsets, k)
    assert np.array_equal(got_i, ref_i)
    # against the fp64 oracle: no candidate outside the GPU's top 50 beats one inside it by
    # more than the scoring tolerance (checked on the top 50 and a random sample of 500 others)
    rng = np.random.default_rng(0)
    top = got_i[0, :50]
    rest = rng.choice(np.setdiff1d(np.arange(dw.n_cand), got_i[0]), 500, replace=False)
    ref = oracle.score_request(w, dw.params, dw.reqs[0], cand=np.concatenate([top, rest])).scores
    tol = 2e-2 * float(np.max(np.abs(ref)))
    assert ref[:50].min() >= ref[50:].max() - tol


def test_topk_all_equal_scores_take_lowest_indices():
    """Every score equal: the threshold ties straddle the k-th place, so the index-ordered
    ranking decides (lowest indices first)."""
    off = [0, 10000, 10003]
    scores = np.full(off[-1], 1.5, np.float32)
    got_i, got_v = _run(scores, off, 100)
    assert got_i[0].tolist() == list(range(100))
    assert got_i[1].tolist() == [0, 1, 2] + [-1] * 97
    assert np.all(got_v[0] == 1.5)


def test_topk_empty_requests():
    off = [0, 0, 0]
    got_i, got_v = _run(np.zeros(1, np.float32)[:0], off, 5)
    assert np.all(got_i == -1) and np.all(np.isneginf(got_v))


@pytest.mark.gpu
@pytest.mark.parametrize("n,k,levels,cuts", [(40000, 2000, 50, [0, 19968, 40000]), (1000, 300, 4, [0, 384, 640, 1000]),
                                             (300, 500, 0, [0, 0, 300])])
def test_split_request_topk_merge_on_device(n, k, levels, cuts):
    """A request's candidates in slices (emulated ranks on one GPU): tr_topk per slice,
    indices offset, packed, then merged with tr_topk as the selection; equal to tr_topk
    over the whole request, ties and padding included."""
    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.shard import merge_gathered, pack_topk
    rng = np.random.default_rng(n + k)
    raw = rng.integers(0, levels, size=n) if levels else rng.normal(size=n)
    scores = torch.from_numpy(raw.astype(np.float32)).cuda()
    parts = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        idx = torch.full((k,), -1, dtype=torch.int64, device="cuda")
        sc = torch.full((k,), float("-inf"), dtype=torch.float32, device="cuda")
        if hi > lo:
            pi, ps = api.topk(scores[lo:hi].contiguous(), [0, hi - lo], k)
            idx = torch.where(pi[0] >= 0, pi[0] + lo, pi[0])
            sc = ps[0]
        parts.append(pack_topk(idx, sc, k))
    got_idx, got_sc = merge_gathered(parts, k)
    want_idx, want_sc = api.topk(scores, [0, n], k)
    torch.cuda.synchronize()
    assert api.sync_status() == 0
    assert torch.equal(got_idx, want_idx[0]), (got_idx[:10], want_idx[0][:10])
    assert torch.equal(got_sc, want_sc[0])
