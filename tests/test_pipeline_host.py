"""Host-side scheduling logic of the pipeline (no GPU): where the score call is split so
that the next request can start beside the score kernel's last partial round of units
(two 128-candidate tiles of one request per CTA)."""
import itertools

import numpy as np
import pytest

from transformer_candidate_scoring_b200.pipeline import SCORE_TILE, SCORE_UNIT, score_split

PER = SCORE_TILE * SCORE_UNIT


def _units(off):
    return [-(-(off[r + 1] - off[r]) // PER) for r in range(len(off) - 1)]


def _unit_index(off, c):
    """Number of units that lie wholly before packed candidate c (c on a unit boundary)."""
    t = 0
    for r in range(len(off) - 1):
        if c >= off[r + 1]:
            t += -(-(off[r + 1] - off[r]) // PER)
        elif c > off[r]:
            assert (c - off[r]) % PER == 0, "split not on a unit boundary of its request"
            t += (c - off[r]) // PER
    return t


def test_single_request_of_the_128d5l_workload():
    # 40,000 candidates = 313 tiles = 157 units = one full round of 148 + 9: the split is
    # after 148 units (296 tiles)
    assert score_split([0, 40000], 148) == 296 * 128


@pytest.mark.parametrize("off,n_sms", [([0, 296 * 128], 148), ([0, 100], 148), ([0, 295 * 128 + 5], 148),
                                       ([0, 0], 148), ([0, 40000], 0), ([0, 300, 300, 900], 5)])
def test_no_split_without_a_partial_round(off, n_sms):
    # an exact number of rounds, a single round, no candidates or no SM count: nothing to
    # split (the last case: 2 + 0 + 3 = 5 units, one round of 5)
    assert score_split(off, n_sms) is None


def test_split_at_a_request_boundary_and_inside_a_request():
    off = [300 * i for i in range(17)]             # 16 requests of 2 units (3 tiles; the last unit short)
    assert score_split(off, 7) == 4200             # 32 = 28 + 4: after request 13
    assert score_split(off, 10) == 4500            # 32 = 30 + 2: after request 14
    off = [1000 * i for i in range(4)]             # 3 requests of 4 units
    assert score_split(off, 5) == 2000 + 2 * PER   # 12 = 10 + 2: two units into request 2


def test_split_properties_over_random_batches():
    rng = np.random.default_rng(3)
    for _ in range(400):
        R = int(rng.integers(1, 12))
        sizes = rng.integers(0, 2000, size=R)
        sizes[rng.random(R) < 0.2] = 0             # some empty requests
        off = [0] + list(itertools.accumulate(int(x) for x in sizes))
        n_sms = int(rng.integers(1, 40))
        U = sum(_units(off))
        cut = score_split(off, n_sms)
        if U <= n_sms or U % n_sms == 0:
            assert cut is None
            continue
        assert cut is not None and 0 < cut < off[-1]
        a = _unit_index(off, cut)
        assert a == U - U % n_sms                  # the full rounds before the cut
        assert a % n_sms == 0


# ---------------------------------------------------------------- stream-order race check
#
# Overlapped and HostFeed.run_overlapped issue work on several CUDA streams ordered only by
# events.  The fakes below stand in for torch's streams, events and buffers and record, for
# every launch and copy, the stream it went to and the buffers it reads and writes.  The
# check then requires every pair of conflicting accesses (one of them a write) to be
# ordered on the device in the order the host issued them: by stream order, or through a
# chain of event records and waits.

class _Log:
    def __init__(self):
        self.ops = []                    # (stream, index on stream, reads, writes, label)
        self.waits = []                  # (waiting stream, index on it, recording stream, count)


class _Stream:
    _n = 0

    def __init__(self, log, *a, **k):
        self.log, self.n_ops = log, 0
        self.deps = []                   # every (stream, count) this stream has waited for
        _Stream._n += 1
        self.id = _Stream._n

    def wait_event(self, ev):
        if ev.at is None:                # never recorded: no dependency (as in torch)
            return
        # an event covers the recording stream's earlier operations and everything that
        # stream had waited for before the record (as a CUDA event does)
        for rs, count in [ev.at] + ev.deps:
            self.log.waits.append((self, self.n_ops, rs, count))
            self.deps.append((rs, count))

    def launch(self, reads, writes, label):
        self.log.ops.append((self, self.n_ops, tuple(reads), tuple(writes), label))
        self.n_ops += 1


class _Event:
    def __init__(self, *a, **k):
        self.at = None
        self.deps = []

    def record(self, stream):
        self.at = (stream, stream.n_ops)   # covers the stream's first n_ops operations
        self.deps = list(stream.deps)


class _Cuda:
    def __init__(self, log):
        self.log = log
        self.cur = [_Stream(log)]

        def make_stream(*a, **k):
            return _Stream(log)
        make_stream.priority_range = lambda: (0, -1)
        self.Stream = make_stream

    def Event(self, *a, **k):
        return _Event()

    def current_stream(self, *a):
        return self.cur[-1]

    def stream(self, s):
        cuda = self

        class _Ctx:
            def __enter__(self):
                cuda.cur.append(s)

            def __exit__(self, *exc):
                cuda.cur.pop()
        return _Ctx()

    def get_device_properties(self, dev):
        class _P:
            multi_processor_count = 148
        return _P()


class _Buf:
    def __init__(self, cuda, name, n=1):
        self.cuda, self.name, self.n = cuda, name, n
        self.dtype = "i64"

    def numel(self):
        return self.n

    def element_size(self):
        return 4

    def __getitem__(self, sl):
        return self

    def copy_(self, src, non_blocking=False):
        self.cuda.current_stream().launch([src.name], [self.name], f"copy {src.name} -> {self.name}")
        return self


class _Torch:
    def __init__(self, log):
        self.cuda = _Cuda(log)
        self._k = 0

    def empty(self, n, dtype=None, device=None):
        self._k += 1
        return _Buf(self.cuda, f"dev{self._k}", n)


class _Slot:
    """DeviceWorkload stand-in: each stage reads and writes the named buffers."""

    def __init__(self, cuda, name, n_cand):
        self.cuda, self.name, self.device = cuda, name, "cpu"
        self.req_offsets = [0, n_cand]
        self.scores = _Buf(cuda, f"{name}.scores")
        self.ub = self.tb = None

    @property
    def n_cand(self):
        return self.req_offsets[-1]

    def use_bags(self, ub, tb, reqs):
        self.ub, self.tb = ub, tb

    def _bags(self, bags):
        return [x.name for b in bags for x in (b.offsets, b.keys, b.weights, b.bag_table)]

    def user_aggregate(self, s):
        s.launch(self._bags([self.ub]), [f"{self.name}.user_tokens"], f"{self.name} user_aggregate")

    def user_prefill(self, s):
        s.launch([f"{self.name}.user_tokens"], [f"{self.name}.kv"], f"{self.name} prefill")

    def target_aggregate(self, s):
        s.launch(self._bags([self.tb]), [getattr(self, "xname", f"{self.name}.X")], f"{self.name} target_aggregate")

    def compress(self, s):
        s.launch([f"{self.name}.X"], [f"{self.name}.tokens"], f"{self.name} compress")

    def compress_range(self, c0, c1, s):
        s.launch([f"{self.name}.X"], [f"{self.name}.tokens"], f"{self.name} compress[{c0}:{c1})")

    def score(self, s):
        s.launch([f"{self.name}.tokens", f"{self.name}.kv"], [f"{self.name}.scores"], f"{self.name} score")

    def score_range(self, c0, c1, s):
        s.launch([f"{self.name}.tokens", f"{self.name}.kv"], [f"{self.name}.scores"], f"{self.name} score[{c0}:{c1})")


def _races(log):
    """Pairs of conflicting accesses that the device may run out of issue order."""
    ops = log.ops
    node = {(o[0].id, o[1]): k for k, o in enumerate(ops)}
    # happens-before: op k precedes every later op of its stream, and every op after a wait
    # that covers it
    succ = {k: set() for k in range(len(ops))}
    by_stream = {}
    for k, o in enumerate(ops):
        by_stream.setdefault(o[0].id, []).append(k)
    for ks in by_stream.values():
        for a, b in zip(ks, ks[1:]):
            succ[a].add(b)
    for s, idx, rs, count in log.waits:
        if count == 0:
            continue
        src = node[(rs.id, count - 1)]
        nxt = [k for k in by_stream.get(s.id, []) if ops[k][1] >= idx]
        if nxt:
            succ[src].add(nxt[0])

    def reach(a):
        seen, todo = set(), [a]
        while todo:
            for b in succ[todo.pop()]:
                if b not in seen:
                    seen.add(b)
                    todo.append(b)
        return seen

    after = [reach(k) for k in range(len(ops))]
    bad = []
    for a in range(len(ops)):
        for b in range(a + 1, len(ops)):
            ra, wa, rb, wb = set(ops[a][2]), set(ops[a][3]), set(ops[b][2]), set(ops[b][3])
            if (wa & (rb | wb)) or (ra & wb):
                if b not in after[a]:
                    bad.append((ops[a][4], ops[b][4]))
    return bad


@pytest.fixture
def fake_cuda(monkeypatch):
    from transformer_candidate_scoring_b200 import pipeline
    log = _Log()
    fake = _Torch(log)
    monkeypatch.setattr(pipeline, "torch", fake)
    return pipeline, fake, log


def test_race_check_detects_a_missing_wait(fake_cuda):
    # the checker itself: a consumer on another stream without the wait is a race
    pipeline, fake, log = fake_cuda
    a, b = fake.cuda.Stream(), fake.cuda.Stream()
    a.launch([], ["x"], "produce")
    b.launch(["x"], [], "consume")
    assert _races(log) == [("produce", "consume")]
    ev = fake.cuda.Event()
    ev.record(a)
    b.wait_event(ev)
    b.launch(["x"], [], "consume again")
    assert ("produce", "consume again") not in _races(log)


@pytest.mark.parametrize("n_cand,count", [(40000, 6), (1000, 5)])
def test_overlapped_steps_have_no_stream_races(fake_cuda, n_cand, count):
    pipeline, fake, log = fake_cuda
    slots = [_Slot(fake.cuda, f"slot{k}", n_cand) for k in range(2)]
    resident = [(_Bags(fake.cuda, f"set{k}.user"), _Bags(fake.cuda, f"set{k}")) for k in range(3)]   # read-only

    def bind(i, dw, main):
        dw.use_bags(*resident[i % 3], None)

    def scored(i, dw, back):
        with fake.cuda.stream(back):
            out = _Buf(fake.cuda, f"out{i}")
            out.copy_(dw.scores)

    ov = pipeline.Overlapped(slots)
    ov.run(0, count, fake.cuda.current_stream(), bind=bind, scored=scored)
    assert len(log.ops) > 5 * count
    assert _races(log) == []


def _Bags(cuda, name):
    from transformer_candidate_scoring_b200.pipeline import DeviceBags
    return DeviceBags(*(_Buf(cuda, f"{name}.{f}") for f in ("offsets", "keys", "weights", "bag_table")))


def test_host_feed_overlapped_has_no_stream_races(fake_cuda):
    pipeline, fake, log = fake_cuda
    slots = [_Slot(fake.cuda, f"slot{k}", 40000) for k in range(2)]
    batches = [(_Bags(fake.cuda, f"host{k}.user"), _Bags(fake.cuda, f"host{k}.target"), None) for k in range(3)]
    feed = pipeline.HostFeed(slots[0], batches)
    ov = pipeline.Overlapped(slots)
    host_scores = [_Buf(fake.cuda, f"host_scores{k}") for k in range(2)]
    feed.run_overlapped(ov, 0, 7, host_scores, fake.cuda.current_stream())
    labels = [o[4] for o in log.ops]
    assert sum(l.startswith("copy host") for l in labels) == 7 * 8      # 2 bags x 4 arrays per batch
    assert sum("-> host_scores" in l for l in labels) == 7
    assert _races(log) == []


# ---------------------------------------------------------------- range calls (host marshalling)

def _range_workload(sizes, L_u, D=4):
    """A DeviceWorkload's request bookkeeping on CPU tensors (no model, no GPU)."""
    import torch
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload
    dw = object.__new__(DeviceWorkload)
    off = [0]
    for n in sizes:
        off.append(off[-1] + n)
    dw.req_offsets = off
    dw.L_u = list(L_u)
    dw.domain = [r % 3 for r in range(len(sizes))]
    dw.kv = [torch.full((16,), r, dtype=torch.uint8) for r in range(len(sizes))]
    dw.model = "model"
    n = off[-1]
    dw.tokens = torch.arange(n * D, dtype=torch.float32).view(n, D)
    dw.X = torch.arange(n * 2 * D, dtype=torch.float32).view(n, 2 * D)
    dw.scores = torch.zeros(n)
    return dw


def test_score_range_slices_requests_and_keeps_their_caches(monkeypatch):
    from transformer_candidate_scoring_b200 import pipeline
    calls = []
    monkeypatch.setattr(pipeline.api, "score_candidates",
                        lambda model, tokens, off, kv, lu, dm, scores, stream=None:
                        calls.append((tokens, list(off), [int(k[0]) for k in kv], list(lu), list(dm), scores)))
    dw = _range_workload([300, 0, 500, 200], [64, 10, 128, 32])
    cut = 300 + 128                               # one tile into request 2
    dw.score_range(0, cut, "s")
    dw.score_range(cut, dw.n_cand, "s")
    (t0, off0, kv0, lu0, dm0, s0), (t1, off1, kv1, lu1, dm1, s1) = calls
    # head: request 0 whole, the empty request 1 dropped, the first 128 of request 2
    assert off0 == [0, 300, 428] and kv0 == [0, 2] and lu0 == [64, 128] and dm0 == [0, 2]
    # tail: the rest of request 2 and request 3, offsets rebased to the range
    assert off1 == [0, 372, 572] and kv1 == [2, 3] and lu1 == [128, 32] and dm1 == [2, 0]
    # the token and score views start at the cut and cover the range
    assert t0.shape[0] == cut and t1.shape[0] == dw.n_cand - cut
    assert t1.data_ptr() == dw.tokens[cut:].data_ptr() and s1.data_ptr() == dw.scores[cut:].data_ptr()
    # a range with no candidates makes no call
    dw.score_range(300, 300, "s")
    assert len(calls) == 2


def test_compress_range_passes_row_views(monkeypatch):
    from transformer_candidate_scoring_b200 import pipeline
    calls = []
    monkeypatch.setattr(pipeline.api, "compress_targets",
                        lambda model, x, tokens, stream=None: calls.append((x, tokens)))
    dw = _range_workload([300, 500], [64, 64])
    dw.compress_range(0, 512, None)
    dw.compress_range(512, 800, None)
    dw.compress_range(800, 800, None)           # empty: no call
    assert len(calls) == 2
    (x0, t0), (x1, t1) = calls
    assert x0.shape[0] == 512 and x1.shape[0] == 288
    assert x1.data_ptr() == dw.X[512:].data_ptr() and t1.data_ptr() == dw.tokens[512:].data_ptr()


# ---------------------------------------------------------------- the candidate stream (Streamed)

def _check_plan(plan, n, count, first, n_slots, comp_chunk, bounds, score_units, group=1):
    """Every candidate is gathered, compressed and scored once, in that order, each before
    its ring slot is gathered over; launches have their full size except where a ring wrap,
    a slot reuse or the end of the run cuts them; score launches end on unit ends."""
    ring = n_slots * n
    base = first * n
    ends = {j * n + b for j in range(count) for b in bounds}      # unit ends of the stream
    gathered, comp, score = -1, 0, 0
    wraps = {w - base for w in range(ring, base + count * n + ring, ring)}
    for step in plan:
        if step[0] == "gather":
            j = step[1]
            assert j == gathered + 1
            gathered = j
            assert comp >= (j - n_slots + 1) * n and score >= (j - n_slots + 1) * n   # slot j - n_slots is done
            continue
        kind, a, b = step
        assert b > a
        assert not any(a < w < b for w in wraps)                 # never across the ring's end
        cut = b in wraps or b == count * n or b % n == 0
        if kind == "compress":
            assert a == comp and b <= (gathered + 1) * n
            assert b - a == comp_chunk or cut
            comp = b
        else:
            assert a == score and b <= comp and b in ends
            units = sum(1 for e in ends if a < e <= b)
            assert units == score_units or (units < score_units and cut)
            score = b
    assert gathered == count - 1 and comp == score == count * n


@pytest.mark.parametrize("group", [1, 2, 3])
@pytest.mark.parametrize("n,count,first,n_slots,comp_chunk,units", [
    (40000, 12, 3, 64, 294 * 128, 148),      # the 128D-5L batch: no wrap inside the run
    (40000, 12, 3, 4, 294 * 128, 148),       # wraps every four batches
    (300, 9, 0, 2, 1000, 3),                 # chunks longer than a batch: slot reuse forces flushes
    (1000, 7, 5, 3, 384, 5),
])
def test_stream_plan_covers_every_candidate_once(n, count, first, n_slots, comp_chunk, units, group):
    from transformer_candidate_scoring_b200.pipeline import stream_plan, unit_bounds
    bounds = unit_bounds([0, n])
    plan = stream_plan(n, count, first, n_slots, comp_chunk, bounds, units, group)
    _check_plan(plan, n, count, first, n_slots, comp_chunk, bounds, units)
    if group > 1:                             # compute launches only after every group-th gather
        last_gather = -1
        for step in plan:
            if step[0] == "gather":
                last_gather = step[1]
            elif last_gather + 1 < count and (last_gather + 1) % group:
                assert step[2] <= (last_gather + 1) * n and any(
                    s[0] == "gather" and s[1] == last_gather + 1 for s in plan)   # a forced flush


def test_stream_plan_packed_batches_and_steady_state():
    from transformer_candidate_scoring_b200.pipeline import stream_plan, unit_bounds
    rng = np.random.default_rng(3)
    for _ in range(30):
        sizes = rng.integers(1, 700, size=rng.integers(1, 6))
        off = np.concatenate([[0], np.cumsum(sizes)]).tolist()
        n = off[-1]
        bounds = unit_bounds(off)
        assert bounds[-1] == n and sorted(bounds) == bounds
        count, first, n_slots = int(rng.integers(1, 9)), int(rng.integers(0, 5)), int(rng.integers(2, 6))
        comp_chunk, units = int(rng.integers(1, 2000)), int(rng.integers(1, 12))
        plan = stream_plan(n, count, first, n_slots, comp_chunk, bounds, units, int(rng.integers(1, 4)))
        _check_plan(plan, n, count, first, n_slots, comp_chunk, bounds, units)
    # the 128D-5L batch in steady state: every launch between the first and the last two is
    # full size (294 compressor tiles, 148 score units)
    bounds = unit_bounds([0, 40000])
    plan = stream_plan(40000, 20, 0, 64, 294 * 128, bounds, 148)
    comp = [b - a for k, a, b in (s for s in plan if s[0] == "compress")]
    assert all(c == 294 * 128 for c in comp[:-1])
    score = [(a, b) for k, a, b in (s for s in plan if s[0] == "score")]
    for a, b in score[:-1]:
        assert sum(1 for j in range(20) for e in bounds if a < j * 40000 + e <= b) == 148


class _RingView:
    def __init__(self, names):
        self.names = names
        self.name = "+".join(names)


class _Ring(_Buf):
    """A ring of m slots of n rows: a row range names the slots it touches (ring.X#k), so
    that the race check sees which batches a launch reads or writes."""

    def __init__(self, cuda, name, n, m):
        super().__init__(cuda, name)
        self.rows, self.m = n, m

    def slot(self, k):
        return _Buf(self.cuda, f"{self.name}#{k % self.m}")

    def __getitem__(self, sl):
        a, b = sl.start, sl.stop
        return _RingView([f"{self.name}#{k % self.m}" for k in range(a // self.rows, (b - 1) // self.rows + 1)])


def _names(x):
    return list(getattr(x, "names", [x.name]))


def _stream_slot(cuda, name, n_cand, k=None, ring=None):
    s = _Slot(cuda, name, n_cand)
    s.L_u, s.domain = [64], [1]
    s.kv = [_Buf(cuda, f"{name}.kv")]
    s.model = "model"
    if ring is not None:   # a Streamed slot: its X, tokens and scores are rows of the rings
        s.xname = ring[0].slot(k).name
        s.scores = ring[2].slot(k)
    return s


def _streamed(pipeline, cuda, n_cand, n_slots):
    st = object.__new__(pipeline.Streamed)
    st.n = n_cand
    st.X, st.tokens, st.scores = (_Ring(cuda, "ring.X", n_cand, n_slots), _Ring(cuda, "ring.tokens", n_cand, n_slots),
                                  _Ring(cuda, "ring.scores", n_cand, n_slots))
    st.slots = [_stream_slot(cuda, f"slot{k}", n_cand, k, (st.X, st.tokens, st.scores)) for k in range(n_slots)]
    st.user = cuda.Stream()
    return st


class _FakeApi:
    def __init__(self, cuda):
        self.cuda = cuda

    def compress_targets(self, model, x, tokens, stream=None):
        stream.launch(_names(x), _names(tokens), f"compress {_names(x)}")

    def score_candidates(self, model, tokens, off, kv, lu, dm, scores, stream=None):
        stream.launch(_names(tokens) + [k.name for k in kv], _names(scores), f"score {[k.name for k in kv]}")

    def kernel_launches(self):
        return 0


@pytest.mark.parametrize("n_cand,count,n_slots,group", [(40000, 9, 4, 1), (300, 8, 3, 1), (40000, 9, 4, 2),
                                                        (300, 8, 3, 3)])
def test_streamed_steps_have_no_stream_races(fake_cuda, monkeypatch, n_cand, count, n_slots, group):
    from transformer_candidate_scoring_b200.pipeline import unit_bounds
    pipeline, fake, log = fake_cuda
    monkeypatch.setattr(pipeline, "api", _FakeApi(fake.cuda))
    st = _streamed(pipeline, fake.cuda, n_cand, n_slots)
    st.comp_chunk, st.score_units, st.bounds = 294 * 128 if n_cand > 1000 else 500, 148 if n_cand > 1000 else 2, \
        unit_bounds([0, n_cand])
    st.group = group
    resident = [(_Bags(fake.cuda, f"set{k}.user"), _Bags(fake.cuda, f"set{k}")) for k in range(3)]
    done = []

    def bind(i, dw, main):
        dw.use_bags(*resident[i % 3], None)

    def scored(i, dw, s):
        done.append(i)
        out = _Buf(fake.cuda, f"out{i}")
        with fake.cuda.stream(s):
            out.copy_(dw.scores)

    st.run(2, count, fake.cuda.current_stream(), bind=bind, scored=scored)
    assert done == list(range(2, 2 + count))
    assert _races(log) == []


@pytest.mark.parametrize("n_bag_slots", [2, 3])
def test_host_feed_streamed_has_no_stream_races(fake_cuda, monkeypatch, n_bag_slots):
    from transformer_candidate_scoring_b200.pipeline import unit_bounds
    pipeline, fake, log = fake_cuda
    monkeypatch.setattr(pipeline, "api", _FakeApi(fake.cuda))
    st = _streamed(pipeline, fake.cuda, 40000, 4)
    st.comp_chunk, st.score_units, st.bounds = 294 * 128, 148, unit_bounds([0, 40000])
    st.group = 2
    batches = [(_Bags(fake.cuda, f"host{k}.user"), _Bags(fake.cuda, f"host{k}.target"), None) for k in range(3)]
    feed = pipeline.HostFeed(st.slots[0], batches, n_bag_slots=n_bag_slots)
    host_scores = [_Buf(fake.cuda, f"host_scores{k}") for k in range(2)]
    feed.run_overlapped(st, 0, 9, host_scores, fake.cuda.current_stream())
    labels = [o[4] for o in log.ops]
    assert sum(l.startswith("copy host") for l in labels) == 9 * 8
    assert sum("-> host_scores" in l for l in labels) == 9
    assert _races(log) == []


def test_launch_sizes_are_whole_rounds():
    from transformer_candidate_scoring_b200.pipeline import SCORE_TILE, launch_sizes, unit_bounds
    units = len(unit_bounds([0, 40000]))          # 313 tiles: 156 pairs and one single
    assert units == 157
    # the 128D-5L batch on 148 SMs: groups of four give eight compressor rounds (one tile per
    # SM on 147 SMs each), four score rounds
    assert launch_sizes(40000, units, 148, 4) == (8 * 147 * SCORE_TILE, 4 * 148)
    assert launch_sizes(40000, units, 148, 2) == (4 * 147 * SCORE_TILE, 2 * 148)
    assert launch_sizes(40000, units, 148, 1) == (2 * 147 * SCORE_TILE, 1 * 148)
    # small batches still take one whole round
    assert launch_sizes(300, 2, 148, 4) == (2 * 147 * SCORE_TILE, 148)
    for n, u, sms, g in [(65536, 256, 148, 4), (520000, 2032, 148, 4), (1000, 4, 8, 3)]:
        c, s = launch_sizes(n, u, sms, g)
        assert c % (2 * (sms - 1) * SCORE_TILE) == 0 and c >= 2 * (sms - 1) * SCORE_TILE
        assert s % sms == 0 and s >= sms
        assert c <= max(g * n, 2 * (sms - 1) * SCORE_TILE) and s <= max(g * u, sms)
