"""Device-resident workload and the whole scoring step through the C ABI.

One step of TransRetrieval candidate scoring (§3.1 stages (1)-(4) and the head):
  per request: tr_aggregate(user fields) -> tr_prefill_user (K/V cache)
  all requests packed: tr_aggregate(target fields) -> tr_compress_targets -> tr_score_candidates
Inputs come from ``datagen`` (seeded synthetic tables and bags); tables are filled on the
device by datagen's counter-based generator.
"""
from __future__ import annotations

import bisect
import copy
import math
from dataclasses import dataclass
from typing import List

import numpy as np
import torch

import datagen

from . import api


def _dev(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


@dataclass
class DeviceBags:
    offsets: torch.Tensor
    keys: torch.Tensor
    weights: torch.Tensor
    bag_table: torch.Tensor

    @staticmethod
    def of(b: "datagen.Bags", device) -> "DeviceBags":
        return DeviceBags(_dev(b.offsets.astype(np.int64), device), _dev(b.keys.astype(np.int32), device),
                          _dev(b.weights.astype(np.float32), device), _dev(b.bag_table.astype(np.int32), device))


def _pack(bag_sets) -> "datagen.Bags":
    offs, keys, wts, tabs = [np.zeros(1, np.int64)], [], [], []
    base = 0
    for b in bag_sets:
        offs.append(b.offsets[1:] + base)
        base += b.nnz
        keys.append(b.keys)
        wts.append(b.weights)
        tabs.append(b.bag_table)
    return datagen.Bags(np.concatenate(offs), np.concatenate(keys), np.concatenate(wts), np.concatenate(tabs))


def pack_target_bags(reqs: List["datagen.Request"]) -> "datagen.Bags":
    """Every request's target bags, one after the other (candidate order)."""
    return _pack([r.target for r in reqs])


def pack_user_bags(reqs: List["datagen.Request"]) -> "datagen.Bags":
    """Every request's user-field bags, one after the other (request r's fields follow those
    of requests 0 .. r-1)."""
    return _pack([r.user for r in reqs])


class DeviceWorkload:
    """Tables, model, bags and activation buffers of a workload on one GPU."""

    def __init__(self, w: "datagen.Workload", device="cuda", reqs=None, params=None, tables=None):
        self.w = w
        self.device = torch.device(device)
        dims = w.dims
        self.dt = api.torch_dtype(dims.dtype)
        self.params = params if params is not None else datagen.workload_params(w)
        self.model = api.Model(dims, self.params)
        if tables is None:
            tables = self.make_tables(w, self.device)
        self.user_tables, self.target_tables = tables
        self.reqs = reqs if reqs is not None else datagen.make_requests(w)
        self.set_requests(self.reqs)

    @staticmethod
    def make_tables(w, device):
        dt = api.torch_dtype(w.dims.dtype)
        D = w.dims.D
        ut, tt = [], []
        for t in range(w.user_tables):
            x = torch.empty(w.user_rows, D, dtype=dt, device=device)
            datagen.fill_table_device(x, w.seed, datagen.user_table_id(w, t))
            ut.append(x)
        for t, rows in enumerate(w.target_rows):
            x = torch.empty(rows, D, dtype=dt, device=device)
            datagen.fill_table_device(x, w.seed, datagen.target_table_id(w, t))
            tt.append(x)
        return ut, tt

    def set_requests(self, reqs) -> None:
        w, dims, dev = self.w, self.w.dims, self.device
        self.reqs = reqs
        self.user_bags = DeviceBags.of(pack_user_bags(reqs), dev)
        self.target_bags = DeviceBags.of(pack_target_bags(reqs), dev)
        self.L_u = [r.L_u for r in reqs]
        self.domain = [r.domain for r in reqs]
        off = [0]
        for r in reqs:
            off.append(off[-1] + r.n_cand)
        self.req_offsets = off
        n = off[-1]
        D, F = dims.D, dims.n_target_fields
        self._user_buffers()
        self.X = torch.empty(n, F * D, dtype=self.dt, device=dev)
        self.tokens = torch.empty(n, D, dtype=torch.float32, device=dev)     # compressed tokens (fp32)
        self.scores = torch.empty(n, dtype=torch.float32, device=dev)

    def _user_buffers(self) -> None:
        """Every request's user tokens in one buffer (one aggregation call fills them all)
        and its K/V cache."""
        D, dev = self.w.dims.D, self.device
        uoff = np.concatenate([[0], np.cumsum(self.L_u)]).astype(int)
        self.user_tokens_all = torch.empty(max(int(uoff[-1]), 1), D, dtype=torch.float32, device=dev)
        self.user_tokens = [self.user_tokens_all[uoff[r]:uoff[r] + max(l, 1)] if l else self.user_tokens_all[:1]
                            for r, l in enumerate(self.L_u)]
        self.n_user = int(uoff[-1])
        self.kv = [torch.empty(max(api.kv_cache_bytes(self.model, l), 16), dtype=torch.uint8, device=dev)
                   for l in self.L_u]

    def clone_slot(self, activations: bool = True) -> "DeviceWorkload":
        """Another slot of the same workload: shares the model, tables and current bags,
        owns its user tokens and K/V caches (and, unless ``activations`` is False, its X,
        tokens and scores)."""
        c = copy.copy(self)
        c._user_buffers()
        if activations:
            c.X, c.tokens, c.scores = (torch.empty_like(self.X), torch.empty_like(self.tokens),
                                       torch.empty_like(self.scores))
        return c

    @property
    def n_cand(self) -> int:
        return self.req_offsets[-1]

    def use_bags(self, user_bags, target_bags, reqs) -> None:
        """Point the next step at other device bags of requests with the same L_u and
        candidate counts as the current ones (no reallocation of activations)."""
        if [r.L_u for r in reqs] != self.L_u or [r.n_cand for r in reqs] != [r.n_cand for r in self.reqs]:
            raise ValueError("use_bags: requests differ in L_u or candidate count; call set_requests")
        self.user_bags, self.target_bags, self.reqs = user_bags, target_bags, reqs
        self.domain = [r.domain for r in reqs]

    # -------------------------------------------------------------- the step
    def user_aggregate(self, stream=None) -> None:
        """Every request's user fields in one tr_aggregate call."""
        if self.n_user:
            b = self.user_bags
            api.aggregate(self.user_tables, b.bag_table, b.offsets, b.keys, b.weights,
                          self.user_tokens_all[:self.n_user], stream=stream)

    def user_prefill(self, stream=None) -> None:
        """Every request's user side in one tr_prefill_users call."""
        if self.n_user:
            api.prefill_users(self.model, self.user_tokens, self.L_u, self.domain, self.kv, stream=stream)

    def user_side(self, stream=None) -> None:
        self.user_aggregate(stream)
        self.user_prefill(stream)

    def target_aggregate(self, stream=None) -> None:
        b = self.target_bags
        api.aggregate(self.target_tables, b.bag_table, b.offsets, b.keys, b.weights,
                      self.X.view(-1, self.w.dims.D), stream=stream)

    def compress(self, stream=None) -> None:
        api.compress_targets(self.model, self.X, self.tokens, stream=stream)

    def compress_range(self, c0: int, c1: int, stream=None) -> None:
        """tr_compress_targets over the packed candidates [c0, c1) only (rows are independent)."""
        if c1 > c0:
            api.compress_targets(self.model, self.X[c0:c1], self.tokens[c0:c1], stream=stream)

    def score(self, stream=None) -> None:
        api.score_candidates(self.model, self.tokens, self.req_offsets, self.kv, self.L_u, self.domain,
                             self.scores, stream=stream)

    def score_range(self, c0: int, c1: int, stream=None) -> None:
        """tr_score_candidates over the packed candidates [c0, c1) only: each request's share
        of the range keeps its K/V cache, L_u and domain.  A candidate's score depends on
        its own token and its request's cache alone, so scoring a batch in two ranges gives
        the same scores as one call."""
        off, kv, lu, dm = [0], [], [], []
        for r in range(len(self.L_u)):
            lo, hi = max(self.req_offsets[r], c0), min(self.req_offsets[r + 1], c1)
            if hi <= lo:
                continue
            off.append(off[-1] + hi - lo)
            kv.append(self.kv[r])
            lu.append(self.L_u[r])
            dm.append(self.domain[r])
        if len(off) > 1:
            api.score_candidates(self.model, self.tokens[c0:c1], off, kv, lu, dm, self.scores[c0:c1],
                                 stream=stream)

    def select(self, k: int, stream=None):
        """Per-request top-k of the last step's scores (tr_topk): (indices within each
        request [R, k] int64, scores [R, k] fp32), padded with -1 / -inf."""
        if not hasattr(self, "_sel") or self._sel[0].shape != (len(self.reqs), k):
            self._sel = (torch.empty(len(self.reqs), k, dtype=torch.int64, device=self.device),
                         torch.empty(len(self.reqs), k, dtype=torch.float32, device=self.device))
        return api.topk(self.scores, self.req_offsets, k, self._sel[0], self._sel[1], stream=stream)

    def capture_stream(self) -> "torch.cuda.Stream":
        """The stream this workload captures graphs on (created once)."""
        if not hasattr(self, "_cap"):
            self._cap = torch.cuda.Stream(self.device)
        return self._cap

    def capture_step(self, stream=None) -> "torch.cuda.CUDAGraph":
        """One step with the current bags, captured into a CUDA graph (replay it to run the
        step again without host launch overhead; the bags, caches and activations it reads
        and writes are the ones bound now).  The first capture on a stream runs the step
        once eagerly on it: the library sets up per-device state and, for its CUDA-core
        kernels, per-stream scratch on first use, which a capture does not allow."""
        cap = stream if stream is not None else self.capture_stream()
        warm_up_stream(cap, lambda: self.step(cap))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            self.step()
        return g

    def step(self, stream=None, events=None) -> torch.Tensor:
        """One request batch.  The user aggregation (a few small launches) runs first on the
        caller's stream; then the user prefill (one CTA per request, which needs a whole SM)
        runs on a high-priority side stream while the target aggregation and compression run
        on the caller's stream.  Both become ready together, so the prefill CTAs are placed
        before the gather fills the SMs, and the prefill ends before the compressor needs
        every SM.  The scoring waits for both.  ``events``: optional dict of CUDA events
        recorded at stage boundaries (keys user0, user1 on the side stream; t0, agg, comp, s0,
        score on the main)."""
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        if not hasattr(self, "_side"):
            lo, hi = torch.cuda.Stream.priority_range()
            self._side = torch.cuda.Stream(self.device, priority=hi)
        side = self._side
        if events:
            events["user0"].record(main)
        self.user_aggregate(main)
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        self.user_prefill(side)
        if events:
            events["user1"].record(side)
        join = torch.cuda.Event()
        join.record(side)
        if events:
            events["t0"].record(main)
        self.target_aggregate(main)
        if events:
            events["agg"].record(main)
        self.compress(main)
        if events:
            events["comp"].record(main)
        main.wait_event(join)
        if events:
            events["s0"].record(main)
        self.score(main)
        if events:
            events["score"].record(main)
        return self.scores


_WARM_STREAMS = set()


def warm_up_stream(stream, run) -> None:
    """Runs ``run()`` eagerly once per stream (then waits for it), before the first capture
    on that stream."""
    key = (stream.device.index, int(stream.cuda_stream))
    if key in _WARM_STREAMS:
        return
    run()
    stream.synchronize()
    _WARM_STREAMS.add(key)


SCORE_TILE = 128   # candidates per tile of the tensor-core score kernel
SCORE_UNIT = 2     # tiles of one request that a CTA of the score kernel holds at a time


def score_split(req_offsets, n_sms: int, tile: int = SCORE_TILE, unit: int = SCORE_UNIT):
    """The packed candidate index at which the score kernel's last, partial round of work
    begins, or None when it has none.  The kernel cuts every request into tiles of ``tile``
    candidates and groups a request's tiles into units of ``unit`` consecutive tiles (its last
    unit may be shorter), in request order; one persistent CTA per SM takes units b,
    b + n_sms, b + 2 n_sms, ...  With U units and U mod n_sms = u > 0 (and more than one
    round), the last u units form a round of their own on u SMs while the other SMs wait.
    The split index lies on a unit boundary of its request.  Both parts are valid batches
    and the scores do not change."""
    per = tile * unit
    units = [-(-(req_offsets[r + 1] - req_offsets[r]) // per) for r in range(len(req_offsets) - 1)]
    U = sum(units)
    if n_sms <= 0 or U <= n_sms or U % n_sms == 0:
        return None
    cut = U - U % n_sms
    acc = 0
    for r, u in enumerate(units):
        if acc + u == cut:
            return req_offsets[r + 1]
        if acc + u > cut:
            return req_offsets[r] + (cut - acc) * per
        acc += u
    return None


class Overlapped:
    """Request batches scored back to back, consecutive batches overlapped on the device.

    The compressor and the score kernel both run one persistent CTA per SM over the batch
    (the compressor one 128-candidate tile at a time, the score kernel two), so a batch whose
    work is not a multiple of the SM count ends each of them with a partial round that leaves
    most SMs idle.  Here a batch is cut at score_split into a head (the full rounds of the
    score kernel) and a tail:
      main stream  user aggregation -> target aggregation -> compress(head) -> score(head)
      user stream  (high priority) user prefill, joined before score(head)
      back stream  (high priority) compress(tail) -> score(tail), after score(head)
    The next batch follows score(head) on the main stream, so the tail's compression and
    scoring (one partial wave of each, on a few SMs) run beside the next batch's gather.
    The back stream's priority places the tail's CTAs, which need whole SMs, before the
    gather's many small blocks fill them.

    Batches alternate between two DeviceWorkload slots (activations, caches and scores);
    batch i + 2 reuses slot i % 2 only after batch i's tail has finished (an event the main
    stream waits for, long satisfied by then).  Scores are identical to those of
    DeviceWorkload.step.
    """

    def __init__(self, slots: List[DeviceWorkload]):
        if len(slots) != 2:
            raise ValueError("Overlapped needs two DeviceWorkload slots")
        self.slots = slots
        dev = slots[0].device
        _, hi = torch.cuda.Stream.priority_range()
        self.user = torch.cuda.Stream(dev, priority=hi)
        self.back = torch.cuda.Stream(dev, priority=hi)
        self.cap = torch.cuda.Stream(dev)
        self.n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.launches_per_step = None

    def run(self, first: int, count: int, stream=None, bind=None, fronted=None, scored=None) -> None:
        """Batches first .. first + count - 1 on ``stream`` (the caller's), which waits for
        all of them at the end.  Hooks, each given (i, slot, stream):
          bind(i, dw, main)     before batch i's first launch (point ``dw`` at its bags);
          fronted(i, dw, main)  after its target aggregation (its bags are no longer read);
          scored(i, dw, s)      after its last score launch, on that launch's stream; it may
                                return a CUDA event, and ``dw.scores`` is not written again
                                before that event.
        ``first``/``count`` only name the batches for the hooks and pick slot i % 2."""
        main = stream if stream is not None else torch.cuda.current_stream(self.slots[0].device)
        start = torch.cuda.Event()
        start.record(main)
        self.back.wait_event(start)
        self.user.wait_event(start)
        tails = {}                                  # batch -> event: its tail launches are done
        released = {}                               # batch -> event from the scored hook
        for i in range(first, first + count):
            dw = self.slots[i % 2]
            if i - 2 in tails:                      # the slot's previous batch has finished
                main.wait_event(tails.pop(i - 2))
            if released.get(i - 2) is not None:     # ... and its scores have been read
                main.wait_event(released.pop(i - 2))
            if bind is not None:
                bind(i, dw, main)
            dw.user_aggregate(main)
            fork = torch.cuda.Event()
            fork.record(main)
            self.user.wait_event(fork)
            dw.user_prefill(self.user)
            join = torch.cuda.Event()
            join.record(self.user)
            dw.target_aggregate(main)
            if fronted is not None:
                fronted(i, dw, main)
            n = dw.n_cand
            cut = score_split(dw.req_offsets, self.n_sms)
            head = n if cut is None else cut
            dw.compress_range(0, head, main)
            main.wait_event(join)
            if cut is None:
                dw.score(main)
                if scored is not None:
                    released[i] = scored(i, dw, main)
                continue
            dw.score_range(0, cut, main)
            full = torch.cuda.Event()
            full.record(main)
            self.back.wait_event(full)
            dw.compress_range(cut, n, self.back)
            dw.score_range(cut, n, self.back)
            if scored is not None:
                released[i] = scored(i, dw, self.back)
            tails[i] = torch.cuda.Event()
            tails[i].record(self.back)
        for ev in tails.values():
            main.wait_event(ev)
        for ev in released.values():
            if ev is not None:
                main.wait_event(ev)

    def capture(self, first: int, count: int, **hooks) -> "torch.cuda.CUDAGraph":
        """run(first, count, ...) captured into one CUDA graph (replay it to run the same
        batches again; the overlap holds between the captured batches, not across replays).
        The first capture runs the batches once eagerly on the capture stream: the library
        sets up per-device state and per-stream scratch on first use, which capture does
        not allow."""
        g = torch.cuda.CUDAGraph()
        cap = self.cap
        warm_up_stream(cap, lambda: self.run(first, count, cap, **hooks))
        l0 = api.kernel_launches()
        with torch.cuda.graph(g, stream=cap):
            self.run(first, count, cap, **hooks)
        self.launches_per_step = (api.kernel_launches() - l0) / max(count, 1)
        return g


def unit_bounds(req_offsets, tile: int = SCORE_TILE, unit: int = SCORE_UNIT) -> List[int]:
    """End offsets (within a batch) of the score kernel's units: every request is cut into
    runs of ``unit`` tiles of ``tile`` candidates from its own start, the last one shorter."""
    out = []
    per = tile * unit
    for r in range(len(req_offsets) - 1):
        s, e = req_offsets[r], req_offsets[r + 1]
        out.extend(range(s + per, e, per))
        if e > s:
            out.append(e)
    return out


def launch_sizes(n: int, units_per_batch: int, sms: int, group: int):
    """Default launch sizes of Streamed: (candidates per compress launch, score-kernel units
    per score launch), each as many whole rounds as the ``group`` batches between two launch
    points fill, at least one.  The compressor's unit is two rounds, two 128-candidate tiles
    on each SM but one (the prefill CTA's); the score kernel's is one round, one unit on
    every SM.  A launch has a fixed
    cost (~7 us of ramp for the score kernel), so the stream takes a few large launches
    rather than many one-round ones: at 40,000 candidates a batch and group 4, eight rounds
    of compressor tiles and four of score units; a batch's scores then complete up to four
    batches after its gather."""
    comp_round = 2 * (sms - 1) * SCORE_TILE
    return comp_round * max(1, group * n // comp_round), sms * max(1, group * units_per_batch // sms)


def stream_plan(n: int, count: int, first: int, n_slots: int, comp_chunk: int, bounds: List[int],
                score_units: int, group: int = 1):
    """The launch order of Streamed.run over batches first .. first + count - 1 of n
    candidates each: a list of ("gather", j), ("compress", a, b) and ("score", a, b) with
    candidate positions a, b counted from the start of batch ``first`` (batch j covers
    [j n, (j + 1) n)).  A compress launch takes ``comp_chunk`` candidates of the stream and a
    score launch ``score_units`` of the score kernel's units (``bounds``: their end offsets
    within a batch, unit_bounds), both across batch boundaries.  A launch is shorter only
    where it meets the end of the activation ring (n_slots batches, batch i in slot
    i mod n_slots), the end of the run, or a slot that the next batch is about to reuse
    (everything of batch j - n_slots is compressed and scored before batch j is gathered).
    With ``group`` > 1, compress and score launches are issued only after every group-th
    gather, so that launches of one kernel follow each other (a kernel that follows another
    kind of kernel starts with cold instruction and data caches)."""
    if n <= 0 or count <= 0:
        return []
    ring = n_slots * n
    base = first * n                          # absolute stream position of the run's start
    K = len(bounds)

    def wrap_end(a):
        return ((base + a) // ring + 1) * ring - base

    def unit_end(a, units):                   # the position `units` unit ends after a
        j = a // n
        t = j * K + bisect.bisect_right(bounds, a - j * n) + units
        return (t // K) * n + (bounds[t % K - 1] if t % K else 0)

    def step_end(kind, done):
        return done + comp_chunk if kind == "compress" else unit_end(done, score_units)

    def full(done, limit, kind, out):
        while True:
            e = min(step_end(kind, done), wrap_end(done))
            if e > limit:
                return done
            out.append((kind, done, e))
            done = e

    def flush(done, target, kind, out):
        while done < target:
            e = min(step_end(kind, done), wrap_end(done), target)
            out.append((kind, done, e))
            done = e
        return done

    plan = []
    comp = score = 0
    for j in range(count):
        need = (j - n_slots + 1) * n          # batch j - n_slots leaves its slot
        if need > 0:
            comp = flush(comp, need, "compress", plan)
            score = flush(score, need, "score", plan)
        plan.append(("gather", j))
        if (j + 1) % group and j + 1 < count:
            continue
        comp = full(comp, (j + 1) * n, "compress", plan)
        score = full(score, comp, "score", plan)
    comp = flush(comp, count * n, "compress", plan)
    flush(score, count * n, "score", plan)
    return plan


class Streamed:
    """Request batches scored as one stream of candidate tiles.

    Overlapped cuts every batch at the score kernel's last partial round and runs the tail
    beside the next batch.  Here the compressor and the score kernel instead take
    fixed-size chunks of one stream of candidates that runs across batch boundaries
    (stream_plan): by default every compress launch is a whole number of rounds (two
    128-candidate tiles per SM on the SMs left beside one prefill CTA) and every score
    launch a whole number of rounds of the score kernel's two-tile units on all SMs, as many
    as the batches between two launch points fill,
    whichever batches the chunk falls in.  A launch that spans two batches scores
    each candidate against its own request's cache (the kernels take a list of requests).
      main stream  target aggregation of batch i, then every compress and score chunk that
                   has become complete (a score chunk after the prefills of the batches it
                   covers)
      user stream  (high priority) user aggregation and prefill of batch i, once batch
                   i - n_slots (the same slot's previous batch) has been scored
    The slots are clones of one DeviceWorkload (DeviceWorkload.clone_slot) whose X, tokens
    and scores are views of ring buffers laid out slot after slot, so that a chunk spanning
    consecutive batches is one contiguous range; by default the ring takes up to 64 batches
    within ``ring_bytes``, so its wrap (where one compress and one score launch are cut
    short) comes rarely.  Scores are identical to those of DeviceWorkload.step.
    """

    def __init__(self, dw: DeviceWorkload, n_slots: int = None, comp_chunk: int = None, score_units: int = None,
                 ring_bytes: int = 8 << 30, group: int = 4):
        n = dw.n_cand
        dims = dw.w.dims
        F, D = dims.n_target_fields, dims.D
        per_batch = n * (F * D * dw.X.element_size() + 4 * D + 4)
        if n_slots is None:                   # a ring wrap costs one partial round of each kernel
            n_slots = int(max(4, min(64, ring_bytes // max(per_batch, 1))))
        if n_slots < 2:
            raise ValueError("Streamed needs at least two slots")
        m = n_slots
        dev = dw.device
        self.n = n
        self.X = torch.empty(m * n, F * D, dtype=dw.dt, device=dev)
        self.tokens = torch.empty(m * n, D, dtype=torch.float32, device=dev)
        self.scores = torch.empty(m * n, dtype=torch.float32, device=dev)
        self.slots = []
        for k in range(m):
            c = dw.clone_slot(activations=False)
            c.X = self.X[k * n:(k + 1) * n]
            c.tokens = self.tokens[k * n:(k + 1) * n]
            c.scores = self.scores[k * n:(k + 1) * n]
            self.slots.append(c)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.bounds = unit_bounds(dw.req_offsets)
        dc, du = launch_sizes(n, len(self.bounds), sms, group)
        self.comp_chunk = comp_chunk if comp_chunk is not None else dc
        self.score_units = score_units if score_units is not None else du
        self.group = group
        _, hi = torch.cuda.Stream.priority_range()
        self.user = torch.cuda.Stream(dev, priority=hi)
        self.cap = torch.cuda.Stream(dev)
        self.launches_per_step = None

    def _pos(self, first: int, a: int) -> int:
        """Ring row of stream position a of a run that starts with batch ``first``."""
        return (first * self.n + a) % (len(self.slots) * self.n)

    def _score(self, first: int, a: int, b: int, stream) -> None:
        n, m = self.n, len(self.slots)
        off, kv, lu, dm = [0], [], [], []
        for j in range(a // n, (b - 1) // n + 1):
            dw = self.slots[(first + j) % m]
            lo, hi = max(a, j * n) - j * n, min(b, (j + 1) * n) - j * n
            for r in range(len(dw.L_u)):
                r0, r1 = max(dw.req_offsets[r], lo), min(dw.req_offsets[r + 1], hi)
                if r1 > r0:
                    off.append(off[-1] + r1 - r0)
                    kv.append(dw.kv[r])
                    lu.append(dw.L_u[r])
                    dm.append(dw.domain[r])
        p = self._pos(first, a)
        api.score_candidates(self.slots[0].model, self.tokens[p:p + b - a], off, kv, lu, dm,
                             self.scores[p:p + b - a], stream=stream)

    def run(self, first: int, count: int, stream=None, bind=None, fronted=None, scored=None,
            timing=None) -> None:
        """Batches first .. first + count - 1 on ``stream`` (the caller's), which waits for
        all of them at the end.  Hooks as in Overlapped.run: bind(i, dw, main) before batch
        i's first launch, fronted(i, dw, main) after its target aggregation, scored(i, dw, s)
        after the launch that completes its scores (``dw.scores``; an event it returns is
        waited for before the slot's scores are written again).  ``timing``: a list that
        receives (kind, start event, end event, candidates) for every compress and score
        launch (timing events around each; not for graph capture)."""
        n, m = self.n, len(self.slots)
        main = stream if stream is not None else torch.cuda.current_stream(self.slots[0].device)
        start = torch.cuda.Event()
        start.record(main)
        self.user.wait_event(start)
        prefilled, done_ev, released = {}, {}, {}
        waited = set()
        score_end = 0
        for step in stream_plan(n, count, first, m, self.comp_chunk, self.bounds, self.score_units, self.group):
            if step[0] == "gather":
                j = step[1]
                i, dw = first + j, self.slots[(first + j) % m]
                if bind is not None:
                    bind(i, dw, main)
                fork = torch.cuda.Event()
                fork.record(main)
                self.user.wait_event(fork)
                if j - m in done_ev:                # the slot's previous batch is scored
                    self.user.wait_event(done_ev.pop(j - m))
                dw.user_aggregate(self.user)
                user_read = torch.cuda.Event()      # the batch's user bags are read
                user_read.record(self.user)
                dw.user_prefill(self.user)
                prefilled[j] = torch.cuda.Event()
                prefilled[j].record(self.user)
                dw.target_aggregate(main)
                main.wait_event(user_read)
                if fronted is not None:
                    fronted(i, dw, main)
            elif step[0] == "compress":
                _, a, b = step
                p = self._pos(first, a)
                t0 = self._mark(main, timing)
                api.compress_targets(self.slots[0].model, self.X[p:p + b - a], self.tokens[p:p + b - a],
                                     stream=main)
                if timing is not None:
                    timing.append(("compress", t0, self._mark(main, timing), b - a))
            else:
                _, a, b = step
                for j in range(a // n, (b - 1) // n + 1):
                    if j not in waited:
                        main.wait_event(prefilled.pop(j))
                        if released.get(j - m) is not None:   # the slot's last scores were read
                            main.wait_event(released.pop(j - m))
                        waited.add(j)
                t0 = self._mark(main, timing)
                self._score(first, a, b, main)
                if timing is not None:
                    timing.append(("score", t0, self._mark(main, timing), b - a))
                for j in range(score_end // n, b // n):   # batches completed by this launch
                    if scored is not None:
                        released[j] = scored(first + j, self.slots[(first + j) % m], main)
                    done_ev[j] = torch.cuda.Event()
                    done_ev[j].record(main)
                score_end = b
        end = torch.cuda.Event()
        end.record(self.user)
        main.wait_event(end)
        for ev in released.values():
            if ev is not None:
                main.wait_event(ev)

    @staticmethod
    def _mark(stream, timing):
        if timing is None:
            return None
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        return ev

    def capture(self, first: int, count: int, **hooks) -> "torch.cuda.CUDAGraph":
        """run(first, count, ...) captured into one CUDA graph (warmed as in
        Overlapped.capture)."""
        g = torch.cuda.CUDAGraph()
        cap = self.cap
        warm_up_stream(cap, lambda: self.run(first, count, cap, **hooks))
        l0 = api.kernel_launches()
        with torch.cuda.graph(g, stream=cap):
            self.run(first, count, cap, **hooks)
        self.launches_per_step = (api.kernel_launches() - l0) / max(count, 1)
        return g


def _bag_tensors(b: DeviceBags):
    return (b.offsets, b.keys, b.weights, b.bag_table)


class HostFeed:
    """Request batches whose bags sit in pinned host memory, scored back to back (the
    serving case).  The bags of the next ``n_bag_slots - 1`` batches are copied to the device
    on a copy stream while batch i computes (``n_bag_slots`` device slots, guarded by
    events); each batch's scores are copied back to a pinned host buffer on the stream that
    scored them.

    ``batches``: list of (user bags, target bags, requests) -- each the requests' bags packed
    as pack_user_bags / pack_target_bags do, every tensor in pinned host memory; all batches
    have the requests' L_u and candidate counts of ``dw``.  With a Streamed scheduler, whose
    gathers come ``group`` at a time, ``n_bag_slots`` should exceed its group (the default 5
    covers the default group of 4): otherwise a batch's bag copy waits for the gather of the
    batch before it in the same slot and lands on the critical path.
    """

    def __init__(self, dw: DeviceWorkload, batches, n_bag_slots: int = 5):
        if n_bag_slots < 2:
            raise ValueError("HostFeed needs at least two bag slots")
        self.dw = dw
        self.batches = batches
        dev = dw.device
        self.slots = []
        for _ in range(n_bag_slots):   # device buffers with the largest size any batch needs
            def alloc(pick):
                return DeviceBags(*(torch.empty(max(int(getattr(pick(bt), f).numel()) for bt in batches),
                                                dtype=getattr(pick(batches[0]), f).dtype, device=dev)
                                    for f in ("offsets", "keys", "weights", "bag_table")))
            self.slots.append((alloc(lambda bt: bt[0]), alloc(lambda bt: bt[1])))
        self.copy_stream = torch.cuda.Stream(dev)
        self.d2h_stream = torch.cuda.Stream(dev)
        self.ready = [torch.cuda.Event() for _ in range(n_bag_slots)]
        self.free = [torch.cuda.Event() for _ in range(n_bag_slots)]
        self.h2d_bytes = [sum(x.numel() * x.element_size() for b in (bt[0], bt[1]) for x in _bag_tensors(b))
                          for bt in batches]

    def _views(self, i):
        """Device views of bag slot i mod n_bag_slots sized for batch i."""
        users, target = self.slots[i % len(self.slots)]
        hu, ht, _ = self.batches[i % len(self.batches)]

        def fit(dst, src):
            return DeviceBags(*(d[:s.numel()] for d, s in zip(_bag_tensors(dst), _bag_tensors(src))))
        return fit(users, hu), fit(target, ht)

    def _copy_in(self, i):
        hu, ht, _ = self.batches[i % len(self.batches)]
        du, dt = self._views(i)
        cs = self.copy_stream
        S = len(self.slots)
        cs.wait_event(self.free[i % S])            # batch i - S is done with this slot
        with torch.cuda.stream(cs):
            for d, h in ((du, hu), (dt, ht)):
                for dx, hx in zip(_bag_tensors(d), _bag_tensors(h)):
                    dx.copy_(hx, non_blocking=True)
        self.ready[i % S].record(cs)

    def capture(self) -> None:
        """Capture one CUDA graph per (device slot, host batch) pair, so that run() replays
        the step instead of launching its kernels one by one (on the workload's capture
        stream; see DeviceWorkload.capture_step)."""
        self.graphs = {}
        n, S = len(self.batches), len(self.slots)
        for i in range(n * S // math.gcd(n, S)):       # every (slot, batch) pair occurs
            du, dt = self._views(i)
            self.dw.use_bags(du, dt, self.batches[i % n][2])
            self.graphs[(i % S, i % n)] = self.dw.capture_step()

    def run(self, first: int, count: int, host_scores, stream=None) -> None:
        """Score batches first .. first + count - 1 (batch i uses host batch i mod len);
        the scores of batch i land in ``host_scores[i % len(host_scores)]`` (pinned)."""
        main = stream if stream is not None else torch.cuda.current_stream(self.dw.device)
        graphs = getattr(self, "graphs", None)
        start = torch.cuda.Event()
        start.record(main)
        self.copy_stream.wait_event(start)         # copies begin after work already on main
        S = len(self.slots)
        end = first + count
        for i in range(first, min(first + S - 1, end)):
            self._copy_in(i)
        for i in range(first, end):
            if i + S - 1 < end:
                self._copy_in(i + S - 1)
            main.wait_event(self.ready[i % S])
            if graphs is not None:
                with torch.cuda.stream(main):
                    graphs[(i % S, i % len(self.batches))].replay()
            else:
                du, dt = self._views(i)
                self.dw.use_bags(du, dt, self.batches[i % len(self.batches)][2])
                self.dw.step(main)
            self.free[i % S].record(main)
            host_scores[i % len(host_scores)].copy_(self.dw.scores, non_blocking=True)

    def run_overlapped(self, ov, first: int, count: int, host_scores, stream=None) -> None:
        """run() through an Overlapped or a Streamed scheduler ``ov`` (its slots are
        ``self.dw`` or clones of it): batch i reads bag slot i mod n_bag_slots, the bags of
        the next n_bag_slots - 1 batches are copied while batch i computes, a bag slot is
        refilled once its previous batch has finished its target aggregation, and each
        batch's scores are copied to the host right after the launch that completes them, on
        a stream of their own (the caller's stream waits for the last copy)."""
        main = stream if stream is not None else torch.cuda.current_stream(self.dw.device)
        S = len(self.slots)
        self.ready = [torch.cuda.Event() for _ in range(S)]   # fresh: no wait on an earlier run
        self.free = [torch.cuda.Event() for _ in range(S)]
        start = torch.cuda.Event()
        start.record(main)
        self.copy_stream.wait_event(start)
        end = first + count
        for i in range(first, min(first + S - 1, end)):
            self._copy_in(i)

        def bind(i, dw, m):
            if i + S - 1 < end:
                self._copy_in(i + S - 1)
            m.wait_event(self.ready[i % S])
            du, dt = self._views(i)
            dw.use_bags(du, dt, self.batches[i % len(self.batches)][2])

        def fronted(i, dw, m):
            self.free[i % S].record(m)

        def scored(i, dw, s):
            # on a stream of its own: a device-to-host copy queued behind the bag copies
            # must not hold up the next launches of the stream that scored the batch
            ev = torch.cuda.Event()
            ev.record(s)
            self.d2h_stream.wait_event(ev)
            with torch.cuda.stream(self.d2h_stream):
                host_scores[i % len(host_scores)].copy_(dw.scores, non_blocking=True)
            read = torch.cuda.Event()
            read.record(self.d2h_stream)
            return read                   # the slot's scores may be overwritten after this

        ov.run(first, count, main, bind=bind, fronted=fronted, scored=scored)
        done = torch.cuda.Event()
        done.record(self.d2h_stream)
        main.wait_event(done)

    def copies_only(self, first: int, count: int, host_scores, scores, stream=None) -> None:
        """The host traffic of run() alone, on ``stream``: each batch's bags in (the same
        copies into the same slots) and ``scores`` [n] back out, with no compute.  Timing it
        gives the copy-bound floor of the host-fed step."""
        main = stream if stream is not None else torch.cuda.current_stream(self.dw.device)
        with torch.cuda.stream(main):
            for i in range(first, first + count):
                hu, ht, _ = self.batches[i % len(self.batches)]
                du, dt = self._views(i)
                for d, h in ((du, hu), (dt, ht)):
                    for dx, hx in zip(_bag_tensors(d), _bag_tensors(h)):
                        dx.copy_(hx, non_blocking=True)
                host_scores[i % len(host_scores)].copy_(scores, non_blocking=True)

    def capture_overlapped(self, ov, first: int, count: int, host_scores) -> "torch.cuda.CUDAGraph":
        """run_overlapped(...) captured into one CUDA graph, host copies included (on
        ``ov``'s capture stream, warmed as in Overlapped.capture)."""
        g = torch.cuda.CUDAGraph()
        cap = ov.cap
        warm_up_stream(cap, lambda: self.run_overlapped(ov, first, count, host_scores, cap))
        with torch.cuda.graph(g, stream=cap):
            self.run_overlapped(ov, first, count, host_scores, cap)
        return g


def compress_corpus(model, target_tables, bags: DeviceBags, n_items: int, n_fields: int, out: torch.Tensor,
                    chunk: int = 1 << 18, stream=None) -> torch.Tensor:
    """Near-line index build (TransRetrieval §3.3: the compressed target token is also the
    item's index vector, computed off the request path): every item of a corpus, its
    ``n_fields`` target-field bags aggregated (tr_aggregate) and compressed
    (tr_compress_targets) into ``out`` [n_items, D] fp32, ``chunk`` items at a time through one
    [chunk, F*D] buffer of the model's dtype.  ``bags`` holds the corpus's bags on the device,
    item i's fields at bags i*F .. i*F+F-1 (CSR offsets into the full key/weight arrays)."""
    D = out.shape[1]
    X = torch.empty(min(chunk, max(n_items, 1)), n_fields * D, dtype=api.torch_dtype(model.dims.dtype),
                    device=out.device)
    for c0 in range(0, n_items, chunk):
        c1 = min(n_items, c0 + chunk)
        m = c1 - c0
        b0, b1 = c0 * n_fields, c1 * n_fields
        api.aggregate(target_tables, bags.bag_table[b0:b1], bags.offsets[b0:b1 + 1], bags.keys, bags.weights,
                      X[:m].view(-1, D), stream=stream)
        api.compress_targets(model, X[:m], out[c0:c1], stream=stream)
    return out
