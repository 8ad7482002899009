#!/usr/bin/env python
"""Throughput of the TransRetrieval candidate-scoring step on B200.

A step is one pass of the whole scoring path over one request of the 128D-5L workload
(40,000 candidates, L_u = 64, 8 target fields over 4M-row tables):
  [side stream] tr_aggregate(user fields) -> tr_prefill_user
  [main stream] tr_aggregate(target fields) -> tr_compress_targets
  -> (join) tr_score_candidates.
Stage times come from CUDA events on the stream each stage runs on; the user side
overlaps the target side, so the stages do not add up to the step.
``value`` is candidates scored per second over all ranks, with inputs resident in HBM: the
K timed steps are one stream of candidate tiles, captured into one CUDA graph, whose
compress and score launches take fixed chunks across request boundaries (two compressor
rounds, one score round each; pipeline.Streamed).  The same steps with each request's last
partial rounds run beside the next request (pipeline.Overlapped) are reported as
``overlapped_graph_ms_per_step``, and run one after the other as ``serial_graph_ms_per_step``.  ``e2e`` repeats the K steps with each
request's bags copied from pinned host memory (during the previous request) and its scores
copied back, all inside the timed region.  Requests rotate over several seeded request sets and the
embedding tables (24.6 GB) are far larger than L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --case bulk|uncompressed|fused [--case-n N]  side measurements (JSON line)
  python bench.py --case score|compress|prefill|all          one stage, for a profiler

Multi-GPU: one process per GPU (torchrun); every rank scores its own requests (weak
scaling, no collective on the data path); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import datagen  # noqa: E402

WORKLOAD = "128d5l"
METRIC = "candidates scored/sec at 128D5L, 40k cands/request; % bf16 tensor peak"
N_REQUEST_SETS = 4
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary under profiles/,
    or None when there is none or the kernel's sources changed since it was captured."""
    import glob
    import hashlib
    import re

    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(path).read()
        m = re.search(r"kernel: (\S+)\ntraffic_bytes_per_launch: (\d+)\nsources: ([^\n]+)\nsources_sha256: ([0-9a-f]+)", text)
        if not m or m.group(1) != kernel:
            continue
        h = hashlib.sha256()
        try:
            for f in m.group(3).split():
                with open(os.path.join(ROOT, f), "rb") as fh:
                    h.update(fh.read())
        except OSError:
            return None
        return int(m.group(2)) if h.hexdigest() == m.group(4) else None
    return None


# ------------------------------------------------------------------ algorithmic work

def stack_flops_per_candidate(dims, L_u):
    """N*(16 D^2 + 4 (L_u+1) D) + 2D (TransRetrieval §3.3 count plus own key/value and head)."""
    return dims.n_layer * (16 * dims.D ** 2 + 4 * (L_u + 1) * dims.D) + 2 * dims.D


def compressor_flops_per_candidate(dims):
    c = dims.comp_dims
    return 2 * sum(c[i] * c[i + 1] for i in range(3))


def aggregate_bytes(bags, D, elem_bytes, out_bytes):
    """Rows gathered + keys/weights + offsets/table ids + output rows."""
    nnz, n_bags = bags.nnz, bags.n_bags
    return nnz * D * elem_bytes + nnz * 8 + n_bags * 12 + 8 + n_bags * D * out_bytes


# ------------------------------------------------------------------ clocks

class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r for r in self.rows if len(r) >= 7]
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(r[0]) for r in rows]
        reasons = set()
        for r in rows:
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"), r[3:7]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.nanmedian(sm)), "sm_max_mhz": num(rows[0][1]),
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ CPU (oracle) leg

def time_oracle(w, P, req, target_seconds=15.0, max_cand=None):
    """The fp64 oracle on a bounded sample of one request: user side once, then a
    contiguous slice of candidates.  Returns (candidates/s for the whole request
    extrapolated from the sample, description, threads)."""
    import oracle
    from threadpoolctl import threadpool_info

    threads = max([t.get("num_threads", 1) for t in threadpool_info()] + [1])
    t0 = time.perf_counter()
    user_tokens = oracle.aggregate_bags(w, req.user, "user")
    K, V = oracle.prefill_user(P, w.dims.n_head, user_tokens, req.domain)
    t_user = time.perf_counter() - t0

    def cand_time(n):
        t = time.perf_counter()
        oracle.score_request_candidates(w, P, req, np.arange(n), K, V)
        return time.perf_counter() - t
    n = 200
    dt = cand_time(n)
    per = dt / n
    n2 = int(min(req.n_cand if max_cand is None else max_cand, max(n, target_seconds / max(per, 1e-9))))
    if n2 > n:
        dt = cand_time(n2)
        n = n2
        per = dt / n
    total = t_user + per * req.n_cand
    rate = req.n_cand / total
    desc = (f"oracle (fp64 numpy) on {n} of {req.n_cand} candidates of one {w.name} request plus its user side "
            f"({t_user:.2f} s user side, {dt:.2f} s candidates); rate = n_cand / (t_user + n_cand * t_cand/n)")
    return rate, desc, threads, t_user + dt


def oracle_rates(w, P, req, seconds_all=15.0, seconds_one=6.0):
    """The oracle's candidates/s on one request with every host thread its BLAS uses and
    with one thread, plus the host's core counts."""
    from threadpoolctl import threadpool_limits
    rate, desc, threads, _ = time_oracle(w, P, req, target_seconds=seconds_all)
    with threadpool_limits(limits=1):
        rate1, _, _, _ = time_oracle(w, P, req, target_seconds=seconds_one)
    return {"value": rate, "unit": "candidates/s", "cores": threads, "kind": "oracle", "sample": desc,
            "one_thread": rate1, "nproc": os.cpu_count(), "affinity": len(os.sched_getaffinity(0))}


def bench_config(n_cand: int, L_u: int, world: int) -> dict:
    """The workload both arms report."""
    return {"workload": "128D-5L, 1 request x 40,000 candidates per GPU, L_u=64, 8 target fields, "
                        "16+8 tables of 4M rows (24.6 GB bf16)",
            "n_cand_per_gpu": n_cand, "L_u": L_u, "request_sets": N_REQUEST_SETS,
            "l2": "inputs larger than L2: tables 24.6 GB, uniform target keys, rotating request sets",
            "parallelism": f"candidate shards, {world} GPU(s), no collective"}


def run_reference(args, rank, world):
    """Reference arm: the oracle as it stands on the host cores (rank 0 only)."""
    if rank != 0:
        return
    w = datagen.WORKLOADS[WORKLOAD]
    P = datagen.workload_params(w)
    req = datagen.make_requests(w)[0]
    # each step is a bounded sample of the request (its user side and a slice of its
    # candidates), sized so that the W + K steps stay within a few minutes; ms_per_step is
    # the time one such step took
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    vals, secs_all = [], []
    for i in range(args.warmup + args.steps):
        rate, desc, threads, secs = time_oracle(w, P, req, target_seconds=budget)
        if i >= args.warmup:
            vals.append(rate)
            secs_all.append(secs)
    v = float(np.median(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "candidates/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(secs_all)) * 1e3,
        "step": "one bounded sample of the request per step (its user side plus a slice of its candidates); "
                "value = the request's candidates / (user side + per-candidate time x candidates)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w.n_cand_per_request, 64, 1),
        "cpu_baseline": {"value": v, "unit": "candidates/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": "candidates/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU leg

STAGE_SPANS = {"user_side": ("user0", "user1"), "target_aggregate": ("t0", "agg"), "compress": ("agg", "comp"),
               "score": ("s0", "score")}
EV_KEYS = ["user0", "user1", "t0", "agg", "comp", "s0", "score"]


def stage_rooflines(dims, reqs, stage_ms, peaks, peak_kind):
    """Achieved rate and fraction of the measured peak of the three bulk stages of one step."""
    n_cand = sum(r.n_cand for r in reqs)
    fl_stack = sum(stack_flops_per_candidate(dims, r.L_u) * r.n_cand for r in reqs)
    fl_comp = compressor_flops_per_candidate(dims) * n_cand
    eb = 2 if dims.dtype == "bf16" else 4
    agg_bytes = sum(aggregate_bytes(r.target, dims.D, eb, eb) for r in reqs)
    roof = {
        "score": {"bound": "tensor", "achieved": fl_stack / (stage_ms["score"] / 1e3) / 1e12,
                  "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"},
        "compress": {"bound": "tensor", "achieved": fl_comp / (stage_ms["compress"] / 1e3) / 1e12,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"},
        "target_aggregate": {"bound": "hbm", "achieved": agg_bytes / (stage_ms["target_aggregate"] / 1e3) / 1e9,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s"},
    }
    for r in roof.values():
        r["frac"] = r["achieved"] / r["peak"]
        r["peak_source"] = peak_kind
    return roof


def measure_side(name, w, params, tables, reqs, dev, steps, warmup, peaks, peak_kind, cpu_seconds):
    """One of the other workloads on the same GPU (every stage through the C calls): stage
    times from eager steps, the step from one CUDA graph per step replayed back to back, the
    overlapped requests and the stream of candidate tiles (one graph each; the value is the
    stream's); the oracle's rate on the same request."""
    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload, Overlapped, Streamed

    stream = torch.cuda.current_stream()
    dw = DeviceWorkload(w, device=dev, reqs=reqs, params=params, tables=tables)
    for _ in range(warmup):
        dw.step(stream)
    torch.cuda.synchronize()
    ev = [{k: torch.cuda.Event(enable_timing=True) for k in EV_KEYS} for _ in range(steps)]
    for i in range(steps):
        dw.step(stream, ev[i])
    torch.cuda.synchronize()
    stage_ms = {n: float(np.mean([ev[i][a].elapsed_time(ev[i][b]) for i in range(steps)]))
                for n, (a, b) in STAGE_SPANS.items()}
    g = dw.capture_step()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = e0.elapsed_time(e1) / steps
    del g
    dw2 = DeviceWorkload(w, device=dev, reqs=reqs, params=params, tables=tables)
    ov = Overlapped([dw, dw2])
    ov.run(0, warmup, stream)
    torch.cuda.synchronize()
    g = ov.capture(0, steps)
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ov_ms = e0.elapsed_time(e1) / steps
    del g
    st = Streamed(dw)
    st.run(0, warmup, stream)
    torch.cuda.synchronize()
    g = st.capture(warmup, steps)
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    st_ms = e0.elapsed_time(e1) / steps
    del g
    if api.sync_status() != 0:
        raise RuntimeError(f"device status word set during the {name} measurement")
    n_cand = dw.n_cand
    out = {"workload": w.name, "candidates_per_step": n_cand, "requests": len(reqs),
           "L_u": [r.L_u for r in reqs] if len(reqs) > 1 else reqs[0].L_u,
           "value": n_cand / (st_ms / 1e3), "unit": "candidates/s", "ms_per_step": st_ms,
           "overlapped_graph_ms_per_step": ov_ms, "serial_graph_ms_per_step": serial_ms,
           "stages": {k: {"ms": v} for k, v in stage_ms.items()}}
    for k, r in stage_rooflines(w.dims, reqs, stage_ms, peaks, peak_kind).items():
        out["stages"][k].update(r)
    if cpu_seconds > 0:
        out["cpu_baseline"] = oracle_rates(w, params, reqs[0], cpu_seconds, cpu_seconds / 2)
    del dw, dw2, ov, st
    torch.cuda.empty_cache()
    return out


def run_side_configs(args, dev, main_dw, peaks, peak_kind):
    """The 64D-3L, packed 16 x 4,096 and 52M-row large-corpus workloads (the other
    single-GPU configurations the headline is reported beside)."""
    import torch

    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload

    res = {}
    cpu_s = 0.0 if args.no_cpu_baseline else 6.0
    steps, warm = max(3, min(args.steps, 10)), 3
    # 64D-3L: its own tables (16 of 1M rows x 64) and parameters
    w = datagen.WORKLOADS["64d3l"]
    res["64d3l"] = measure_side("64d3l", w, datagen.workload_params(w), DeviceWorkload.make_tables(w, dev),
                                datagen.make_requests(w), dev, steps, warm, peaks, peak_kind, cpu_s)
    torch.cuda.empty_cache()
    # packed: 16 requests of the 128D-5L model, L_u ~ U{16..128}, 4,096 candidates each (the
    # headline workload's tables and parameters; the request shapes are the packed recipe's)
    w = datagen.WORKLOADS["packed"]
    tables = (main_dw.user_tables, main_dw.target_tables)
    res["packed"] = measure_side("packed", w, main_dw.params, tables, datagen.make_requests(w), dev, steps, warm,
                                 peaks, peak_kind, cpu_s)
    res["packed"]["tables"] = "the 128D-5L workload's tables and parameters"
    # large corpus: target field 0 reads one 52M-row table (uniform keys); the other tables
    # are the headline workload's
    w = datagen.WORKLOADS["large"]
    big = torch.empty(w.target_rows[0], w.dims.D, dtype=torch.bfloat16, device=dev)
    datagen.fill_table_device(big, w.seed, datagen.target_table_id(w, 0))
    tables = (main_dw.user_tables, [big] + list(main_dw.target_tables[1:]))
    res["large"] = measure_side("large", w, main_dw.params, tables, datagen.make_requests(w), dev,
                                max(3, steps // 2), 2, peaks, peak_kind, cpu_s)
    res["large"]["tables"] = "one 52M x 128 bf16 table (13.3 GB) for field 0 plus the 128D-5L workload's tables"
    del big
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import (DeviceBags, DeviceWorkload, HostFeed, Overlapped, Streamed,
                                                             score_split)
    from transformer_candidate_scoring_b200.shard import max_over_ranks, rank_seed

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = datagen.WORKLOADS[WORKLOAD]
    dims = w.dims
    # distinct request sets per rank and per step (seeded)
    sets = [datagen.make_requests(w, seed=rank_seed(w.seed, rank, s)) for s in range(N_REQUEST_SETS)]
    dw = DeviceWorkload(w, device=dev, reqs=sets[0])
    dsets = []
    for reqs in sets:
        dw.set_requests(reqs)
        dsets.append((dw.user_bags, dw.target_bags, reqs))
    stream = torch.cuda.current_stream()

    def use(i):
        ub, tb, reqs = dsets[i % N_REQUEST_SETS]
        dw.user_bags, dw.target_bags, dw.reqs = ub, tb, reqs
        dw.L_u = [r.L_u for r in reqs]
        dw.domain = [r.domain for r in reqs]

    stage_names = ["user_side", "target_aggregate", "compress", "score"]
    ev_keys = ["user0", "user1", "t0", "agg", "comp", "s0", "score"]

    def step(i, events=None):
        use(i)
        dw.step(stream, events)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if api.sync_status() != 0:
        raise RuntimeError("device reported an out-of-range key during warm-up")

    clocks = ClockSampler(local_rank)
    clocks.start()
    ev = [{k: torch.cuda.Event(enable_timing=True) for k in ev_keys} for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    launches0 = api.kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = api.kernel_launches() - launches0
    elapsed = t0.elapsed_time(t1) / 1e3
    spans = {"user_side": ("user0", "user1"), "target_aggregate": ("t0", "agg"), "compress": ("agg", "comp"),
             "score": ("s0", "score")}
    stage_ms = {n: float(np.mean([ev[i][a].elapsed_time(ev[i][b]) for i in range(args.steps)]))
                for n, (a, b) in spans.items()}
    elapsed = max_over_ranks(elapsed)
    eager_ms = elapsed / args.steps * 1e3

    # ---- the same steps, one CUDA graph per step (one per request set), replayed back to
    # back: every step starts after the previous one has ended
    graphs = []
    for s_i in range(N_REQUEST_SETS):
        use(s_i)
        graphs.append(dw.capture_step())
    for i in range(args.warmup):
        graphs[i % N_REQUEST_SETS].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for i in range(args.steps):
        graphs[(args.warmup + i) % N_REQUEST_SETS].replay()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    if api.sync_status() != 0:
        raise RuntimeError("device status word set during the graph replays")
    serial_elapsed = max_over_ranks(g0.elapsed_time(g1) / 1e3)
    del graphs

    def bind(i, slot, main):
        ub, tb, reqs = dsets[i % N_REQUEST_SETS]
        slot.use_bags(ub, tb, reqs)

    def replay_time(runner, label):
        runner.run(0, args.warmup, stream, bind=bind)          # eager warm-up of the slots
        torch.cuda.synchronize()
        g = runner.capture(args.warmup, args.steps, bind=bind)
        g.replay()                                             # warm-up replay (K more steps)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        g0.record(stream)
        g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        barrier()
        if api.sync_status() != 0:
            raise RuntimeError(f"device status word set during the {label} replays")
        del g
        return max_over_ranks(g0.elapsed_time(g1) / 1e3)

    # ---- consecutive requests overlapped over two activation slots (Overlapped: each
    # request's last partial rounds of compression and scoring run beside the next request's
    # aggregation), captured into one CUDA graph
    dw2 = DeviceWorkload(w, device=dev, reqs=sets[0], params=dw.params,
                         tables=(dw.user_tables, dw.target_tables))
    ov = Overlapped([dw, dw2])
    overlapped_elapsed = replay_time(ov, "overlapped")
    # ---- the timed value: the K steps as one stream of candidate tiles (Streamed: after
    # every fourth request's gather, one compress launch of eight rounds of tiles and one score
    # launch of four rounds of two-tile units at 40,000 candidates a request, across request
    # boundaries, over a ring of activation slots), one CUDA graph
    st = Streamed(dw)
    graph_elapsed = replay_time(st, "streamed")
    launches = st.launches_per_step * args.steps
    # the same K steps once more, eagerly, with CUDA events around every compress and score
    # launch on the stream that issues them: the kernels' own times inside the schedule
    # (the graph's kernels cannot be bracketed one by one)
    timing = []
    st.run(args.warmup, args.steps, stream, bind=bind, timing=timing)
    torch.cuda.synchronize()
    in_sched = {}
    for kind, a, b, n in timing:
        d = in_sched.setdefault(kind, {"launches": 0, "ms": 0.0, "candidates": 0})
        d["launches"] += 1
        d["ms"] += a.elapsed_time(b)
        d["candidates"] += n
    use_graphs = True                     # the timed value is always graph-replayed
    elapsed = graph_elapsed
    clk = clocks.stop()
    n_cand = dw.n_cand
    value = n_cand * args.steps * world / elapsed

    # ---- per-request top-k of the scores (the selection step after scoring; timed on its
    # own, it is not one of the step's stages)
    TOPK = 2000
    dw.select(TOPK, stream)
    torch.cuda.synchronize()
    gk = torch.cuda.CUDAGraph()          # replayed, so the time is the kernel's, not the host's
    with torch.cuda.graph(gk, stream=torch.cuda.Stream()):
        dw.select(TOPK)
    gk.replay()
    torch.cuda.synchronize()
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    for _ in range(args.steps):
        gk.replay()
    k1.record(stream)
    torch.cuda.synchronize()
    topk_ms = k0.elapsed_time(k1) / args.steps

    # ---- end to end: host bags in, scores out, through the package's host feed (the bags
    # of batch i + 1 are copied while batch i computes)
    host_batches = []
    for ub, tb, reqs in dsets:
        hu = DeviceBags(*(x.cpu().pin_memory() for x in (ub.offsets, ub.keys, ub.weights, ub.bag_table)))
        ht = DeviceBags(*(x.cpu().pin_memory() for x in (tb.offsets, tb.keys, tb.weights, tb.bag_table)))
        host_batches.append((hu, ht, reqs))
    feed = HostFeed(dw, host_batches)
    # the host-fed stream runs its launches after every second request: with the bag copies
    # beside it, evenly spaced launches overlap them better than the resident stream's
    # groups of four (measured: 0.382 against 0.411 ms per step)
    st_feed = Streamed(dw, group=2)
    h2d = float(np.mean(feed.h2d_bytes))
    host_scores = [torch.empty(n_cand, dtype=torch.float32).pin_memory() for _ in range(2)]
    d2h = n_cand * 4

    feed.run_overlapped(st_feed, 0, args.warmup, host_scores, stream)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    feed.run_overlapped(st_feed, args.warmup, args.steps, host_scores, stream)   # eager launches
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_eager_ms = max_over_ranks(e0.elapsed_time(e1) / 1e3) / args.steps * 1e3
    # the same launch mode as the timed value: one graph of the K steps, host copies inside
    g_e2e = feed.capture_overlapped(st_feed, args.warmup, args.steps, host_scores)
    g_e2e.replay()
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    g_e2e.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_elapsed = e0.elapsed_time(e1) / 1e3
    e2e_elapsed = max_over_ranks(e2e_elapsed)
    e2e_value = n_cand * args.steps * world / e2e_elapsed
    # the same host traffic with no compute: the copy-bound floor of the e2e step
    feed.copies_only(0, args.warmup, host_scores, dw.scores, stream)
    torch.cuda.synchronize()
    e0.record(stream)
    feed.copies_only(args.warmup, args.steps, host_scores, dw.scores, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    copy_ms = max_over_ranks(e0.elapsed_time(e1) / 1e3) / args.steps * 1e3

    # ---- rooflines of the stages
    peaks, peak_kind = load_peaks()
    L_u = dw.L_u[0]
    stage_roof = stage_rooflines(dims, sets[0], stage_ms, peaks, peak_kind)
    # the dominant kernel of the timed schedule (the score kernel), from its launches in the
    # eager run of that schedule: algorithmic FLOPs of each launch's candidates over the
    # launches' total event time
    sched_roof = {}
    for kind, per_cand, kernel in (("score", stack_flops_per_candidate(dims, L_u), "stack_kernel"),
                                   ("compress", compressor_flops_per_candidate(dims), "compress_kernel")):
        d = in_sched[kind]
        ach = per_cand * d["candidates"] / (d["ms"] / 1e3) / 1e12
        sched_roof[kind] = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                            "frac": ach / peaks["bf16_tflops"], "peak_source": peak_kind, "kernel": kernel,
                            "launches": d["launches"], "mean_ms": d["ms"] / d["launches"],
                            "candidates_per_launch": d["candidates"] / d["launches"]}
    dominant = max(sched_roof, key=lambda k: in_sched[k]["ms"])
    roof = dict(sched_roof[dominant])
    roof["measured"] = "CUDA events around each launch in an eager run of the timed schedule"
    # DRAM bytes per launch from the committed ncu summary of a full-size launch of the
    # kernel (null once its sources changed)
    roof["traffic"] = profiled_traffic(roof["kernel"]) if dominant == "score" else None
    # the score kernel over its full rounds alone (the candidates before score_split: every
    # CTA busy until the end), eager launches timed with events on the launching stream
    cut = score_split(dw.req_offsets, torch.cuda.get_device_properties(dev).multi_processor_count)
    full_round = None
    if cut is not None:
        use(0)
        dw.step(stream)
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dw.score_range(0, cut, stream)
        f0.record(stream)
        for _ in range(args.steps):
            dw.score_range(0, cut, stream)
        f1.record(stream)
        torch.cuda.synchronize()
        fr_ms = f0.elapsed_time(f1) / args.steps
        fr_ach = stack_flops_per_candidate(dims, L_u) * cut / (fr_ms / 1e3) / 1e12
        full_round = {"candidates": cut, "ms": fr_ms, "achieved": fr_ach, "unit": "TFLOP/s",
                      "peak": peaks["bf16_tflops"], "frac": fr_ach / peaks["bf16_tflops"], "peak_source": peak_kind}
    roof_score_full = full_round
    side = None if (args.no_side_configs or world > 1) else run_side_configs(args, dev, dw, peaks, peak_kind)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = oracle_rates(w, dw.params, sets[0][0], args.cpu_seconds, args.cpu_seconds / 2)
    line = {
        "metric": METRIC, "value": value, "unit": "candidates/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(n_cand, L_u, world),
        "roofline": roof,
        "stages": {k: {"ms": stage_ms[k], **({kk: vv for kk, vv in stage_roof[k].items()} if k in stage_roof else {})}
                   for k in stage_names},
        "pct_bf16_peak_score_kernel": sched_roof["score"]["frac"] * 100,
        "schedule_kernels": sched_roof,
        "score_full_rounds": roof_score_full,
        "configs": side,
        "topk": {"k": TOPK, "ms": topk_ms, "note": "tr_topk over the step's scores, timed separately"},
        "e2e": {"value": e2e_value, "unit": "candidates/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_elapsed / args.steps * 1e3,
                "eager_ms_per_step": e2e_eager_ms,
                "copies_only_ms_per_step": copy_ms,
                "h2d_gbs_copies_only": h2d / (copy_ms / 1e3) / 1e9},
        "gpu_launches": int(launches),
        "launch": {"graphs": bool(use_graphs), "e2e_graphs": bool(use_graphs), "group": st.group,
                   "e2e_group": st_feed.group,
                   "overlap": ("one stream of candidate tiles across requests: compress launches of whole rounds "
                               "of tiles, score launches of whole rounds of two-tile units, as many as four "
                               "requests fill (pipeline.Streamed)"),
                   "ring_slots": len(st.slots),
                   "graph_ms_per_step": graph_elapsed / args.steps * 1e3,
                   "overlapped_graph_ms_per_step": overlapped_elapsed / args.steps * 1e3,
                   "serial_graph_ms_per_step": serial_elapsed / args.steps * 1e3,
                   "eager_ms_per_step": eager_ms},
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_case(args):
    """One stage of the 128D-5L path on stand-alone seeded inputs, a few launches, no JSON:
    the target of profiler captures (small inputs; the gather case builds 8 target tables of
    --case-rows rows, 2 GB at the default 1M, larger than L2; the stream case runs the timed
    schedule itself on the full workload, eagerly, for a launch list)."""
    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceBags

    w = datagen.WORKLOADS[WORKLOAD]
    dims = w.dims
    n = args.case_n
    if args.case == "stream":
        # the timed schedule itself, eagerly: --case-reps batches of the 128D-5L workload
        # through pipeline.Streamed (after two warm-up batches), for a launch list
        from transformer_candidate_scoring_b200.pipeline import DeviceWorkload, Streamed
        dw = DeviceWorkload(w, device=torch.device("cuda"))
        st = Streamed(dw)
        st.run(0, 2)
        torch.cuda.synchronize()
        st.run(2, args.case_reps)
        torch.cuda.synchronize()
        if api.sync_status() != 0:
            raise RuntimeError("device status word set")
        print("case stream: ok")
        return
    if args.case == "gather":
        ws = datagen.scaled(w, n_cand_per_request=n, rows=args.case_rows or 1_000_000)
        tables = [torch.empty(r, dims.D, dtype=torch.bfloat16, device="cuda") for r in ws.target_rows]
        for t, x in enumerate(tables):
            datagen.fill_table_device(x, ws.seed, datagen.target_table_id(ws, t))
        bags = DeviceBags.of(datagen.make_target_bags(np.random.default_rng(ws.seed), ws, n), "cuda")
        X = torch.empty(n * dims.n_target_fields, dims.D, dtype=torch.bfloat16, device="cuda")
        for _ in range(args.case_reps):
            api.aggregate(tables, bags.bag_table, bags.offsets, bags.keys, bags.weights, X)
        torch.cuda.synchronize()
        if api.sync_status() != 0:
            raise RuntimeError("device status word set")
        print("case gather: ok")
        return
    m = api.Model(dims, datagen.workload_params(w))
    U = torch.from_numpy(datagen.rand_matrix(1, (64, dims.D), 0.01, "f32")).cuda()
    kv = torch.zeros(api.kv_cache_bytes(m, 64), dtype=torch.uint8, device="cuda")
    X = torch.from_numpy(datagen.rand_matrix(3, (n, dims.comp_dims[0]), 0.01, "bf16")).cuda().to(torch.bfloat16)
    T = torch.empty(n, dims.D, dtype=torch.float32, device="cuda")
    s = torch.empty(n, dtype=torch.float32, device="cuda")
    for _ in range(args.case_reps):
        if args.case in ("prefill", "all"):
            api.prefill_user(m, U, 64, 1, kv)
        if args.case in ("compress", "score", "all"):
            api.compress_targets(m, X, T)
        if args.case in ("score", "all"):
            api.score_candidates(m, T, [0, n], [kv], [64], [1], s)
    torch.cuda.synchronize()
    if api.sync_status() != 0:
        raise RuntimeError("device status word set")
    print(f"case {args.case}: ok")


def run_bulk(args):
    """Near-line bulk compression (the index-build path): --case-n items of the 128D-5L
    workload's target side (8 fields over the 4M-row target tables, uniform keys),
    aggregated and compressed in chunks of 256K items; prints one JSON line with items/s.
    Not the headline: the step above is."""
    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, DeviceWorkload, compress_corpus

    w = datagen.WORKLOADS[WORKLOAD]
    dims = w.dims
    n = args.case_n
    tables = DeviceWorkload.make_tables(w.with_(user_tables=0), torch.device("cuda"))
    model = api.Model(dims, datagen.workload_params(w))
    bags = DeviceBags.of(datagen.make_target_bags(np.random.default_rng(w.seed + 77), w, n), "cuda")
    out = torch.empty(n, dims.D, dtype=torch.float32, device="cuda")
    F = dims.n_target_fields
    compress_corpus(model, tables[1], bags, n, F, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.case_reps)
    e0.record()
    for _ in range(reps):
        compress_corpus(model, tables[1], bags, n, F, out)
    e1.record()
    torch.cuda.synchronize()
    if api.sync_status() != 0:
        raise RuntimeError("device status word set")
    sec = e0.elapsed_time(e1) / 1e3 / reps
    print(json.dumps({"case": "bulk_compression", "items": n, "items_per_s": n / sec, "ms": sec * 1e3,
                      "workload": "128D-5L target side, 8 fields, 4M-row tables, chunks of 262144 items"}),
          flush=True)


def run_uncompressed(args):
    """The cost target compression removes (§3.3): --case-n candidates of one 128D-5L request
    scored as L_t = 8 uncompressed field tokens and as one compressed token, on the
    tensor-core stack kernel (the serving kernel) and, for reference, on the CUDA-core
    kernels (a second model handle made with TR_FORCE_SIMT=1); prints one JSON line with the
    device times (CUDA events) and the FLOP ratio."""
    import os

    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceWorkload

    w = datagen.scaled(datagen.WORKLOADS[WORKLOAD], n_cand_per_request=args.case_n, rows=200_000)
    dims = w.dims
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    F, D, n = dims.n_target_fields, dims.D, dw.n_cand
    X = dw.X.view(n, F, D)
    s = torch.empty(n, dtype=torch.float32, device="cuda")
    args_kv = (dw.req_offsets, dw.kv, dw.L_u, dw.domain, s)
    os.environ["TR_FORCE_SIMT"] = "1"
    try:
        simt_model = api.Model(dims, dw.params)
    finally:
        del os.environ["TR_FORCE_SIMT"]

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps
    tc8 = timed(lambda: api.score_candidates_uncompressed(dw.model, X, F, *args_kv))
    tc1 = timed(lambda: api.score_candidates(dw.model, dw.tokens, *args_kv))
    cc8 = timed(lambda: api.score_candidates_uncompressed(simt_model, X, F, *args_kv), reps=2)
    cc1 = timed(lambda: api.score_candidates_uncompressed(simt_model, dw.tokens, 1, *args_kv), reps=2)
    if api.sync_status() != 0:
        raise RuntimeError("device status word set")
    L_u = dw.L_u[0]
    f8 = dims.n_layer * (16 * F * D * D + 4 * F * (L_u + F) * D) + 2 * D * F
    f1 = stack_flops_per_candidate(dims, L_u)
    print(json.dumps({"case": "uncompressed_targets", "candidates": n, "L_t": F, "L_u": L_u,
                      "ms_L_t_8_tensor_cores": tc8, "ms_L_t_1_tensor_cores": tc1,
                      "time_saving_tensor_cores": 1 - tc1 / tc8,
                      "ms_L_t_8_cuda_cores": cc8, "ms_L_t_1_cuda_cores": cc1,
                      "time_saving_cuda_cores": 1 - cc1 / cc8,
                      "tflops_L_t_8_tensor_cores": f8 * n / tc8 / 1e9,
                      "flops_per_candidate_L_t_8": f8, "flops_per_candidate_L_t_1": f1,
                      "flop_saving": 1 - f1 / f8}), flush=True)


def run_fused(args):
    """The target side of one 128D-5L request (--case-n candidates, 8 fields over the 4M-row
    target tables) as two launches (tr_aggregate, then tr_compress_targets) and as one
    (tr_compress_target_bags, the gather feeding the compressor on chip); prints one JSON
    line with both device times (CUDA events, --case-reps launches each after a warm-up) and
    whether the two results are bit-identical."""
    import torch

    from transformer_candidate_scoring_b200 import api
    from transformer_candidate_scoring_b200.pipeline import DeviceBags, DeviceWorkload

    w = datagen.WORKLOADS[WORKLOAD]
    if args.case_rows is not None and args.case_rows < min(w.target_rows):
        w = datagen.scaled(w, rows=args.case_rows)
    dims = w.dims
    n, F, D = args.case_n, dims.n_target_fields, dims.D
    tables = DeviceWorkload.make_tables(w.with_(user_tables=0), torch.device("cuda"))[1]
    model = api.Model(dims, datagen.workload_params(w))
    bags = DeviceBags.of(datagen.make_target_bags(np.random.default_rng(w.seed + 5), w, n), "cuda")
    ba = (bags.bag_table, bags.offsets, bags.keys, bags.weights)
    X = torch.empty(n * F, D, dtype=torch.bfloat16, device="cuda")
    two = torch.empty(n, D, dtype=torch.float32, device="cuda")
    fused = torch.empty_like(two)

    def two_launch():
        api.aggregate(tables, *ba, X)
        api.compress_targets(model, X.view(n, F * D), two)

    def one_launch():
        api.compress_target_bags(model, tables, *ba, fused)

    def timed(fn, reps):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps
    reps = max(1, args.case_reps)
    t_two = timed(two_launch, reps)
    t_one = timed(one_launch, reps)
    if api.sync_status() != 0:
        raise RuntimeError("device status word set")
    print(json.dumps({"case": "fused_target_side", "candidates": n, "ms_gather_then_compress": t_two,
                      "ms_fused": t_one, "speedup": t_two / t_one, "bit_identical": bool(torch.equal(two, fused)),
                      "workload": f"128D-5L target side, 8 fields of 1..8 keys over {min(w.target_rows)}-row "
                                  "bf16 tables"}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side-configs", action="store_true", help="skip the 64D-3L, packed and large workloads")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--case", choices=["score", "compress", "prefill", "all", "gather", "stream", "bulk",
                                       "uncompressed", "fused"],
                    default=None,
                    help="run one stage on stand-alone inputs for a profiler (no timing, no JSON)")
    ap.add_argument("--case-n", type=int, default=40000)
    ap.add_argument("--case-reps", type=int, default=2)
    ap.add_argument("--case-rows", type=int, default=None,
                    help="table rows of the gather case (default 1M) and of the fused case (default 4M)")
    args = ap.parse_args()
    if args.case == "bulk":
        run_bulk(args)
        return
    if args.case == "uncompressed":
        run_uncompressed(args)
        return
    if args.case == "fused":
        run_fused(args)
        return
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
