#!/usr/bin/env python3
"""Benchmark: SAGA + Atop-N decode attention, microseconds per decode step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl ours|reference]

A step is one decode token of the Atop-N loop: the refresh step (exact radix
select of the N-th largest logit, then the decode with it) when t mod n == 0,
otherwise the fused reuse step, always followed by the kept-entry softmax and
gathered value sum.  Warm-up runs steps 0..W-1; the timed region runs steps
W..W+K-1 as one CUDA-graph replay (the pages time their decode loop as
captured CUDA graphs), timed with CUDA events on the capture stream, max over
ranks, and reported as `window`.  The headline value is the schedule's mix,
one refresh step and n - 1 reuse steps per n tokens, each kind timed as
CUDA-graph replays in the same run, so that it does not depend on where the
window falls in the refresh period.  Inputs (K and V caches of 3 GB at the
default workload) are larger than the 126 MB L2, so no flush is needed
between steps; caches under 4x L2 are timed one graph per step with an L2
flush between.  The end-to-end leg runs whole refresh periods through
AtopNDecoder.host_loop (queries from, outputs to pinned host memory).

Prints ONE JSON line (rank 0).  N > 1 runs independent replicas (one batch
per GPU, no collective on the data path; weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

from sparse_decode_attention_saga_b200.workload import CONFIGS, bf16_bits, make_cache, make_queries

DEFAULT_CONFIG = "llama_b16_128k"
L2_BYTES = 126 * 1024 * 1024
METRIC = "Atop-N SAGA decode attn µs/step, HBM GB/s (% peak) at 128K ctx, batch 1/16"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=320)   # 10 runs x 32 tokens
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", action="store_true",
                    help="run a small case once (no timing) for ncu captures: refresh step, "
                         "two reuse steps and one dense call")
    ap.add_argument("--profile-batch", type=int, default=4)
    return ap.parse_args()


def run_profile_case(args):
    """The case the profiles/ captures use: the workload at a smaller batch
    (inputs still larger than L2), steps 0..2 and one dense call."""
    from sparse_decode_attention_saga_b200 import _lib
    from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
    w = CONFIGS[args.config].scaled(batch=args.profile_batch)
    K, V = make_cache(w, args.seed, "cuda")
    qs = make_queries(w, args.seed, "cuda", steps=3)
    dec = AtopNDecoder.for_workload(w)
    for t in range(3):
        dec.step(t, qs[t], K, V)
    try:
        dec.dense(qs[0], K, V)
    except _lib.SagaError:  # shapes the dense kernel does not take
        pass
    torch.cuda.synchronize()
    assert dec.error() == _lib.SAGA_OK
    return 0


def measured_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu record,
    or None if the record is for another workload or the kernel sources have
    changed since the counters were taken."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    path = os.path.join(root, "profiles", f"traffic_qk_stream_select_{workload}.json")
    try:
        rec = json.load(open(path))
        h = hashlib.sha256(b"".join(open(os.path.join(root, p), "rb").read()
                                    for p in rec["sources"])).hexdigest()
        return float(rec["bytes_per_launch"]) if h == rec["sources_sha256"] else None
    except Exception:
        return None


def peaks():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nvml:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nvml:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Largest value over the ranks (device time of the slowest replica)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle

def host_cores() -> int:
    """Host cores this process may run on; the oracle is given as many threads."""
    return len(os.sched_getaffinity(0))


def oracle_sample_us_per_step(w, seed, steps_sample, t0):
    """Times the CPU oracle on one batch element for `steps_sample` steps
    starting at step t0 (refresh steps included as the schedule says) and
    scales to the whole batch.  Returns (us_per_step, cores, description)."""
    import oracle  # test infrastructure: only this leg of the benchmark runs it
    oracle.set_num_threads(host_cores())
    ws = w.scaled(batch=1)
    K, V = make_cache(ws, seed)
    qs = make_queries(ws, seed, steps=t0 + steps_sample)
    Kh, Vh = bf16_bits(K), bf16_bits(V)
    tau = np.full((1, w.h_q), np.nan, np.float32)
    # state entering t0: refresh at the last multiple of n before t0
    t_last = (t0 // w.n) * w.n
    oracle.atopn_step(bf16_bits(qs[t_last]), Kh, Vh, tau, w.N, t_last, w.n)
    times = []
    for t in range(t0, t0 + steps_sample):
        a = time.perf_counter()
        oracle.atopn_step(bf16_bits(qs[t]), Kh, Vh, tau, w.N, t, w.n)
        times.append(time.perf_counter() - a)
    us = float(np.mean(times)) * 1e6 * w.batch
    desc = (f"oracle steps {t0}..{t0 + steps_sample - 1} on 1 of {w.batch} batch elements "
            f"(all {w.h_q} query heads, l_kv={w.l_kv}), scaled x{w.batch}")
    return us, oracle.num_threads(), desc


def oracle_single_thread_us(w, seed, t0):
    """The oracle's step t0 on one batch element on one host thread, scaled
    to the whole batch (the state entering t0 is set up on all threads).
    Returns (us_per_step, description)."""
    import oracle  # test infrastructure: only this leg of the benchmark runs it
    ws = w.scaled(batch=1)
    K, V = make_cache(ws, seed)
    qs = make_queries(ws, seed, steps=t0 + 1)
    Kh, Vh = bf16_bits(K), bf16_bits(V)
    tau = np.full((1, w.h_q), np.nan, np.float32)
    t_last = (t0 // w.n) * w.n
    if t_last < t0:
        oracle.atopn_step(bf16_bits(qs[t_last]), Kh, Vh, tau, w.N, t_last, w.n)
    threads = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        a = time.perf_counter()
        oracle.atopn_step(bf16_bits(qs[t0]), Kh, Vh, tau, w.N, t0, w.n)
        us = (time.perf_counter() - a) * 1e6 * w.batch
    finally:
        oracle.set_num_threads(threads)
    return us, (f"oracle step {t0} on 1 of {w.batch} batch elements, one thread, "
                f"scaled x{w.batch}")


# ------------------------------------------------------------------ reference arm

def run_reference(args, world, rank):
    """The oracle as it stands on the host cores, on the whole batch of the
    workload: steps W, W+1, ... each timed on its own (the state entering
    step W set up first, untimed), as many of the K steps as fit in about
    two minutes of host time."""
    if rank != 0:
        return 0
    import oracle  # test infrastructure: the reference arm is the oracle
    w = CONFIGS[args.config]
    cores = host_cores()
    oracle.set_num_threads(cores)
    K, V = make_cache(w, args.seed)
    qs = make_queries(w, args.seed, steps=args.warmup + args.steps)
    Kh, Vh = bf16_bits(K), bf16_bits(V)
    del K, V
    tau = np.full((w.batch, w.h_q), np.nan, np.float32)
    t_last = (args.warmup // w.n) * w.n
    if t_last < args.warmup:
        oracle.atopn_step(bf16_bits(qs[t_last]), Kh, Vh, tau, w.N, t_last, w.n)
    times, budget_s = [], 120.0
    for t in range(args.warmup, args.warmup + args.steps):
        a = time.perf_counter()
        oracle.atopn_step(bf16_bits(qs[t]), Kh, Vh, tau, w.N, t, w.n)
        times.append(time.perf_counter() - a)
        if sum(times) > budget_s:
            break
    us = float(np.mean(times)) * 1e6
    refreshes = sum(1 for t in range(args.warmup, args.warmup + len(times)) if t % w.n == 0)
    desc = (f"oracle steps {args.warmup}..{args.warmup + len(times) - 1} ({len(times)} of the "
            f"{args.steps} requested, {refreshes} refresh) on the whole batch ({w.batch} x {w.h_q} "
            f"rows, l_kv={w.l_kv}), each step timed on its own")
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us/step",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_k": w.h_k,
                   "h_v": w.h_v, "head_dim": w.head_dim, "v_head_dim": w.dv, "l_kv": w.l_kv,
                   "N": w.N, "n": w.n,
                   "parallelism": "replicas" if args.gpus > 1 else "single",
                   "l2": "host memory (the oracle runs on the CPU)",
                   "timing": "time.perf_counter around each oracle step, mean over the timed steps"},
        "cpu_baseline": {"value": us, "unit": "us/step", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "timed_steps": len(times),
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def distinct_value_rows(idx, cnt, w):
    """Distinct (batch, value head, position) rows kept by any query head."""
    b, hq, l = w.batch, w.h_q, w.l_kv
    vh = torch.arange(hq, device="cuda") * w.h_v // hq
    valid = torch.arange(l, device="cuda")[None, None, :] < cnt[..., None]
    rows = torch.zeros(b, w.h_v, l, dtype=torch.bool, device="cuda")
    bi = torch.arange(b, device="cuda")[:, None, None].expand(b, hq, l)
    vi = vh[None, :, None].expand(b, hq, l)
    pi = idx.long().clamp(min=0)
    rows[bi[valid], vi[valid], pi[valid]] = True
    return int(rows.sum().item()), int(cnt.sum().item())


def run_ours(args, world, rank, local):
    from sparse_decode_attention_saga_b200 import _lib
    from sparse_decode_attention_saga_b200.decoder import AtopNDecoder

    w = CONFIGS[args.config]
    seed = args.seed + rank
    total_steps = args.warmup + args.steps
    # the end-to-end loop runs whole refresh periods: from the first refresh
    # step at or after W, as many periods as cover K steps
    e2e_t0 = -(-args.warmup // w.n) * w.n
    e2e_steps = -(-args.steps // w.n) * w.n
    K, V = make_cache(w, seed, "cuda")
    qs = make_queries(w, seed, "cuda", steps=max(total_steps, e2e_t0 + e2e_steps))
    dec = AtopNDecoder.for_workload(w)
    stream = torch.cuda.Stream()
    # the inputs and the decoder's zeroed workspace were made on the default
    # stream; everything below runs on `stream`
    torch.cuda.synchronize()
    launches0 = _lib.launch_count()

    with torch.cuda.stream(stream):
        # warm-up (eager), steps 0..W-1; also caches device properties
        for t in range(args.warmup):
            dec.step(t, qs[t], K, V)
        dense_out = torch.empty_like(dec.out)
        try:
            dec.dense(qs[0], K, V, out=dense_out)
            has_dense = True
        except _lib.SagaError:  # shapes the dense kernel does not take
            has_dense = False
    stream.synchronize()
    assert dec.error() == _lib.SAGA_OK

    # Caches that are not much larger than L2 are timed cold: every step is
    # its own CUDA graph, replayed between its own events with an L2 flush (a
    # write, then a read, each twice L2) outside them.  Larger caches stream
    # past L2 anyway and are timed as one CUDA-graph replay of the K steps.
    cache_bytes = (K.numel() + V.numel()) * 2
    cold = cache_bytes < 4 * L2_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if cold else None
    flush_rd = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda") if cold else None
    flush_sink = torch.empty((), dtype=torch.float32, device="cuda")

    def flush():
        # a write larger than L2 evicts every line of the inputs; the read
        # after it replaces the dirty lines it leaves with clean ones, so the
        # timed step does not pay for writing the flush back to HBM
        flush_buf.fill_(1)
        torch.sum(flush_rd, dim=0, out=flush_sink)

    def capture(calls):
        """One CUDA graph of the calls (on the launching stream), replayed once
        untimed so that its first, uploading launch stays out of the timing."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for call in calls:
                call()
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        return g

    # The untimed replays run the same steps in the same order before the
    # timed ones; both start on a refresh step when W is a multiple of n.
    before = _lib.launch_count()
    steps = [lambda t=t: dec.step(t, qs[t], K, V) for t in range(args.warmup, total_steps)]
    if not cold:
        graph = capture(steps)
    else:
        step_graphs = [capture([s]) for s in steps]
    gpu_launches = _lib.launch_count() - before
    refresh_steps = sum(1 for t in range(args.warmup, total_steps) if t % w.n == 0)

    # The untimed replays left the thresholds of the window's last refresh;
    # put back those that enter step W (the refresh that opened its period),
    # as in a decode that has just run steps 0..W-1.
    t_open = args.warmup - args.warmup % w.n
    if t_open < args.warmup:
        with torch.cuda.stream(stream):
            dec.refresh(qs[t_open], K)
        stream.synchronize()

    dec.empty_rows(stream)  # clears the count of the untimed replays
    sampler = ClockSampler(local)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        with torch.cuda.stream(stream):   # replay, and its events, on the capture stream
            if not cold:
                ev0.record(stream)
                graph.replay()
                ev1.record(stream)
                torch.cuda.synchronize()
                ms = ev0.elapsed_time(ev1)
            else:
                ms = 0.0
                for g in step_graphs:
                    flush()
                    ev0.record(stream)
                    g.replay()
                    ev1.record(stream)
                    ev1.synchronize()
                    ms += ev0.elapsed_time(ev1)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ms, world)
    us_window = ms * 1e3 / args.steps
    empty_rows = dec.empty_rows(stream)
    assert dec.error() == _lib.SAGA_OK

    # ---- separately timed step kinds (CUDA-graph replays like the timed
    # loop, events on the launching stream)
    def time_steps(fn, reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            fn(0)  # one call outside any capture
        stream.synchronize()
        calls = [lambda r=r: fn(r) for r in range(reps)]
        if cold:
            total = 0.0
            for g in [capture([c]) for c in calls]:
                with torch.cuda.stream(stream):
                    flush()
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                e1.synchronize()
                total += e0.elapsed_time(e1)
            return total * 1e3 / reps
        g = capture(calls)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) * 1e3 / reps

    reuse_t = [t for t in range(1, w.n)]
    us_reuse = time_steps(lambda r: dec.step(reuse_t[r % len(reuse_t)], qs[reuse_t[r % len(reuse_t)]], K, V), 20)
    us_refresh = time_steps(lambda r: dec.step(0, qs[0], K, V), 5)
    us_dense = (time_steps(lambda r: dec.dense(qs[r % 4], K, V, out=dense_out), 10)
                if has_dense else None)
    # The headline: one refresh step and n - 1 reuse steps per n tokens, as
    # the schedule runs them (the K-step window above holds however many
    # refreshes its position in the period gives it)
    us_mix = max_over_ranks((us_refresh + (w.n - 1) * us_reuse) / w.n, world)
    us_per_step = us_mix

    # Dense grouped-query attention of the layer SAGA was converted from
    # (h_k = h_v): the pages' full-attention baseline.  Its own cache (more
    # key heads) is drawn with the same recipe.
    if has_dense and w.h_k != w.h_v:
        wg = w.scaled(h_k=w.h_v)
        Kg, Vg = make_cache(wg, seed, "cuda")
        gdec = AtopNDecoder.for_workload(wg)
        gqa_out = torch.empty_like(gdec.out)
        torch.cuda.synchronize()  # its cache and workspace come from the default stream
        us_dense_gqa = time_steps(lambda r: gdec.dense(qs[r % 4], Kg, Vg, out=gqa_out), 10)
        assert gdec.error() == _lib.SAGA_OK
        del Kg, Vg, gdec, gqa_out
        torch.cuda.empty_cache()
    else:
        us_dense_gqa = us_dense
    ratio = (lambda us: None if us is None else us / us_per_step)

    # ---- dominant kernel: the fused compare kernel of the reuse step
    kern_us = []
    ks, ke = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ks.record(stream)
        ke.record(stream)  # materialise the events before handing them to the library
    stream.synchronize()
    for r in range(20):
        t = reuse_t[r % len(reuse_t)]
        if cold:
            with torch.cuda.stream(stream):
                flush()
        with torch.cuda.stream(stream):
            _lib.set_kernel_events(ks, ke)
            dec.step(t, qs[t], K, V)
            _lib.set_kernel_events(None, None)
        stream.synchronize()
        kern_us.append(ks.elapsed_time(ke) * 1e3)
    kern_us = float(np.mean(kern_us[2:]))

    # kept entries and distinct value rows of a reuse step (measured, not timed)
    idx = torch.empty((w.batch, w.h_q, w.l_kv), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.batch, w.h_q), dtype=torch.int32, device="cuda")
    with torch.cuda.stream(stream):
        dec.step(reuse_t[0], qs[reuse_t[0]], K, V, sel_idx=idx, sel_cnt=cnt)
    stream.synchronize()
    U, kept = distinct_value_rows(idx, cnt, w)
    del idx

    k_bytes = w.batch * w.l_kv * w.h_k * w.head_dim * 2
    small = w.batch * w.h_q * (w.head_dim * 2 + 4)            # q + tau
    kern_bytes = k_bytes + small + kept * 8                   # + kept (pos, logit) lists
    step_ideal = k_bytes + U * w.dv * 2 + w.batch * w.h_q * (w.head_dim * 2 + w.dv * 4 + 4)
    refresh_ideal = step_ideal + 2 * w.batch * w.h_q * w.l_kv * 4   # + logits written and read once
    peak, peak_kind = peaks()
    achieved = kern_bytes / (kern_us * 1e-6) / 1e9

    # ---- end to end through the public API with host buffers
    q_host = qs.cpu().pin_memory()
    out_host = torch.empty((e2e_steps,) + tuple(dec.out.shape), dtype=torch.float32).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    barrier(world)
    torch.cuda.synchronize()
    if not cold:
        # launched like the timed loop above: the K steps as one CUDA graph
        # (AtopNDecoder.host_loop: each step's query copied in from pinned
        # host memory and its output copied out, on two copy streams with
        # double buffers, overlapping the neighbouring steps' kernels)
        # The thresholds entering step W (the refresh that opened its period)
        # are put in place outside the timed region before each replay.
        loop = dec.host_loop(K, V, q_host, out_host, e2e_t0, e2e_steps, stream=stream,
                             restore=False)
        loop.restore_state()
        loop.replay()             # untimed: the first launch uploads the graph
        stream.synchronize()
        loop.restore_state()
        with torch.cuda.stream(stream):
            e0.record(stream)
            loop.replay()
            e1.record(stream)
        stream.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        del loop
    else:
        # cold like the timed loop above: one host loop of one step per step,
        # L2 flushed before every step outside the events
        loops = [dec.host_loop(K, V, q_host, out_host[k:k + 1], e2e_t0 + k, 1, stream=stream,
                               restore=False) for k in range(e2e_steps)]
        loops[0].restore_state()  # each later step follows its predecessor
        for lp in loops:          # untimed first launches, in step order
            lp.replay()
        stream.synchronize()
        loops[0].restore_state()
        e2e_ms = 0.0
        for lp in loops:
            with torch.cuda.stream(stream):
                flush()
                e0.record(stream)
                lp.replay()
                e1.record(stream)
            e1.synchronize()
            e2e_ms += e0.elapsed_time(e1)
        del loops
    barrier(world)
    e2e_us = max_over_ranks(e2e_ms * 1e3 / e2e_steps, world)
    # Each step's own output reached the host: the last two steps (one per
    # buffer), recomputed now from the same thresholds, equal it bit for bit
    # (checked when both are reuse steps after the same refresh).
    last = [(k, e2e_t0 + k) for k in (e2e_steps - 2, e2e_steps - 1)]
    if e2e_steps >= 2 and all(t % w.n for _, t in last) and last[0][1] // w.n == last[1][1] // w.n:
        with torch.cuda.stream(stream):
            for k, t in last:
                o = dec.step(t, qs[t], K, V).cpu()
                assert torch.equal(o, out_host[k]), f"end-to-end output of step {t}"

    # ---- decode with cache growth: each step appends its own K/V rows and attends
    # over l + 1 positions.  The cache memory is reused: the decoder starts at
    # l_kv - G and re-appends rows l_kv - G .. l_kv - 1 (the same values).
    G = 32
    rows_k = K[:, w.l_kv - G:w.l_kv].transpose(0, 1).contiguous()   # [G, b, h_k, d]
    rows_v = V[:, w.l_kv - G:w.l_kv].transpose(0, 1).contiguous()
    grow_us = []
    for rep in range(2):  # the first pass warms up
        gdec = AtopNDecoder(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, w.l_kv - G, w.N, w.n,
                            l_cap=w.l_kv, v_head_dim=w.dv)
        torch.cuda.synchronize()  # rows and workspace come from the default stream
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g0.record(stream)
            for t in range(G):
                gdec.append(rows_k[t], rows_v[t], K, V)
                gdec.step(t, qs[t % qs.shape[0]], K, V)
            g1.record(stream)
        stream.synchronize()
        assert gdec.error() == _lib.SAGA_OK
        grow_us.append(g0.elapsed_time(g1) * 1e3 / G)
        del gdec
    del rows_k, rows_v

    line = {
        "metric": METRIC, "value": us_per_step, "unit": "us/step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": us_per_step / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "h_q": w.h_q, "h_k": w.h_k,
                   "h_v": w.h_v, "head_dim": w.head_dim, "v_head_dim": w.dv, "l_kv": w.l_kv,
                   "N": w.N, "n": w.n,
                   "parallelism": f"replicas x{world}" if world > 1 else "single",
                   "l2": ("inputs larger than L2 (K+V cache %.2f GB)" % (cache_bytes / 1e9)) if not cold
                         else ("L2 flushed before every timed step: a write, then a read, each "
                               "twice L2 (K+V cache %.3f GB)" % (cache_bytes / 1e9)),
                   "timing": ("one CUDA-graph replay of K steps, CUDA events" if not cold
                              else "one CUDA graph per step, CUDA events around each replay, "
                                   "summed over K steps")},
        "value_from": ("one refresh step and n - 1 reuse steps per n tokens, each kind timed as "
                       "CUDA-graph replays (us_refresh_step, us_reuse_step)"),
        "window": {"us_per_step": us_window, "steps": args.steps, "first_step": args.warmup,
                   "refresh_steps": refresh_steps,
                   "what": "the K timed steps W..W+K-1 as one replay (or one replay per step, cold)"},
        "empty_set_rows": {"total": int(empty_rows), "steps": args.steps,
                           "per_step": empty_rows / args.steps,
                           "what": "rows whose threshold lay above every logit (the empty-set rule "
                                   "kept their maxima), counted by the library over the K timed steps"},
        "refresh_steps": refresh_steps,
        "gpu_launches": int(gpu_launches),
        "us_reuse_step": us_reuse, "us_refresh_step": us_refresh,
        "us_mean_step_1_in_n": us_mix,
        "us_dense_step": us_dense, "speedup_vs_dense": ratio(us_dense),
        "us_dense_gqa_step": us_dense_gqa, "speedup_vs_dense_gqa": ratio(us_dense_gqa),
        "dense_gqa": f"h_k = h_v = {w.h_v} (the GQA layer before key-head merging)",
        "kept_entries_per_step": kept, "distinct_value_rows": U,
        "roofline": {"kernel": "qk_stream_kernel (fused compare, reuse step)", "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "bytes_per_launch": kern_bytes, "us_per_launch": kern_us,
                     "traffic": measured_traffic(w.name)},
        "step_roofline": {"what": "reuse step (streaming kernel + gather with row merge) vs ideal bytes "
                                  "K + distinct kept V rows + q/tau/out",
                          "ideal_bytes": step_ideal, "us": us_reuse,
                          "achieved": step_ideal / (us_reuse * 1e-6) / 1e9,
                          "frac": step_ideal / (us_reuse * 1e-6) / 1e9 / peak},
        "refresh_roofline": {"what": "refresh step (logits to HBM, radix select, compare/compact, "
                                     "gather with row merge) vs the reuse step's ideal bytes, and vs "
                                     "those plus one write and one read of the logits",
                             "ideal_bytes": step_ideal, "ideal_bytes_with_logits": refresh_ideal,
                             "us": us_refresh,
                             "frac": step_ideal / (us_refresh * 1e-6) / 1e9 / peak,
                             "frac_with_logits": refresh_ideal / (us_refresh * 1e-6) / 1e9 / peak},
        "grow": {"us_per_step": grow_us[-1], "steps": G, "l_kv": [w.l_kv - G + 1, w.l_kv],
                 "what": "append this step's K/V rows, then the Atop-N step over the grown "
                         "cache (refresh every n), eager, CUDA events"},
        "e2e": {"value": e2e_us, "unit": "us/step",
                "h2d_bytes_per_step": int(qs[0].numel() * 2),
                "d2h_bytes_per_step": int(dec.out.numel() * 4),
                "steps": e2e_steps, "first_step": e2e_t0,
                "timing": ("whole refresh periods (steps from the first refresh step at or after W, "
                           "K rounded up to a multiple of n) as one CUDA-graph replay, each step with "
                           "its own copies in and out of pinned host memory on two copy streams "
                           "(double buffers, overlapping the neighbouring steps' kernels)") if not cold
                          else ("whole refresh periods (as above), one host loop (CUDA graph) per step "
                                "with its copies, CUDA events around each replay, L2 flushed before "
                                "each")},
        "clocks": sampler.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        us_cpu, cores, desc = oracle_sample_us_per_step(w, args.seed, 2, w.n - 1)
        us_one, desc_one = oracle_single_thread_us(w, args.seed, w.n - 1)
        line["cpu_baseline"] = {"value": us_cpu, "unit": "us/step", "cores": cores,
                                "kind": "oracle", "sample": desc,
                                "single_thread": {"value": us_one, "unit": "us/step",
                                                  "sample": desc_one}}
    if not cold:
        del graph
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.profile_case:
            return run_profile_case(args)
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
