#!/usr/bin/env python3
"""Benchmark: CSA+HCA hybrid-attention decode at a 1,048,576-token context.

One step is one decode token of every sequence through one CSA layer and one
HCA layer.  Steps walk through a window of 128 consecutive positions centred
on 1,048,576 (contexts 1,048,513 .. 1,048,640), one HCA period, so that the
compressors run exactly where an entry completes: CSA compression on the 32
tokens that close a 4-token group, HCA compression on the one token that
closes a 128-token block.  Every step runs
  CSA layer: [csa_compress] -> indexer_score + indexer_select (= indexer_topk:
             score the ~262,144 visible entries, keep 1,024)
             -> hybrid_attn_decode (1,024 + 128 window)
  HCA layer: [hca_compress] -> hybrid_attn_decode (8,192 dense + 128 window)
The metric is decode queries/s (one query = one token through both layers).

Inputs are seeded synthetic tensors resident in HBM.  R replicas of every
layer's inputs rotate between steps; their per-step bytes total more than 4x
the 126 MB L2, so each step reads HBM.  The timed region replays CUDA graphs
of 128 steps (plus one graph of the remaining steps), exactly K steps.  The
dominant kernel, the indexer's HBM scan (the indexer_score call), is
bracketed by event records inside the graph.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own sequences (weak scaling, no data-path
collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "CSA+HCA decode queries/s at 1M ctx; achieved HBM GB/s vs B200 peak"
UNIT = "queries/s"


# ------------------------------------------------------------------ helpers

_FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def max_over_ranks(ms, dev, world):
    """The slowest rank's time (every rank takes this collective step)."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, ms, world):
    """Units of all ranks per second over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def rank_seed(base, rank):
    """Each rank's replicas draw their own inputs (independent sequences)."""
    return base + 7919 * rank


def _peaks(kind="hbm_gbs"):
    """A measured peak from MEASURED_PEAKS.json (HBM copy GB/s, or cuBLAS bf16
    TFLOP/s as a burst or sustained), else the earlier measurement on this
    pool that stands in for it."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if kind in d:
            return float(d[kind]), "measured"
    return _FALLBACK_PEAKS[kind], "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the GPU is loaded."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- our path

PERIOD = 128       # one HCA block: every compression pattern of the window repeats


class Schedule:
    """Positions of the decode window: step s queries position T0 + s with
    ctx_len T0 + s + 1 (T0 = T - 64, T the workload context)."""

    def __init__(self, wl, dev):
        self.T0 = wl.T - PERIOD // 2
        self.q_pos, self.ctx, self.tb, self.te = [], [], [], []
        self.csa_fires, self.hca_fires = [], []
        for step in range(PERIOD):
            p = self.T0 + step
            self.q_pos.append(torch.full((wl.B, 1), p, dtype=torch.int64, device=dev))
            self.ctx.append(torch.full((wl.B,), p + 1, dtype=torch.int64, device=dev))
            self.tb.append(torch.full((wl.B,), p, dtype=torch.int64, device=dev))
            self.te.append(torch.full((wl.B,), p + 1, dtype=torch.int64, device=dev))
            self.csa_fires.append((p + 1) // wl.csa_stride > p // wl.csa_stride)
            self.hca_fires.append((p + 1) // wl.hca_stride > p // wl.hca_stride)

    @property
    def t_end(self):
        return self.T0 + PERIOD


class Replica:
    """One sequence batch's CSA and HCA layer inputs on the device, holding
    every position of the decode window."""

    def __init__(self, wl, sched, seed, dev):
        from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
        wlw = wl.with_(T=sched.t_end)
        self.csa_L = W.make_csa_layer(wlw, device=dev, seed=seed)
        self.hca_L = W.make_hca_layer(wlw, device=dev, seed=seed + 500_000)
        self.csa = CSALayer(self.csa_L)
        self.hca = HCALayer(self.hca_L)
        self.sched = sched

    def step(self, s, hook=None, pos=None, split_select=True):
        """Enqueue decode step s of the window on the current stream.
        hook(name) runs before each call (names in CALLS) and hook("end")
        after the last.  indexer_score + indexer_select is the indexer_topk
        call (one call, "indexer_topk", when split_select is False).
        pos = (q_pos, ctx_len, t_begin, t_end) device tensors replace the
        schedule's."""
        sc = self.sched
        q_pos, ctx, tb, te = pos if pos is not None else (sc.q_pos[s], sc.ctx[s], sc.tb[s],
                                                          sc.te[s])
        mark = hook or (lambda name: None)
        if sc.csa_fires[s]:
            mark("csa_compress")
            self.csa.compress(tb, te, 1)
        if split_select:
            mark("indexer_score")
            self.csa.select(q_pos, phase="score")
            mark("indexer_select")
            self.csa.select(q_pos, phase="pick")
        else:
            mark("indexer_topk")
            self.csa.select(q_pos)
        mark("csa_attention")
        self.csa.attend(pos=ctx)
        if sc.hca_fires[s]:
            mark("hca_compress")
            self.hca.compress(tb, te, 1)
        mark("hca_attention")
        self.hca.attend(pos=ctx)
        mark("end")


def _rt():
    from cuda.bindings import runtime as rt
    return rt


def _ok(res, what):
    err = res[0] if isinstance(res, tuple) else res
    if int(err) != 0:
        raise RuntimeError(f"{what}: {err}")
    return res[1] if isinstance(res, tuple) and len(res) == 2 else res


EVENT_EVERY = 2   # steps between in-graph event pairs around the indexer scoring call
CALLS = ("csa_compress", "indexer_score", "indexer_select", "csa_attention", "hca_compress",
         "hca_attention")


class StepGraph:
    """CUDA graph of G consecutive decode steps (step i of the timed sequence
    uses replica i % R and window position i % PERIOD).  In every
    EVENT_EVERY-th step, external event records on a side stream mark the end
    of the call before the indexer scoring and the end of the scoring: each
    record only depends on the kernels before it, so the main chain keeps its
    programmatic launch overlap and the pair measures the scoring call's share
    of the step as it runs."""

    def __init__(self, replicas, G, stream, i0=0):
        rt = _rt()
        self.G = G
        timed = [i for i in range(G) if i % EVENT_EVERY == 0]
        self.events = [[_ok(rt.cudaEventCreate(), "event") for _ in range(2)] for _ in timed]
        self.side = torch.cuda.Stream(device=stream.device)
        side = rt.cudaStream_t(self.side.cuda_stream)
        self.forks = [_ok(rt.cudaEventCreateWithFlags(rt.cudaEventDisableTiming), "event")
                      for _ in range(2 * len(timed) + 1)]
        forks = iter(self.forks)
        sh = rt.cudaStream_t(stream.cuda_stream)

        def mark_on_side(ev):
            f = next(forks)
            _ok(rt.cudaEventRecord(f, sh), "fork")
            _ok(rt.cudaStreamWaitEvent(side, f, 0), "fork wait")
            _ok(rt.cudaEventRecordWithFlags(ev, side, rt.cudaEventRecordExternal), "record")

        def hook_for(ev):
            def hook(name):
                if name == "indexer_score":
                    mark_on_side(ev[0])
                elif name == "indexer_select":
                    mark_on_side(ev[1])
            return hook

        with torch.cuda.stream(stream):
            _ok(rt.cudaStreamBeginCapture(
                sh, rt.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal), "capture")
            for i in range(G):
                rep = replicas[(i0 + i) % len(replicas)]
                if i % EVENT_EVERY:
                    rep.step((i0 + i) % PERIOD)
                    continue
                rep.step((i0 + i) % PERIOD, hook=hook_for(self.events[i // EVENT_EVERY]))
            # join the side stream back before the capture ends
            j = next(forks)
            _ok(rt.cudaEventRecord(j, side), "join")
            _ok(rt.cudaStreamWaitEvent(sh, j, 0), "join wait")
            self.graph = _ok(rt.cudaStreamEndCapture(sh), "end capture")
        self.exec = _ok(rt.cudaGraphInstantiate(self.graph, 0), "instantiate")
        self.kernels = self._count_kernels()
        self.sh = sh

    def _count_kernels(self):
        rt = _rt()
        res = rt.cudaGraphGetNodes(self.graph)
        n = res[-1]
        res = rt.cudaGraphGetNodes(self.graph, n)
        nodes = res[1]
        kern = 0
        for nd in nodes:
            t = _ok(rt.cudaGraphNodeGetType(nd), "node type")
            if t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                kern += 1
        return kern

    def launch(self):
        _ok(_rt().cudaGraphLaunch(self.exec, self.sh), "graph launch")

    def indexer_ms(self):
        rt = _rt()
        return [_ok(rt.cudaEventElapsedTime(a, b), "elapsed") for a, b in self.events]


class CallGraph:
    """CUDA graph of G decode steps with an event recorded on the step's own
    stream before every call and after the last one: each call then runs on
    its own (its kernels start once the previous call has finished), and
    consecutive events give its duration.  Replayed after the timed region;
    every replay adds one sample per call and step."""

    def __init__(self, replicas, G, stream, i0=0):
        rt = _rt()
        self.sh = rt.cudaStream_t(stream.cuda_stream)
        self.marks = []          # (name, event) in stream order
        with torch.cuda.stream(stream):
            _ok(rt.cudaStreamBeginCapture(
                self.sh, rt.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal), "capture")

            def hook(name):
                ev = _ok(rt.cudaEventCreate(), "event")
                _ok(rt.cudaEventRecordWithFlags(ev, self.sh, rt.cudaEventRecordExternal),
                    "record")
                self.marks.append((name, ev))

            for i in range(G):
                replicas[(i0 + i) % len(replicas)].step((i0 + i) % PERIOD, hook=hook)
            self.graph = _ok(rt.cudaStreamEndCapture(self.sh), "end capture")
        self.exec = _ok(rt.cudaGraphInstantiate(self.graph, 0), "instantiate")

    def run(self, samples):
        """Replay once and append each call's duration (ms) to samples[name]."""
        rt = _rt()
        _ok(rt.cudaGraphLaunch(self.exec, self.sh), "graph launch")
        _ok(rt.cudaStreamSynchronize(self.sh), "sync")
        for (name, a), (_, b) in zip(self.marks, self.marks[1:]):
            if name != "end":
                samples.setdefault(name, []).append(
                    _ok(rt.cudaEventElapsedTime(a, b), "elapsed"))


def ik_key_bytes(wl):
    """Bytes of one indexer key: FP8 codes and one fp32 scale per vector or
    per 64 dims, or MXFP4 codes (two per byte) and one E8M0 byte per 32 dims."""
    if wl.ik_fmt == "mxfp4":
        return wl.d_I // 2 + wl.d_I // 32
    return wl.d_I + 4 * (1 if wl.ik_fmt == "e4m3vec" else wl.d_I // 64)


def indexer_bytes(wl):
    """Algorithmic HBM bytes of one indexer scoring launch: every visible CSA
    entry's indexer key, the query heads in the same layout and the head
    weights.  (The scores, 4 bytes per entry, stay in L2 for the selection.)"""
    n_c = wl.T // wl.csa_stride
    q = wl.H_I * ik_key_bytes(wl) + 4 * wl.H_I
    return wl.B * (n_c * ik_key_bytes(wl) + q)


def call_bytes(wl):
    """Algorithmic bytes of one call of each kind in a decode step: what the
    definition must read and write once (a KV entry is 448 FP8 codes, 7 fp32
    block scales and 64 BF16 RoPE values = 604 bytes; an indexer key 128 codes
    and one or two scales).  The selection's scores live in L2."""
    entry = wl.d_nope + 2 * wl.d_rope + 4 * (wl.d_nope // 64)
    ik = ik_key_bytes(wl)
    n_c = wl.T // wl.csa_stride
    n_h = wl.T // wl.hca_stride
    q = wl.Hq * wl.D * 2
    out = wl.Hq * wl.D * 4 + wl.Hq * 4
    return {
        "csa_compress": wl.B * (wl.csa_pool * (entry + ik) + entry + ik) + 4 * (wl.D + wl.csa_pool),
        "indexer_score": indexer_bytes(wl),
        "indexer_select": wl.B * (4 * n_c + 8 * wl.k),
        "csa_attention": wl.B * (4 * wl.k + (wl.k + wl.window) * entry + q + out),
        "hca_compress": wl.B * (wl.hca_pool * entry + entry) + 4 * (wl.D + wl.hca_pool),
        "hca_attention": wl.B * ((n_h + wl.window) * entry + q + out),
    }


def step_bytes(wl):
    """Algorithmic HBM bytes of one decode step (both layers), compression
    averaged over the 128-step window (32 CSA entries and 1 HCA entry)."""
    cb = call_bytes(wl)
    fixed = sum(cb[n] for n in ("indexer_score", "csa_attention", "hca_attention"))
    fixed += wl.B * 4 * wl.k          # the selection's output (its scores stay in L2)
    compress = ((PERIOD // wl.csa_stride) * cb["csa_compress"]
                + (PERIOD // wl.hca_stride) * cb["hca_compress"]) / PERIOD
    return int(fixed + compress)


def per_call_report(wl, samples, peak):
    """Per-call mean duration and achieved bytes/s against the HBM peak."""
    cb = call_bytes(wl)
    out = {}
    for name in CALLS:
        v = samples.get(name)
        if not v:
            continue
        us = float(np.mean(v)) * 1e3
        gbs = cb[name] / (us * 1e-6) / 1e9
        out[name] = {"us": round(us, 3), "us_median": round(float(np.median(v)) * 1e3, 3),
                     "samples": len(v), "algorithmic_bytes": int(cb[name]),
                     "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    return out


def _time_decode(args, wl, rank, world, dev, steps, seed0, clocks=True, call_replays=None):
    """Build the rotating replicas of `wl`, warm up, capture the step graph and
    time exactly `steps` steps (max over ranks).  Returns the timing record."""
    per_rep_bytes = step_bytes(wl)
    # enough replicas that one rotation touches > 4x the 126 MB L2 (unless set)
    R = args.replicas if args.replicas > 0 else math.ceil(4 * 126e6 / per_rep_bytes) + 1
    sched = Schedule(wl, dev)
    replicas = [Replica(wl, sched, rank_seed(seed0 + r, rank), dev) for r in range(R)]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)
    # warm-up: W steps eagerly through the public API (also performs the
    # library's one-time kernel attribute set-up outside any graph capture)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            replicas[i % R].step(i % PERIOD)
    stream.synchronize()
    G = max(1, min(args.graph_steps, steps))
    graph = StepGraph(replicas, G, stream)
    rest = steps % G
    tail = StepGraph(replicas, rest, stream, i0=(steps // G) * G) if rest else None

    sampler = ClockSampler(dev.index if dev.index is not None else 0) if clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    # untimed graph replays so the clock sampler sees the GPU under load
    with torch.cuda.stream(stream):
        for _ in range(max(1, int(0.2 / max(1e-6, 30e-6 * G)))):
            graph.launch()
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    n_launch = steps // G
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(n_launch):
            graph.launch()
        if tail:
            tail.launch()
        t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = sampler.stop() if sampler else None
    ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    idx = graph.indexer_ms()
    # every call on its own: events before and after each call of PERIOD steps
    # (each replica set in turn, so the inputs still come from HBM), replayed
    calls = {}
    n_rep = args.call_replays if call_replays is None else call_replays
    if n_rep > 0:
        cg = CallGraph(replicas, PERIOD, stream)
        for _ in range(n_rep):
            cg.run(calls)
        del cg
    return {"ms": ms, "steps": n_launch * G + rest, "idx_ms": float(np.mean(idx)),
            "idx_samples": len(idx), "calls": calls,
            "clocks": clk, "replicas": replicas, "R": R, "sched": sched,
            "per_rep_bytes": per_rep_bytes,
            "launches": graph.kernels * n_launch + (tail.kernels if tail else 0)}


def _other_layouts(args, wl, rank, world, dev):
    """The same step with each other indexer layout (FP8 with the other scale
    granularity, FP4 MXFP4), timed briefly: the layout comparison rides along
    with the headline number."""
    peak, _ = _peaks()
    out = []
    for fmt in ("e4m3vec", "e4m3", "mxfp4"):
        if fmt == wl.ik_fmt:
            continue
        other = wl.with_(ik_fmt=fmt)
        t = _time_decode(args, other, rank, world, dev, args.alt_steps, 5000, clocks=False,
                         call_replays=0)
        ib = indexer_bytes(other)
        achieved = ib / (t["idx_ms"] / 1e3) / 1e9
        out.append({"indexer_layout": fmt, "indexer_scales": _scales_text(other),
                    "value": round(other.B * t["steps"] * world / (t["ms"] / 1e3), 2),
                    "unit": UNIT, "steps": t["steps"], "ms_per_step": t["ms"] / t["steps"],
                    "indexer_score_us": round(t["idx_ms"] * 1e3, 3),
                    "indexer_samples": t["idx_samples"],
                    "indexer_algorithmic_bytes": ib, "indexer_frac": round(achieved / peak, 4)})
        del t
        torch.cuda.empty_cache()
    return out


def _scales_text(wl):
    return {"e4m3vec": "FP8 E4M3, one fp32 scale per key / query head",
            "e4m3": "FP8 E4M3, one fp32 scale per 64 dims",
            "mxfp4": "FP4 MXFP4: E2M1 codes, one E8M0 exponent per 32 dims"}[wl.ik_fmt]


def run_ours(args, rank, world, dev):
    import compressed_sparse_kv_softmax_b200 as C  # noqa: F401  (fails loudly without the .so)
    wl = W.get(args.workload).with_(ik_fmt=args.ik_fmt)
    torch.cuda.set_device(dev)
    t = _time_decode(args, wl, rank, world, dev, args.steps, 1000)
    replicas, R, sched, per_rep_bytes = t["replicas"], t["R"], t["sched"], t["per_rep_bytes"]
    ms, steps_done, idx_ms, clocks = t["ms"], t["steps"], t["idx_ms"], t["clocks"]
    value = whole_job_rate(wl.B * steps_done, ms, world)

    peak, peak_kind = _peaks()
    ib = indexer_bytes(wl)
    achieved = ib / (idx_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "kernel": f"{_scoring_kernel(wl)} (lightning-indexer scoring: the "
                          f"indexer_score call, one launch)",
                "peak_kind": f"{peak_kind} HBM copy bandwidth (burst)",
                "algorithmic_bytes_per_launch": ib, "avg_launch_us": round(idx_ms * 1e3, 3),
                "samples": t["idx_samples"],
                "timed_launches": f"every {EVENT_EVERY}nd step of the last timed graph replay, "
                                  f"events on a side stream (no serialisation of the step)"}
    traffic = _profile_traffic(_scoring_kernel(wl), wl)
    if traffic is not None:
        roofline["traffic"] = traffic
    roofline["single_launch_floor"] = read_floor(ib, dev, peak)
    kernels = per_call_report(wl, t["calls"], peak)

    res = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
           "steps": steps_done, "warmup": args.warmup, "ms_per_step": ms / steps_done,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3/bf16 storage, fp32 math",
           "data": "synthetic (seeded Gaussian FP8 E4M3 + BF16 caches with needles)",
           "config": {"workload": f"{wl.name}: 1 CSA + 1 HCA layer decode, B={wl.B}/GPU, "
                                  f"ctx {sched.T0 + 1}..{sched.T0 + PERIOD} (128-token window "
                                  f"around {wl.T}: 32 CSA + 1 HCA compressions), Hq={wl.Hq}, "
                                  f"D={wl.d_nope}+{wl.d_rope}, H_I={wl.H_I}x{wl.d_I}, k={wl.k}, "
                                  f"window={wl.window}",
                      "indexer_scales": _scales_text(wl),
                      "global_batch": wl.B * world, "seq_len": wl.T,
                      "parallelism": f"replicas x{world} (weak)",
                      "l2": f"{R} rotating input replicas, {R * per_rep_bytes / 1e6:.0f} MB "
                            f"touched per cycle ({R * per_rep_bytes / 126e6:.1f}x the 126 MB L2)",
                      "step_bytes": per_rep_bytes},
           "roofline": roofline,
           "kernels": {"per_call": kernels,
                       "how": f"each call alone (events before and after it on the step's "
                              f"stream), {args.call_replays} replays of a {PERIOD}-step graph "
                              f"over the rotating replicas; frac = algorithmic bytes / time / "
                              f"{peak_kind} HBM copy bandwidth (the selection's scores are "
                              f"L2-resident)"},
           "gpu_launches": t["launches"],
           "clocks": clocks}
    del t
    if args.alt_steps > 0:
        res["other_indexer_layouts"] = _other_layouts(args, wl, rank, world, dev)
    return res, replicas, wl


def _scoring_kernel(wl):
    """The kernel that the indexer_score call launches for this workload."""
    if wl.ik_fmt == "mxfp4":
        return "indexer_mxf4_kernel"
    if wl.Tq > 1 and wl.ik_fmt == "e4m3vec":
        return "indexer_rows_kernel"
    return "indexer_tc_kernel"


def _profile_traffic(kernel, wl):
    """DRAM bytes per launch of `kernel` on this workload from the committed
    ncu record (profiles/ncu_traffic.json), when the kernel's sources still
    hash to the ones the counters were taken on; None otherwise (the
    counters describe another build)."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("workload") != wl.name or rec.get("ik_fmt", wl.ik_fmt) != wl.ik_fmt:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        h.update(open(os.path.join(ROOT, "compressed_sparse_kv_softmax_b200", "csrc", f), "rb").read())
    if h.hexdigest()[:16] != rec["sources_sha256_16"]:
        return None
    return int(rec["dram_bytes_per_launch"])


def read_floor(nbytes, dev, peak, reps=24):
    """What one launch that only reads `nbytes` reaches on this GPU: torch's
    fp32 sum over a buffer of that size, rotated over enough buffers that
    every launch reads HBM (more than 4x the L2).  Timed with CUDA events
    around each launch alone, and as the mean of launches back to back; both
    in GB/s and as a fraction of the same peak as the roofline.  A reference
    for the scoring launch, which reads the same bytes once per call."""
    if nbytes < (8 << 20):
        return {"what": "not measured: under 8 MB per launch (L2-resident scans)"}
    n = int(nbytes) // 4
    k = min(64, max(4, math.ceil(4 * 126e6 / (4 * n)) + 1))
    bufs = [torch.randn(n, device=dev) for _ in range(k)]
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for b in bufs:
            b.sum()
        stream.synchronize()
        alone = []
        for i in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            bufs[i % k].sum()
            e1.record(stream)
            stream.synchronize()
            alone.append(e0.elapsed_time(e1))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(reps):
            bufs[i % k].sum()
        e1.record(stream)
        stream.synchronize()
        b2b = e0.elapsed_time(e1) / reps
    del bufs
    us_alone, us_b2b = float(np.median(alone)) * 1e3, b2b * 1e3
    gbs = lambda us: 4 * n / (us * 1e-6) / 1e9
    return {"what": f"torch fp32 sum over {4 * n:,} bytes per launch, {k} buffers rotated "
                    f"(every launch reads HBM)",
            "us_alone": round(us_alone, 3), "frac_alone": round(gbs(us_alone) / peak, 4),
            "us_back_to_back": round(us_b2b, 3), "frac_back_to_back": round(gbs(us_b2b) / peak, 4)}


def _pack(tensors, device, pin=False):
    """One contiguous byte buffer holding the tensors (256-byte aligned
    sections) and views of it shaped like them."""
    offs, n = [], 0
    for t in tensors:
        offs.append(n)
        n = (n + t.numel() * t.element_size() + 255) & ~255
    buf = torch.empty(max(n, 256), dtype=torch.uint8, device=device, pin_memory=pin)
    views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for o, t in zip(offs, tensors)]
    return buf, views


def run_e2e(args, replicas, wl, dev, world):
    """Same metric through the public API with per-step host<->device copies.
    Every step: one host->device copy of the step's inputs from pinned host
    memory (both layers' queries, the indexer query, its scales and head
    weights, the positions, and the new token's raw KV and indexer key), the
    cskv_ring_store call that appends that token to the step's rings, the
    layer calls (csa_compress, indexer_topk, hybrid_attn_decode, hca_compress,
    hybrid_attn_decode), and one device->host copy of both layers' outputs.
    Steps rotate over the same replicas as the timed graph (HBM-resident
    inputs, more than 4x L2).  Timed twice: the calls launched eagerly on one
    stream, and replayed from CUDA graphs with the copies overlapping the
    neighbouring steps' kernels (the reported value)."""
    import compressed_sparse_kv_softmax_b200 as C
    K = max(3, min(args.steps, args.e2e_steps))
    sc = replicas[0].sched
    cl0, hl0 = replicas[0].csa_L, replicas[0].hca_L
    cap = cl0["ring_k"]["cap"]

    def token(L, key, s):
        # the new token of position T0 + s: its ring slot's planes, as a
        # one-slot cache per sequence
        slot = (sc.T0 + s) % cap
        c = L[key]
        return [c[p][:, slot:slot + 1] for p in ("data", "scale", "rope") if c.get(p) is not None]

    def small(s):
        return ([cl0["q"], hl0["q"], cl0["q_ik"], cl0["q_ik_scale"], cl0["head_w"], sc.q_pos[s],
                 sc.ctx[s], sc.tb[s], sc.te[s]] + token(cl0, "ring_k", s) + token(hl0, "ring_k", s)
                + token(cl0, "ring_ik", s))

    # the step's inputs in pinned host memory, taken before the layers are
    # pointed at the staging buffer
    host_small = []
    for s in range(PERIOD):
        hb, hv = _pack(small(s), "cpu", pin=True)
        for v, t in zip(hv, small(s)):
            v.copy_(t.cpu())
        host_small.append(hb)
    dev_buf, views = _pack(small(0), dev)
    dev_buf.copy_(host_small[0])
    q_c, q_h, q_ik, q_ik_s, head_w, q_pos, ctx, tb, te = views[:9]
    tok = views[9:]

    def one_slot(c, planes):
        d = {k: c[k] for k in ("fmt", "d_nope", "d_rope")}
        d.update(ring=False, cap=1, data=planes[0], scale=planes[1],
                 rope=planes[2] if len(planes) > 2 else None)
        return d

    src = [one_slot(cl0["ring_k"], tok[0:3]), one_slot(hl0["ring_k"], tok[3:6]),
           one_slot(cl0["ring_ik"], tok[6:8])]
    src = [C.cache_struct(c) for c in src]
    # every replica's layers read the step's inputs from the staging views and
    # write their outputs into one output buffer
    out_buf, out_views = _pack([replicas[0].csa.out, replicas[0].csa.lse, replicas[0].hca.out,
                                replicas[0].hca.lse], dev)
    rings = []
    for rep in replicas:
        cl, hl = rep.csa_L, rep.hca_L
        cl["q"], hl["q"], cl["q_ik"], cl["q_ik_scale"], cl["head_w"] = q_c, q_h, q_ik, q_ik_s, head_w
        rep.csa.out, rep.csa.lse, rep.hca.out, rep.hca.lse = out_views
        rings.append([rep.csa.cs["ring_k"], rep.hca.cs["ring_k"], rep.csa.cs["ring_ik"]])
    host_out = torch.empty(out_buf.shape, dtype=torch.uint8, pin_memory=True)
    bi = host_small[0].numel()
    bo = host_out.numel()
    stream = torch.cuda.Stream(device=dev)
    pos = (q_pos, ctx, tb, te)
    R = len(replicas)

    stores = []

    def one(i):
        s = i % PERIOD
        rep = replicas[i % R]
        dev_buf.copy_(host_small[s], non_blocking=True)
        stores[i % R]()
        rep.step(s, pos=pos, split_select=False)
        host_out.copy_(out_buf, non_blocking=True)

    with torch.cuda.stream(stream):
        # (the layers and the ring append marshal their arguments once per
        # set of buffers; a step then costs the host the launches)
        stores.extend(C.prepare("cskv_ring_store", wl.B, tb, src, r) for r in rings)
        for i in range(3):
            one(i)
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K):
            one(i)
        e1.record(stream)
    stream.synchronize()
    ms_eager = max_over_ranks(e0.elapsed_time(e1), dev, world)

    # The same steps replayed from CUDA graphs, as a serving loop runs them,
    # with the copies on streams of their own so that they overlap the
    # neighbouring steps' kernels.  Two device input buffers and two output
    # buffers alternate between steps; one graph per replica, buffer and
    # pattern of compressor firings (the only part of a step the host
    # decides) holds the step's public API calls (ring append and the layer
    # calls).  Per step i (buffer b = i % 2):
    #   host: waits until step i-2's outputs are back on the host (its inputs
    #         then are long consumed), writes step i's inputs into pinned
    #         staging b;
    #   H2D stream: once step i-2's kernels are done with device buffer b,
    #         copies the staging into it;
    #   compute stream: waits for that copy, replays the step's graph;
    #   D2H stream: after the graph, copies output buffer b to pinned host
    #         memory.
    # Step i+1's input copy is issued while step i computes.
    dev_bufs = [dev_buf, _pack(small(0), dev)[0]]
    out_bufs = [out_buf, _pack([replicas[0].csa.out, replicas[0].csa.lse, replicas[0].hca.out,
                                replicas[0].hca.lse], dev)[0]]
    host_in = [torch.empty_like(host_small[0]).pin_memory() for _ in range(2)]
    host_outs = [torch.empty(out_buf.shape, dtype=torch.uint8, pin_memory=True)
                 for _ in range(2)]

    def views_of(buf, like):
        out, o = [], 0
        for t in like:
            n = t.numel() * t.element_size()
            out.append(buf[o:o + n].view(t.dtype).view(t.shape))
            o = (o + n + 255) & ~255
        return out

    first = {}
    for s in range(PERIOD):
        first.setdefault((sc.csa_fires[s], sc.hca_fires[s]), s)
    graphs = {}
    rt = _rt()
    h2d, d2h = rt.cudaMemcpyKind.cudaMemcpyHostToDevice, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost
    hs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def copy(dst, src, n, kind, st):
        _ok(rt.cudaMemcpyAsync(dst.data_ptr(), src.data_ptr(), n, kind,
                               rt.cudaStream_t(st.cuda_stream)), "cudaMemcpyAsync")

    like_in = small(0)
    like_out = [replicas[0].csa.out, replicas[0].csa.lse, replicas[0].hca.out,
                replicas[0].hca.lse]
    with torch.cuda.stream(stream):
        for b in range(2):
            v = views_of(dev_bufs[b], like_in)
            ov = views_of(out_bufs[b], like_out)
            pos_b = tuple(v[5:9])
            tk = v[9:]
            src_b = [C.cache_struct(c) for c in (one_slot(cl0["ring_k"], tk[0:3]),
                                                 one_slot(hl0["ring_k"], tk[3:6]),
                                                 one_slot(cl0["ring_ik"], tk[6:8]))]
            for r in range(R):
                rep = replicas[r]
                cl, hl = rep.csa_L, rep.hca_L
                cl["q"], hl["q"], cl["q_ik"], cl["q_ik_scale"], cl["head_w"] = v[:5]
                rep.csa.out, rep.csa.lse, rep.hca.out, rep.hca.lse = ov
                store = C.prepare("cskv_ring_store", wl.B, pos_b[2], src_b, rings[r])
                for key, s in first.items():
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        store()
                        rep.step(s, pos=pos_b, split_select=False)
                    graphs[(r, key, b)] = g
    ev_h2d = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def load(i):
        s, b = i % PERIOD, i % 2
        ev_d2h[b].synchronize()           # step i-2 is over, its outputs on the host
        host_in[b].copy_(host_small[s])
        hs.wait_event(ev_cmp[b])
        copy(dev_bufs[b], host_in[b], bi, h2d, hs)
        ev_h2d[b].record(hs)

    def run(i):
        s, b = i % PERIOD, i % 2
        stream.wait_event(ev_h2d[b])
        stream.wait_event(ev_d2h[b])
        graphs[(i % R, (sc.csa_fires[s], sc.hca_fires[s]), b)].replay()
        ev_cmp[b].record(stream)
        ds.wait_event(ev_cmp[b])
        copy(host_outs[b], out_bufs[b], bo, d2h, ds)
        ev_d2h[b].record(ds)

    def pipeline(n):
        hs.wait_stream(stream)
        load(0)
        for i in range(n):
            run(i)
            if i + 1 < n:
                load(i + 1)
        stream.wait_event(ev_d2h[(n - 1) % 2])

    with torch.cuda.stream(stream):
        # every graph runs once before the timed region (its first launch
        # uploads it), on the inputs of a step of its own pattern
        for (r, key, b), g in graphs.items():
            stream.synchronize()
            host_in[b].copy_(host_small[first[key]])
            copy(dev_bufs[b], host_in[b], bi, h2d, stream)
            g.replay()
        stream.synchronize()
        pipeline(4)
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    with torch.cuda.stream(stream):
        e0.record(stream)
        pipeline(K)
        e1.record(stream)
    stream.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dev, world)
    del graphs
    return {"value": round(whole_job_rate(wl.B * K, ms, world), 2), "unit": UNIT,
            "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo), "steps": K,
            "path": f"public API calls (cskv_ring_store, csa_compress, indexer_topk, "
                    f"hybrid_attn_decode, hca_compress, hybrid_attn_decode) replayed from "
                    f"CUDA graphs; per step one pinned host->device copy of all inputs "
                    f"(written by the host once the step two back has its outputs on the "
                    f"host) and one device->host copy of both layers' outputs, each on a "
                    f"copy stream of its own so that they overlap the neighbouring steps' "
                    f"kernels (two device input and output buffers alternate); {R} rotating "
                    f"replicas as in the timed region",
            "eager_value": round(whole_job_rate(wl.B * K, ms_eager, world), 2),
            "eager_path": "the same calls launched eagerly from Python on one stream "
                          "(arguments marshalled once per buffer set)"}


# ------------------------------------------------------------- the oracle

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _cpu_layer(L):
    out = {}
    for k, v in L.items():
        if isinstance(v, torch.Tensor):
            out[k] = v.detach().cpu()
        elif isinstance(v, dict):
            out[k] = {kk: (vv.detach().cpu() if isinstance(vv, torch.Tensor) else vv)
                      for kk, vv in v.items()}
        else:
            out[k] = v
    return out


def oracle_query(Lc, Lh, frac=1.0, trace=None):
    """One decode query through the oracle: CSA indexer + top-k + sparse
    attention, HCA dense attention.  frac < 1 runs the same steps over the
    first frac of the compressed entries (a bounded sample of the query).
    trace (a list) receives each sequence's (scores, selection)."""
    import oracle as O
    from oracle.layer import as_numpy_cache, _q, _q_ik
    wl = Lc["wl"]
    res = []
    for b in range(wl.B):
        pos = int(Lc["q_pos"][b, 0])
        n_c = max(1, int(O.n_entries(pos + 1, wl.csa_stride) * frac))
        ik = as_numpy_cache(Lc["comp_ik"])
        s = O.indexer_scores(_q_ik(Lc, b, 0), Lc["head_w"][b, 0].double().numpy(),
                             O.dequant_slots(ik, b, np.arange(n_c)))
        k = max(1, int(round(wl.k * frac)))
        idx = O.topk(s, n_c, k)
        if trace is not None:
            trace.append((s, idx))
        ck = as_numpy_cache(Lc["comp_k"])
        sel = idx[idx >= 0]
        rk = as_numpy_cache(Lc["ring_k"])
        wlen = max(1, int(round(wl.window * frac)))
        wpos = O.window_positions(pos, wlen)
        win = O.dequant_slots(rk, b, O.ring_slots(wpos, rk["cap"]))
        comp = O.dequant_slots(ck, b, sel)
        res.append(O.hybrid_attention(_q(Lc, b, 0), comp, comp, win, win, wl.sm_scale))
        n_h = max(1, int(O.n_entries(pos + 1, wl.hca_stride) * frac))
        hk = as_numpy_cache(Lh["comp_k"])
        hr = as_numpy_cache(Lh["ring_k"])
        comp = O.dequant_slots(hk, b, np.arange(n_h))
        win = O.dequant_slots(hr, b, O.ring_slots(wpos, hr["cap"]))
        res.append(O.hybrid_attention(_q(Lh, b, 0), comp, comp, win, win, wl.sm_scale))
    return res


# the parity rules of the tests: top-k sets equal up to swaps whose oracle
# scores lie within 1e-3 of the k-th score; attention max|o - o_ref| within
# 2e-3 of the reference's RMS, |lse - lse_ref| within 1e-4
TOPK_REL, ATTN_REL, LSE_TOL = 1e-3, 2e-3, 1e-4


def parity_record(Lc, got, trace, first):
    """The library's answer to one decode query against the oracle's, under
    the tests' rules.  got = (idx [B][1][k], CSA out [B][1][H][Dv], CSA lse,
    HCA out, HCA lse) from the library; trace = the oracle's (scores,
    selection) per sequence and first = its (out, lse) pairs (CSA, HCA per
    sequence) for the same query, as oracle_query leaves them."""
    import oracle as O
    from oracle.layer import as_numpy_cache, _q
    g_idx, g_c, g_cl, g_h, g_hl = got
    wl = Lc["wl"]
    swaps, far, err_c, err_h, err_l = 0, 0, 0.0, 0.0, 0.0
    ck, rk = as_numpy_cache(Lc["comp_k"]), as_numpy_cache(Lc["ring_k"])

    def rel(out, ref_o):
        return float(np.max(np.abs(out - ref_o)) / np.sqrt(np.mean(ref_o ** 2)))
    for b in range(wl.B):
        s, ridx = trace[b]
        G = g_idx[b, 0][g_idx[b, 0] >= 0]
        R = ridx[ridx >= 0]
        gs, rs = set(G.tolist()), set(R.tolist())
        kth = s[R[-1]] if R.size else 0.0
        diff = (gs - rs) | (rs - gs)
        far += sum(1 for j in diff if abs(s[j] - kth) > TOPK_REL * abs(kth))
        far += int(len(G) != len(R))
        swaps += len(gs - rs)
        # CSA attention over the library's own selection, HCA over every entry
        pos = int(Lc["q_pos"][b, 0])
        wpos = O.window_positions(pos, wl.window)
        comp = O.dequant_slots(ck, b, G)
        win = O.dequant_slots(rk, b, O.ring_slots(wpos, rk["cap"]))
        o_c, l_c = O.hybrid_attention(_q(Lc, b, 0), comp, comp, win, win, wl.sm_scale)
        o_h, l_h = first[2 * b + 1]
        err_c = max(err_c, rel(g_c[b, 0], o_c))
        err_h = max(err_h, rel(g_h[b, 0], o_h))
        err_l = max(err_l, float(np.max(np.abs(g_cl[b, 0] - l_c))),
                    float(np.max(np.abs(g_hl[b, 0] - l_h))))
    return {"query": f"position {int(Lc['q_pos'][0, 0]):,}, B={wl.B}, both layers, against "
                     f"the oracle's float64",
            "topk_swaps": int(swaps), "topk_far": int(far),
            "csa_max_err_over_rms": round(err_c, 8), "hca_max_err_over_rms": round(err_h, 8),
            "max_lse_err": round(err_l, 8),
            "bounds": {"topk_rel": TOPK_REL, "attn_rel": ATTN_REL, "lse": LSE_TOL},
            "pass": bool(far == 0 and err_c <= ATTN_REL and err_h <= ATTN_REL
                         and err_l <= LSE_TOL)}


def cpu_baseline(rep, budget_s=12.0):
    """The oracle as it stands on the host cores, whole queries until the
    budget is spent (at least one).  The first of them is also the parity
    record of the run: the same query (replica 0's own positions) through
    the library, compared with the oracle by the tests' rules."""
    rep.csa.select()
    out_c, lse_c = rep.csa.attend()
    out_h, lse_h = rep.hca.attend()
    torch.cuda.synchronize()
    got = (rep.csa.idx.cpu().numpy(), out_c.cpu().double().numpy(),
           lse_c.cpu().double().numpy(), out_h.cpu().double().numpy(),
           lse_h.cpu().double().numpy())
    Lc, Lh = _cpu_layer(rep.csa_L), _cpu_layer(rep.hca_L)
    wl = Lc["wl"]
    t0 = time.perf_counter()
    n = 0
    trace = []
    while True:
        ref = oracle_query(Lc, Lh, trace=trace if n == 0 else None)
        if n == 0:
            first = ref
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    # (the comparison is not part of the timed oracle work)
    parity = parity_record(Lc, got, trace, first)
    parity["query"] = "replica 0 at its own " + parity["query"]
    return {"value": round(wl.B * n / dt, 4), "unit": UNIT, "cores": _threads(),
            "kind": "oracle",
            "sample": f"{n} whole decode queries (B={wl.B}) of the same workload, "
                      f"numpy float64, {dt:.1f} s"}, parity


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is one decode query over a
    bounded sample (the first `frac` of the compressed entries), sized so the
    whole run ends within a few minutes."""
    if rank != 0:
        return None
    wl = W.get(args.workload).with_(ik_fmt=args.ik_fmt)
    Lc = _cpu_layer(W.make_csa_layer(wl, seed=1000))
    Lh = _cpu_layer(W.make_hca_layer(wl, seed=501_000))
    t = time.perf_counter()
    oracle_query(Lc, Lh, frac=1 / 64)
    t_small = max(1e-4, time.perf_counter() - t) * 64    # rough cost of one whole query
    budget = 150.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(1 / 4096, budget / t_small))
    for _ in range(args.warmup):
        oracle_query(Lc, Lh, frac)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_query(Lc, Lh, frac)
    dt = time.perf_counter() - t0
    value = wl.B * frac * args.steps / dt
    cores = _threads()
    return {"metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{wl.name}: 1 CSA + 1 HCA layer decode, B={wl.B}/GPU, "
                                   f"ctx {wl.T}, Hq={wl.Hq}, D={wl.d_nope}+{wl.d_rope}, "
                                   f"H_I={wl.H_I}x{wl.d_I}, k={wl.k}, window={wl.window}",
                       "indexer_scales": _scales_text(wl),
                       "global_batch": wl.B * world, "seq_len": wl.T,
                       "parallelism": "oracle on the host cores, rank 0"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores,
                             "kind": "oracle",
                             "sample": f"each step: one decode query over the first "
                                       f"{frac:.5f} of the compressed entries; value scaled "
                                       f"by that fraction"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------- chunked prefill

def run_prefill(args, rank, world, dev):
    """Chunked prefill (--workload prefill): Tq new tokens per sequence on a
    cached context.  One step = CSA layer (csa_compress of the chunk's
    entries, indexer_score + indexer_select for every new token,
    hybrid_attn_prefill) + HCA layer (hca_compress, hybrid_attn_prefill).
    The step's tensors (queries, outputs, the score workspace) are far larger
    than L2.  The metric is prefill tokens/s; the roofline object reports the
    indexer scoring's tensor FLOP rate against the FP8 peak."""
    from compressed_sparse_kv_softmax_b200.layer import CSALayer, HCALayer
    wl = W.get(args.workload).with_(ik_fmt=args.ik_fmt)
    if args.tq:
        wl = wl.with_(Tq=args.tq)
    torch.cuda.set_device(dev)
    csa = CSALayer(W.make_csa_layer(wl, device=dev, seed=rank_seed(1000, rank)))
    hca = HCALayer(W.make_hca_layer(wl, device=dev, seed=rank_seed(501000, rank)))
    tb = torch.full((wl.B,), wl.T, dtype=torch.int64, device=dev)
    te = torch.full((wl.B,), wl.T + wl.Tq, dtype=torch.int64, device=dev)
    stream = torch.cuda.Stream(device=dev)
    names = ["csa_compress", "indexer_score", "indexer_select", "hybrid_attn_prefill (CSA)",
             "hca_compress", "hybrid_attn_prefill (HCA)"]

    def step(ev=None):
        calls = [lambda: csa.compress(tb, te, wl.Tq // wl.csa_stride),
                 lambda: csa.select(phase="score"), lambda: csa.select(phase="pick"),
                 lambda: csa.attend(), lambda: hca.compress(tb, te, wl.Tq // wl.hca_stride),
                 lambda: hca.attend()]
        for i, c in enumerate(calls):
            if ev:
                ev[i].record(stream)
            c()
        if ev:
            ev[-1].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    K = max(1, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for k in range(K):
            step(evs[k])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    per_call = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(len(names))] for e in evs])
    ms = max_over_ranks(float(sum(e[0].elapsed_time(e[-1]) for e in evs)) / K, dev, world)
    if world > 1:
        torch.distributed.barrier()
    calls_ms = {n: round(float(v), 4) for n, v in zip(names, per_call.mean(axis=0))}
    # FLOPs: visible entries differ per token of the chunk (causal)
    pos = np.arange(wl.T, wl.T + wl.Tq)
    n_c = ((pos + 1) // wl.csa_stride).astype(np.float64)
    n_h = ((pos + 1) // wl.hca_stride).astype(np.float64)
    win = np.minimum(pos + 1, wl.window)
    idx_flop = wl.B * 2.0 * wl.H_I * wl.d_I * n_c.sum()
    csa_flop = wl.B * 4.0 * wl.Hq * wl.D * (wl.k + win).sum()
    hca_flop = wl.B * 4.0 * wl.Hq * wl.D * (n_h + win).sum()
    # a step lasts far longer than a burst: the sustained GEMM figure
    peak, peak_kind = _peaks(kind="bf16_tflops_sustained")
    fp8_peak = 2.0 * peak            # the nominal FP8 : BF16 dense ratio
    idx_tflops = idx_flop / (calls_ms["indexer_score"] / 1e3) / 1e12
    tokens_per_rank = wl.B * wl.Tq
    res = {"metric": f"chunked-prefill tokens/s (CSA+HCA layers, {wl.Tq:,} new tokens on a "
                     f"{wl.T:,}-token context)",
           "value": round(whole_job_rate(tokens_per_rank, ms, world), 2), "unit": "tokens/s",
           "n_gpus": world,
           "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "fp8-e4m3/bf16 storage, fp32 math",
           "data": "synthetic (seeded Gaussian FP8 E4M3 + BF16 caches)",
           "config": {"workload": f"{wl.name}: B={wl.B}, {wl.Tq} new tokens at positions "
                                  f"{wl.T}..{wl.T + wl.Tq - 1}, Hq={wl.Hq}, "
                                  f"D={wl.d_nope}+{wl.d_rope}, H_I={wl.H_I}x{wl.d_I}, "
                                  f"k={wl.k}, window={wl.window}",
                      "indexer_scales": _scales_text(wl),
                      "l2": "per-step tensors (queries 0.5 GB, outputs 2 GB, scores 8.6 GB) "
                            "far above L2"},
           "roofline": {"bound": "tensor", "achieved": round(idx_tflops, 2),
                        "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                        "frac": round(idx_tflops / fp8_peak, 4), "traffic": None,
                        "kernel": f"{_scoring_kernel(wl)} (indexer_score: scoring of every "
                                  f"visible entry for each new token)",
                        "peak_kind": f"{peak_kind} sustained bf16 GEMM x 2 (nominal FP8/BF16 "
                                     f"ratio)",
                        "algorithmic_flop_per_launch": idx_flop},
           "flop": {"indexer": idx_flop, "csa_attention": csa_flop, "hca_attention": hca_flop},
           "calls_ms": calls_ms, "clocks": clocks, "e2e": None}
    return res


def run_other_workloads(args, rank, world, dev):
    """The batched decode workloads (Flash-like B = 8 at 65,536 tokens, k =
    512; Pro-like B = 4 at 131,072 tokens, k = 1,024), the 1M-context step
    with the per-channel gate variant of the compressors and with paged
    compressed caches (256-entry blocks), and the 8,192-token
    chunked prefill on a 1M context, each timed briefly the same way as the
    headline (decode: graph replays over rotating replicas, per-call times;
    prefill: events around each call).  Reported beside the headline, not as
    it."""
    import argparse as _ap
    peak, _ = _peaks()
    out = {}
    for name in ("flash", "pro", "long_channel_gate", "long_paged"):
        if name == "long_channel_gate":
            # the headline step with the per-channel gate variant of the compressors
            wl = W.get("long").with_(ik_fmt=args.ik_fmt, gate_mode="channel")
        elif name == "long_paged":
            # the headline step with its compressed caches paged in 256-entry blocks
            wl = W.get("long").with_(ik_fmt=args.ik_fmt, page_block=256)
        else:
            wl = W.get(name).with_(ik_fmt=args.ik_fmt)
        a = _ap.Namespace(**vars(args))
        a.warmup = max(3, min(args.warmup, 10))
        t = _time_decode(a, wl, rank, world, dev, args.other_steps, 7000, clocks=False,
                         call_replays=1)
        ib = indexer_bytes(wl)
        out[name] = {"metric": f"CSA+HCA decode queries/s ({name}: B={wl.B}, ctx {wl.T}, "
                               f"k={wl.k}, gate {wl.gate_mode}, "
                               f"{'paged %d' % wl.page_block if wl.page_block else 'contiguous'})",
                     "value": round(whole_job_rate(wl.B * t["steps"], t["ms"], world), 2),
                     "unit": UNIT, "steps": t["steps"], "ms_per_step": t["ms"] / t["steps"],
                     "indexer_score_us": round(t["idx_ms"] * 1e3, 3),
                     "indexer_frac": round(ib / (t["idx_ms"] / 1e3) / 1e9 / peak, 4),
                     "per_call": per_call_report(wl, t["calls"], peak)}
        del t
        torch.cuda.empty_cache()
    a = _ap.Namespace(**vars(args))
    a.workload, a.warmup, a.steps, a.tq = "prefill", 1, 2, 0
    r = run_prefill(a, rank, world, dev)
    out["prefill"] = {k: r[k] for k in ("metric", "value", "unit", "steps", "ms_per_step",
                                        "roofline", "flop", "calls_ms")}
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long")
    ap.add_argument("--replicas", type=int, default=0,
                    help="input replicas to rotate (0: enough to exceed 4x L2)")
    ap.add_argument("--graph-steps", type=int, default=PERIOD)
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ik-fmt", default="e4m3vec", choices=["e4m3vec", "e4m3", "mxfp4"],
                    help="indexer layout: FP8 with one scale per vector or per 64 dims, or "
                         "FP4 MXFP4")
    ap.add_argument("--tq", type=int, default=0,
                    help="prefill: new tokens per sequence (0: the workload's chunk); a "
                         "shorter chunk is a smaller case of the same step, for profiling")
    ap.add_argument("--call-replays", type=int, default=4,
                    help="replays of the per-call timing graph (0: skip)")
    ap.add_argument("--other-workloads", type=int, default=1,
                    help="1: also time the Flash-like and Pro-like batched decode and the "
                         "chunked prefill (briefly), reported beside the headline")
    ap.add_argument("--other-steps", type=int, default=1024)
    ap.add_argument("--alt-steps", type=int, default=2048,
                    help="steps timed with the other indexer layout (0: skip)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    if W.get(args.workload).prefill:
        res = run_prefill(args, rank, world, dev)
        if world > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res, replicas, wl = run_ours(args, rank, world, dev)
    res["e2e"] = run_e2e(args, replicas, wl, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"], res["parity"] = cpu_baseline(replicas[0], args.cpu_budget)
    del replicas
    torch.cuda.empty_cache()
    if args.other_workloads:
        res["other_workloads"] = run_other_workloads(args, rank, world, dev)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
