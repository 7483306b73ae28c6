#!/usr/bin/env python
"""Benchmark of the batched 4D FPS tokenizer on B200.

One step = one ``fps_tokenize`` call over one batch (binning, passthrough, FPS
fused with the Voronoi labels, Lloyd if configured, kNN or Voronoi pooling),
inputs resident in HBM.  The headline workload is the batched K = 128 case:
4096 small events (N ~ U{5..400}, about 31% passthrough), Voronoi assign +
mean-pool.  The same JSON line carries a block for the large-event workload
(8 showers of 50k-200k points, 3 charge-weighted Lloyd iterations), one for
the 64-event track batch, and the K sweep (32, 64, 256) of the headline
events, each timed the same way.

Prints one JSON line (rank 0).  ``value`` is events/s over all GPUs; the
per-kernel roofline uses CUDA events recorded by the library around each
internal stage in the timed region, against the measured float32 non-FMA op
rate.  ``--impl reference`` times the CPU oracle instead, on the host cores.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       (N > 1: launch under torch.distributed.run, one process per GPU).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FP32_OPS_PER_EVAL = 11  # 4 sub + 4 mul + 3 add
SM_COUNT = 148
FP32_LANES_PER_SM = 128
FP32_OPS_PER_LANE_CLK = 1  # non-FMA float32: one operation per lane per clock (packed or not)
SM_MAX_MHZ_NOMINAL = 1965.0
SIDE_WORKLOADS = ("c3", "c1")  # extra blocks on the headline line
K_SWEEP = (32, 64, 256)  # the headline events at other K
STAGES = ["bin", "fps_warp", "fps_cta", "fps_cta_smem", "fps_cluster8", "fps_cluster16", "lloyd",
          "knn+pool", "voronoi_pool", "passthrough"]
STAGE_KERNELS = {0: "k_bin", 1: "k_fps_warp", 2: "k_fps_cta", 3: "k_fps_block<1>",
                 4: "k_fps_block<8>", 5: "k_fps_block<16>", 6: "k_lloyd_sums+k_lloyd_step", 7: "k_knn",
                 8: "k_pool_voronoi", 9: "k_passthrough"}
FPS_STAGES = (1, 2, 3, 4, 5)
METRIC = "FPS+assign events/s (K=128)"
DEFAULT_WORKLOAD = "c4"


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--side-steps", type=int, default=300, help="timed steps of each extra block")
    ap.add_argument("--no-side", action="store_true", help="headline workload only (no extra blocks, no K sweep)")
    ap.add_argument("--K", type=int, default=None, help="override K (c4 sweep)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-microbench", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls only")
    ap.add_argument("--no-backward", action="store_true", help="skip the mean-pool backward measurement")
    return ap.parse_args()


# ------------------------------------------------------------------ workload

def global_batch(name, n_gpus, K=None):
    """The workload at n_gpus times its batch size (weak scaling)."""
    kw = {}
    if K is not None:
        kw["K"] = K
    base = workloads.make_workload(name, **kw)
    if n_gpus == 1:
        return base
    kw2 = dict(kw)
    if name != "c0":
        kw2["B"] = base.B * n_gpus
    return workloads.make_workload(name, **kw2)


def event_cost(sizes, K):
    from farthest_point_sampling_b200 import sharding

    return sharding.event_cost(sizes, K)


def partition_events(sizes, K, world):
    from farthest_point_sampling_b200 import sharding

    return sharding.partition_events(sizes, K, world)


def shard(batch, events):
    from farthest_point_sampling_b200 import sharding

    c, f, off = sharding.shard_events(batch.coords, batch.feats, batch.offsets, events)
    return workloads.Batch(c, f, off, batch.K, batch.assign_mode, batch.k, batch.lloyd_iters, batch.charge_col,
                           None, batch.name)


def algorithmic(batch):
    """Distance evaluations and algorithmic bytes of one step."""
    sizes = batch.sizes()
    K, F = batch.K, batch.F
    fpsev = sizes[sizes > K]
    evals = int((fpsev * K).sum()) * (1 + batch.lloyd_iters)
    if batch.assign_mode == 1:
        evals += int((fpsev * K).sum())
    P, B = batch.P, batch.B
    byts = 16 * P + 4 * F * P + 4 * P + 8 * (B + 1) + B * K * (4 + 16 + 4 * F + 4)
    if batch.assign_mode == 1:
        byts += B * K * batch.k * 4
    return evals, byts


# ------------------------------------------------------------------ clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, enabled=True):
        self.gpu = gpu_index
        self.proc = None
        self.enabled = enabled

    def __enter__(self):
        if self.enabled:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        if not getattr(self, "lines", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ profiles (ncu traffic)

def kernel_source_hash():
    """Hash of the FPS kernel sources with comments and blank lines removed
    (a comment edit leaves the compiled kernels, and their traffic, as they
    were)."""
    h = hashlib.sha256()
    for name in ("fps_kernels.cu", "common.cuh", "internal.h"):
        with open(os.path.join(ROOT, "farthest_point_sampling_b200", "csrc", name)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_stage, workload):
    """DRAM bytes per launch recorded in a committed ncu summary, if it was
    taken from the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    pat = re.compile(r"^\|\s*(\S+)\s*\|\s*(\S+)\s*\|\s*([0-9.]+)\s*\|\s*([0-9a-f]{16})\s*\|")
    with open(path) as fh:
        for ln in fh:
            m = pat.match(ln)
            if m and m.group(1) == STAGE_KERNELS[kernel_stage] and m.group(2) == workload and m.group(4) == want:
                return float(m.group(3))
    return None


# ------------------------------------------------------------------ CPU oracle

def cpu_oracle_rate(batch, seconds):
    import oracle

    oracle.build()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.tokenize_batch(batch)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return batch.B * reps / el, reps, el


def _oracle_worker_init():
    import oracle

    oracle.build()


def _oracle_slice(task):
    """Worker of the all-cores CPU baseline: the oracle, as it stands, on one
    slice of the batch's events, ``reps`` times; returns the seconds taken."""
    import oracle

    part, reps = task
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.tokenize_batch(part)
    return time.perf_counter() - t0


def cpu_oracle_rate_parallel(batch, seconds, rate1, max_workers=64):
    """The oracle on all host cores: events are independent, so the batch is
    split into cost-balanced slices (the multi-GPU split) and each worker
    process (started with spawn) runs the unmodified oracle on its slice
    about ``seconds`` long.  Returns (events/s, workers, passes, seconds)."""
    import multiprocessing as mp

    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    w = max(1, min(cores, max_workers, batch.B))
    idx = partition_events(batch.sizes(), batch.K, w)
    parts = [shard(batch, p) for p in idx]
    # passes sized so that the largest slice (the map waits for it) runs about `seconds`
    cost = event_cost(batch.sizes(), batch.K).astype(np.float64)
    total = float(cost.sum())
    share = max(float(cost[p].sum()) for p in idx) / total if total > 0 else 1.0 / w
    t_pass = batch.B / max(rate1, 1e-9)  # one single-core pass over the whole batch
    reps = max(1, int(round(seconds / max(t_pass * share, 1e-9))))
    with mp.get_context("spawn").Pool(w, initializer=_oracle_worker_init) as pool:
        pool.map(_oracle_slice, [(p, 1) for p in parts], chunksize=1)  # warm every worker
        t0 = time.perf_counter()
        pool.map(_oracle_slice, [(p, reps) for p in parts], chunksize=1)
        el = time.perf_counter() - t0
    return batch.B * reps / el, w, reps, el


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    batch = global_batch(args.workload, 1, args.K)
    import oracle

    oracle.build()
    for _ in range(args.warmup):
        oracle.tokenize_batch(batch)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.tokenize_batch(batch)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = batch.B * args.steps / total
    evals, _ = algorithmic(batch)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "events/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded generator)", "config": config_of(batch, args, l2="n/a (host)"),
        "gevals_per_s": evals * args.steps / total / 1e9,
        "cpu_baseline": {"value": value, "unit": "events/s", "cores": 1, "kind": "oracle",
                         "sample": f"the full batch ({batch.B} events) per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "events/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if not args.no_cpu_baseline:
        try:
            rate, w, reps, el = cpu_oracle_rate_parallel(batch, args.cpu_seconds, value)
            line["cpu_all_cores"] = {"value": rate, "unit": "events/s", "cores": w, "kind": "oracle",
                                     "sample": f"the batch split over {w} worker processes by N*K cost, "
                                               f"{reps} passes, {el:.1f} s"}
        except Exception as exc:  # noqa: BLE001
            line["cpu_all_cores"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    print(json.dumps(line))
    return 0


def config_of(batch, args, l2):
    return {"workload": batch.name, "events_per_gpu": batch.B, "points_per_gpu": batch.P, "K": batch.K,
            "assign_mode": "knn" if batch.assign_mode == 1 else "voronoi", "k": batch.k,
            "lloyd_iters": batch.lloyd_iters, "parallelism": f"dp{args.gpus} (events sharded, no collective)",
            "l2": l2}


# ------------------------------------------------------------------ main

def roofline_peak(mb, sm_count):
    """The FP32 roofline denominator: the measured non-FMA float32 op rate
    (the distance is made of separately rounded subtracts, multiplies and
    adds), refused if it exceeds the issue ceiling of one operation per lane
    per clock at the maximum SM clock.  Returns (peak TFLOP/s, source)."""
    ceiling = sm_count * FP32_LANES_PER_SM * FP32_OPS_PER_LANE_CLK * SM_MAX_MHZ_NOMINAL * 1e6 / 1e12
    nominal_src = (f"derived: {sm_count} SMs x {FP32_LANES_PER_SM} FP32 lanes x 1 non-FMA op per lane per clock "
                   f"x {SM_MAX_MHZ_NOMINAL:.0f} MHz")
    meas = (mb or {}).get("non_fma_peak")
    if meas and meas <= 1.02 * ceiling:
        return meas, ("measured in this run: best of the scalar FMUL+FADD and packed add / multiply chains "
                      f"(microbench non_fma_peak); issue ceiling {ceiling:.1f}")
    if meas:
        return ceiling, f"{nominal_src} (the measured {meas:.1f} exceeded that ceiling and was refused)"
    return ceiling, nominal_src


def measure(fps, lib, batch, full, args, dev, world, rank, steps, flush, want_stages=True):
    """Times ``steps`` fps_tokenize calls on ``batch`` (this rank's shard of
    ``full``): eager calls with the library's stage events, then the same call
    replayed from a CUDA graph.  L2 is flushed (256 MiB write) before every
    step, outside the timed events.  Returns a dict; times are the max over
    ranks."""
    import ctypes

    import torch
    import torch.distributed as dist

    vp = ctypes.c_void_p
    coords = torch.from_numpy(batch.coords).to(dev)
    feats = torch.from_numpy(batch.feats).to(dev)
    offsets = torch.from_numpy(batch.offsets).to(dev)
    hint = int(batch.sizes().max()) if batch.B else 0
    kw = dict(K=batch.K, assign_mode=batch.assign_mode, k=max(batch.k, 1), lloyd_iters=batch.lloyd_iters,
              charge_col=batch.charge_col, max_event_hint=hint)
    out = fps.fps_tokenize(coords, feats, offsets, check_device=True, **kw)
    opts = fps.Options(**kw)
    ws = torch.empty(max(lib.fps_workspace_bytes(batch.P, batch.B, batch.F, ctypes.byref(opts.c)), 256),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def make_call(strm):
        """One fps_tokenize call with every argument prebuilt (no Python checks)."""
        a = (vp(coords.data_ptr()), vp(feats.data_ptr()), batch.F, vp(offsets.data_ptr()), batch.B, batch.P,
             None, ctypes.byref(opts.c), vp(out["centroid_idx"].data_ptr()), vp(out["token_id"].data_ptr()),
             vp(out["knn_idx"].data_ptr()) if "knn_idx" in out else None, vp(out["centroids"].data_ptr()),
             vp(out["pooled"].data_ptr()), vp(out["counts"].data_ptr()), vp(ws.data_ptr()), ws.numel(),
             vp(strm.cuda_stream))
        fn = lib.fps_tokenize

        def call():
            rc = fn(*a)
            if rc:
                raise fps.FpsError(rc, "fps_tokenize")
        return call

    step = make_call(stream)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    nst = 2 * len(STAGES)
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst)] for _ in range(steps)] \
        if want_stages else []
    for evs in stage_ev:  # materialise the handles the library records into
        for e in evs:
            e.record(stream)
    stage_arr = [(vp * nst)(*[vp(e.cuda_event) for e in evs]) for evs in stage_ev]
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = fps.launch_count()
    stage_mask = 0  # stages the library actually ran (host-side record of its stage marks)
    for i in range(steps):
        flush.zero_()
        if want_stages:
            lib.fps_set_stage_events(stage_arr[i], nst)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        stage_mask |= lib.fps_stage_mask()
    lib.fps_set_stage_events(None, 0)
    torch.cuda.synchronize(dev)
    launches_per_step = (fps.launch_count() - launches0) / steps
    eager_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps

    # the same step replayed from a CUDA graph (launch overhead removed)
    graph_ms = None
    if not args.no_graph:
        g = torch.cuda.CUDAGraph()
        cap_stream = torch.cuda.Stream(dev)
        cap_stream.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap_stream):
            make_call(cap_stream)()
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        gs = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            gs[i].record(stream)
            g.replay()
            ge[i].record(stream)
        torch.cuda.synchronize(dev)
        graph_ms = sum(a.elapsed_time(b) for a, b in zip(gs, ge)) / steps
        del g
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)

    best_ms = graph_ms if graph_ms is not None else eager_ms
    t = torch.tensor([best_ms, eager_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_per_step, eager_ms = float(t[0].item()), float(t[1].item())

    # per-stage device time (recorded by the library inside the eager steps)
    stage_ms = {}
    for s_ in range(len(STAGES)):
        ts = []
        for evs in stage_ev:
            try:
                ts.append(evs[2 * s_].elapsed_time(evs[2 * s_ + 1]))
            except RuntimeError:
                break
        if stage_ev and len(ts) == steps:
            stage_ms[s_] = float(np.mean(ts))
    ran = {s_ for s_ in range(len(STAGES)) if (stage_mask >> s_) & 1}
    stage_ms = {s_: v for s_, v in stage_ms.items() if s_ in ran}
    # which schedule every event of this shard ran on (the library's own rule)
    sizes = batch.sizes()
    sched = np.array([lib.fps_schedule_for(int(n), batch.K, -1) for n in sizes])
    if (sched >= 0).sum() <= SM_COUNT:  # few events: the warp class runs on the CTA schedule
        sched = np.where(sched == 0, 1, sched)
    if (sched == 2).sum() <= SM_COUNT // 8:  # few mid-size events: 8-CTA clusters
        sched = np.where(sched == 2, 3, sched)
    evals_full, bytes_full = algorithmic(full)
    return {"ms_per_step": ms_per_step, "eager_ms": eager_ms, "graph_ms": graph_ms, "stage_ms": stage_ms,
            "launches_per_step": launches_per_step, "sched": sched, "kw": kw, "value": full.B / (ms_per_step / 1e3),
            "evals": evals_full, "bytes": bytes_full}


def roofline_block(m, batch, peak, peak_source, hbm, workload):
    """Roofline of the dominant stage's kernel, plus the whole step against
    the same bounds (the slower of the bytes at HBM peak and the
    evaluations at the FP32 peak)."""
    stage_ms = m["stage_ms"]
    t_step = m["ms_per_step"] / 1e3
    evals, byts = m["evals"], m["bytes"]
    t_roof = max(byts / (hbm * 1e9), evals * FP32_OPS_PER_EVAL / (peak * 1e12))
    step = {"evals": evals, "bytes": byts, "achieved_tflops": evals * FP32_OPS_PER_EVAL / t_step / 1e12,
            "roofline_ms": t_roof * 1e3, "frac": t_roof / t_step,
            "bound": "alu" if evals * FP32_OPS_PER_EVAL / (peak * 1e12) >= byts / (hbm * 1e9) else "hbm"}
    if not stage_ms:
        return {"step": step}
    # the passthrough stage runs on the lowest-priority helper stream beside
    # the FPS kernels; its span is mostly waiting for SMs, so it is not the
    # dominant kernel unless it is the only stage
    cands = {k: v for k, v in stage_ms.items() if k != 9} or stage_ms
    dom = max(cands, key=cands.get)
    t_dom = stage_ms[dom] / 1e3
    if dom in FPS_STAGES:
        ev = int(sum(int(n) * batch.K for n, s_ in zip(batch.sizes(), m["sched"]) if s_ == dom - 1))
        achieved = ev * FP32_OPS_PER_EVAL / t_dom / 1e12
        roof = {"bound": "alu", "kernel": STAGE_KERNELS[dom], "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_source,
                "algorithmic": f"{ev} point-centroid evals x {FP32_OPS_PER_EVAL} FP32 ops per launch",
                "stage_us": stage_ms[dom] * 1e3,
                "traffic": recorded_traffic(dom, workload)}
    elif dom == 6:  # Lloyd: N*K re-assign evaluations per iteration
        ev = int(sum(int(n) * batch.K for n in batch.sizes() if n > batch.K)) * batch.lloyd_iters
        achieved = ev * FP32_OPS_PER_EVAL / t_dom / 1e12
        roof = {"bound": "alu", "kernel": STAGE_KERNELS[dom], "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_source,
                "algorithmic": f"{ev} point-centroid evals x {FP32_OPS_PER_EVAL} FP32 ops ({batch.lloyd_iters} "
                               "re-assign passes)",
                "stage_us": stage_ms[dom] * 1e3, "traffic": recorded_traffic(dom, workload)}
    else:
        achieved = byts / t_dom / 1e9
        roof = {"bound": "hbm", "kernel": STAGE_KERNELS[dom], "achieved": achieved, "peak": hbm,
                "unit": "GB/s", "frac": achieved / hbm, "stage_us": stage_ms[dom] * 1e3,
                "traffic": recorded_traffic(dom, workload)}
    roof["step"] = step
    return roof


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import farthest_point_sampling_b200 as fps

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def shard_of(name, K=None):
        full_ = global_batch(name, world, K)
        if world > 1:
            parts = partition_events(full_.sizes(), full_.K, world)
            return full_, shard(full_, parts[rank])
        return full_, full_

    full, batch = shard_of(args.workload, args.K)
    fps.build()
    lib = fps.load_library()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    mb = None
    if rank == 0 and not args.no_microbench:
        try:
            mb = microbench_fp32(dev)
        except Exception as exc:  # noqa: BLE001
            mb = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    peak, peak_source = roofline_peak(mb if mb and "error" not in mb else None,
                                      torch.cuda.get_device_properties(dev).multi_processor_count)

    wall0 = time.perf_counter()
    with ClockSampler(local, enabled=not args.no_clocks and rank == 0) as clocks:
        m = measure(fps, lib, batch, full, args, dev, world, rank, args.steps, flush)
    wall = time.perf_counter() - wall0

    result = {
        "metric": METRIC, "value": m["value"], "unit": "events/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded generator shaped like the pages' events)",
        "config": config_of(batch, args, l2="flushed between steps (256 MiB write outside the timed events)"),
        "gevals_per_s": m["evals"] / (m["ms_per_step"] / 1e3) / 1e9,
        "gpu_launches": int(round(m["launches_per_step"] * args.steps)),
        "timing": {"graph_replay_ms_per_step": m["graph_ms"], "eager_ms_per_step": m["eager_ms"],
                   "value_from": "graph replay" if m["graph_ms"] is not None else "eager calls",
                   "kernels_per_step": m["launches_per_step"]},
        "stage_ms": {STAGES[s_]: round(v, 5) for s_, v in sorted(m["stage_ms"].items())},
        "wall_s_timed_region": wall,
    }
    if rank == 0:
        roof = roofline_block(m, batch, peak, peak_source, hbm, args.workload)
        if mb:
            roof["microbench_fp32_tflops"] = mb
        result["roofline"] = roof
        result["clocks"] = clocks.summary()
        if not args.no_e2e:
            result["e2e"] = e2e(fps, batch, m["kw"], dev, args.e2e_steps)

    # extra blocks: other workloads and the K sweep, timed the same way (every rank takes part)
    if not args.no_side:
        side = {}
        for name in SIDE_WORKLOADS:
            if name == args.workload:
                continue
            f_, b_ = shard_of(name)
            with ClockSampler(local, enabled=not args.no_clocks and rank == 0) as ck:
                ms_ = measure(fps, lib, b_, f_, args, dev, world, rank, args.side_steps, flush)
            if rank == 0:
                blk = {"workload": name, "value": ms_["value"], "unit": "events/s", "ms_per_step": ms_["ms_per_step"],
                       "steps": args.side_steps, "gevals_per_s": ms_["evals"] / (ms_["ms_per_step"] / 1e3) / 1e9,
                       "config": config_of(b_, args, l2="flushed between steps"),
                       "stage_ms": {STAGES[s_]: round(v, 5) for s_, v in sorted(ms_["stage_ms"].items())},
                       "roofline": roofline_block(ms_, b_, peak, peak_source, hbm, name),
                       "kernels_per_step": ms_["launches_per_step"], "clocks": ck.summary()}
                if not args.no_e2e:
                    blk["e2e"] = e2e(fps, b_, ms_["kw"], dev, max(20, args.e2e_steps // 4))
                side[name] = blk
        if args.workload == DEFAULT_WORKLOAD and args.K is None:
            sweep = {}
            for Kx in K_SWEEP:
                f_, b_ = shard_of(args.workload, Kx)
                ms_ = measure(fps, lib, b_, f_, args, dev, world, rank, args.side_steps, flush)
                if rank == 0:
                    rb = roofline_block(ms_, b_, peak, peak_source, hbm, f"{args.workload}_K{Kx}")
                    sweep[str(Kx)] = {"value": ms_["value"], "unit": "events/s", "ms_per_step": ms_["ms_per_step"],
                                      "gevals_per_s": ms_["evals"] / (ms_["ms_per_step"] / 1e3) / 1e9,
                                      "stage_ms": {STAGES[s_]: round(v, 5) for s_, v in sorted(ms_["stage_ms"].items())},
                                      "dominant_frac": rb.get("frac"), "step_frac": rb["step"]["frac"]}
            if rank == 0:
                side["k_sweep"] = sweep
        if rank == 0:
            result["workloads"] = side

    if rank == 0:
        if not args.no_backward:  # side measurements: a failure is recorded, the line still prints
            for key, fn in (("pool_backward", pool_backward_roofline), ("token_pack", token_pack_roofline),
                            ("token_summaries", token_summaries_roofline)):
                try:
                    result[key] = fn(fps, dev)
                except Exception as exc:  # noqa: BLE001
                    result[key] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        if world == 1 and not args.no_cpu_baseline:
            rate, reps, el = cpu_oracle_rate(batch, args.cpu_seconds)
            result["cpu_baseline"] = {"value": rate, "unit": "events/s", "cores": 1, "kind": "oracle",
                                      "sample": f"the full batch ({batch.B} events) x {reps} passes, {el:.1f} s"}
            try:
                prate, w, preps, pel = cpu_oracle_rate_parallel(batch, args.cpu_seconds, rate)
                result["cpu_all_cores"] = {"value": prate, "unit": "events/s", "cores": w, "kind": "oracle",
                                           "sample": f"the batch split over {w} worker processes by N*K cost, "
                                                     f"{preps} passes, {pel:.1f} s"}
            except Exception as exc:  # noqa: BLE001
                result["cpu_all_cores"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        print(json.dumps(result))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


MICROBENCH_MODES = {0: "scalar_fmul_fadd", 1: "f32x2_add", 2: "f32x2_mul", 3: "f32x2_fma", 4: "f32x2_distance"}


def microbench_fp32(dev):
    """Measured FP32 rates (TFLOP/s, an FMA counted as two) of the microbenchmark modes.

    The non-FMA peak is the best of the scalar and the separate packed add and
    multiply chains: the roofline denominator.  "f32x2_distance" is the rate of
    the distance exactly as the FPS kernels compute it, every input
    loop-carried; it is reported to show that the packed mix runs at that
    same non-FMA rate (11 ops per evaluation, one per lane per clock).
    """
    import ctypes

    import torch

    import farthest_point_sampling_b200 as fps

    lib = ctypes.CDLL(fps.build_microbench())
    lib.fpstok_microbench_fp32.restype = ctypes.c_double
    lib.fpstok_microbench_fp32.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    blocks = torch.cuda.get_device_properties(dev).multi_processor_count * 8
    out = torch.empty(blocks, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    best = {}
    for mode, name in MICROBENCH_MODES.items():
        rates = []
        for _ in range(4):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)  # creates the underlying events
            b.record(stream)
            torch.cuda.synchronize(dev)
            ops = lib.fpstok_microbench_fp32(mode, blocks, 256, 2048, ctypes.c_void_p(out.data_ptr()),
                                             ctypes.c_void_p(a.cuda_event), ctypes.c_void_p(b.cuda_event),
                                             ctypes.c_void_p(stream.cuda_stream))
            torch.cuda.synchronize(dev)
            if ops > 0:
                rates.append(ops / (a.elapsed_time(b) / 1e3) / 1e12)
        best[name] = max(rates) if rates else None
    vals = [best[k] for k in ("scalar_fmul_fadd", "f32x2_add", "f32x2_mul") if best.get(k)]
    best["non_fma_peak"] = max(vals) if vals else None
    return best


def pool_backward_roofline(fps, dev, reps=50):
    """HBM roofline of the mean-pool backward (C ``segment_pool_backward``),
    called through the C ABI on preallocated buffers.

    Voronoi: the large-event shapes (8 events of 50k-200k points, K = 128,
    F = 6) with seeded random labels; kNN: the 256-event kNN workload's
    shapes (k = 32) with seeded random rows inside each event.  One call is
    captured in a CUDA graph; each replay is timed with CUDA events on the
    current stream, after a 256 MiB write that evicts the inputs from L2
    (outside the events)."""
    import ctypes
    import json as _j

    import torch
    from farthest_point_sampling_b200 import _lib

    lib = fps.load_library()
    peaks = _j.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    vp = ctypes.c_void_p
    out = {}
    for mode, wl in ((_lib.FPS_ASSIGN_VORONOI, "c3"), (_lib.FPS_ASSIGN_KNN, "c2")):
        b = workloads.make_workload(wl)
        sizes = b.sizes()
        B, K, F, P = b.B, b.K, b.feats.shape[1], int(b.offsets[-1])
        rng = np.random.default_rng(90 + mode)
        G = torch.from_numpy(rng.normal(0, 1, (B, K, F)).astype(np.float32)).to(dev)
        offsets = torch.from_numpy(b.offsets).to(dev)
        counts_np = np.zeros((B, K), np.int32)
        if mode == _lib.FPS_ASSIGN_VORONOI:
            tok_np = np.concatenate([rng.integers(0, min(int(n), K), int(n)) for n in sizes]).astype(np.int32)
            np.add.at(counts_np, (np.repeat(np.arange(B), sizes), tok_np), 1)
            tok, knn, k = torch.from_numpy(tok_np).to(dev), None, 0
            byts = 4 * P + 4 * F * P + B * K * (4 * F + 4) + 8 * (B + 1)
            what = "4P token ids + 4FP gradient written + B*K*(4F+4) rows and counts + 8(B+1) offsets"
        else:
            k = b.k
            rows = np.full((B, K, k), -1, np.int32)
            for e, n in enumerate(sizes):
                if n > 0:
                    m = min(int(n), k)
                    rows[e, :min(int(n), K), :m] = b.offsets[e] + np.stack(
                        [rng.choice(int(n), m, replace=False) for _ in range(min(int(n), K))])
            counts_np = (rows >= 0).sum(2).astype(np.int32)
            tok, knn = None, torch.from_numpy(rows).to(dev)
            byts = 4 * B * K * k + B * K * (4 * F + 4) + 4 * F * P
            what = "4*B*K*k rows + B*K*(4F+4) gradient rows and counts + 4FP gradient written"
        counts = torch.from_numpy(counts_np).to(dev)
        grad = torch.empty((P, F), dtype=torch.float32, device=dev)
        nb = lib.segment_pool_backward_workspace_bytes(P, B, K, F, mode)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
        n_before = lib.fps_launch_count()

        def call(strm):
            st = lib.segment_pool_backward(vp(G.data_ptr()), F, vp(offsets.data_ptr()), B, P, K, mode,
                                           vp(tok.data_ptr()) if tok is not None else None,
                                           vp(knn.data_ptr()) if knn is not None else None, k,
                                           vp(counts.data_ptr()), vp(grad.data_ptr()), vp(ws.data_ptr()),
                                           ws.numel(), vp(strm.cuda_stream))
            if st != 0:
                raise RuntimeError(f"segment_pool_backward failed: {st}")

        for _ in range(3):
            call(stream)
        torch.cuda.synchronize(dev)
        n_warm = lib.fps_launch_count() - n_before
        # one call captured in a CUDA graph, replayed after an L2-evicting write
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            call(cap)
        torch.cuda.synchronize(dev)
        for _ in range(3):
            flush.zero_()
            g.replay()
        st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
        for i in range(reps):
            flush.zero_()
            st_ev[i].record(stream)
            g.replay()
            en_ev[i].record(stream)
        torch.cuda.synchronize(dev)
        ms = float(np.mean([a.elapsed_time(c) for a, c in zip(st_ev, en_ev)]))
        del g
        achieved = byts / (ms / 1e3) / 1e9
        out["voronoi" if mode == _lib.FPS_ASSIGN_VORONOI else "knn"] = {
            "workload": f"{wl} shapes: B={B}, P={P}, K={K}, F={F}" + (f", k={k}" if k else ""),
            "us_per_call": ms * 1e3, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "algorithmic_bytes": byts, "algorithmic": what,
            "kernels_per_call": n_warm / 3,
            "note": "memset + per-event row masks and row-order sums + rounding, timed together" if k else "quotient table + gather"}
    return out


def token_summaries_roofline(fps, dev, reps=30):
    """HBM roofline of the charge-weighted token summaries (C
    ``fps_token_summaries``) on the large-event workload's shapes (8 events,
    about 0.9 M points, K = 128, F = 6, charge column 0) with seeded random
    labels.  Graph-replayed and timed like ``pool_backward_roofline``."""
    import ctypes
    import json as _j

    import torch

    lib = fps.load_library()
    peaks = _j.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    b = workloads.make_workload("c3")
    B, K, F, P = b.B, b.K, b.feats.shape[1], int(b.offsets[-1])
    rng = np.random.default_rng(96)
    coords = torch.from_numpy(b.coords).to(dev)
    feats = torch.from_numpy(b.feats).to(dev)
    offsets = torch.from_numpy(b.offsets).to(dev)
    tok = torch.from_numpy(rng.integers(0, K, P).astype(np.int32)).to(dev)
    wsum = torch.empty((B, K), dtype=torch.float32, device=dev)
    wc = torch.empty((B, K, 4), dtype=torch.float32, device=dev)
    wf = torch.empty((B, K, F), dtype=torch.float32, device=dev)
    ws = torch.empty(max(lib.fps_token_summaries_workspace_bytes(B, K, F), 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    vp = ctypes.c_void_p

    def call(strm):
        st = lib.fps_token_summaries(vp(coords.data_ptr()), vp(feats.data_ptr()), F, 0, vp(offsets.data_ptr()), B,
                                     P, K, vp(tok.data_ptr()), vp(wsum.data_ptr()), vp(wc.data_ptr()),
                                     vp(wf.data_ptr()), vp(ws.data_ptr()), ws.numel(), vp(strm.cuda_stream))
        if st != 0:
            raise RuntimeError(f"fps_token_summaries failed: {st}")

    n_before = lib.fps_launch_count()
    for _ in range(3):
        call(stream)
    torch.cuda.synchronize(dev)
    per_call = (lib.fps_launch_count() - n_before) / 3
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap):
        call(cap)
    torch.cuda.synchronize(dev)
    st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        st_ev[i].record(stream)
        g.replay()
        en_ev[i].record(stream)
    torch.cuda.synchronize(dev)
    ms = float(np.mean([a.elapsed_time(c) for a, c in zip(st_ev, en_ev)]))
    del g
    byts = 16 * P + 4 * F * P + 4 * P + 8 * (B + 1) + B * K * (4 + 16 + 4 * F)
    achieved = byts / (ms / 1e3) / 1e9
    return {"workload": f"c3 shapes: B={B}, P={P}, K={K}, F={F}, charge column 0", "us_per_call": ms * 1e3,
            "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "algorithmic_bytes": byts,
            "algorithmic": "16P coords + 4FP feats + 4P token ids + 8(B+1) offsets read, B*K*(4+16+4F) written",
            "kernels_per_call": per_call, "note": "status-word memset + per-range sums + boundary finalize"}


def token_pack_roofline(fps, dev, reps=50):
    """HBM roofline of the packed token layout (C ``fps_pack_tokens``) on the
    small-event workload's shapes: 4096 events, K = 128 slots of F = 6 pooled
    features, v_b = min(N_b, K) tokens each.  Graph-replayed and timed like
    ``pool_backward_roofline``."""
    import ctypes
    import json as _j

    import torch

    lib = fps.load_library()
    peaks = _j.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    b = workloads.make_workload("c4")
    B, K, D = b.B, b.K, b.feats.shape[1]
    v = np.minimum(b.sizes(), K)
    n_tok = int(v.sum())
    src = torch.from_numpy(np.random.default_rng(95).normal(0, 1, (B, K, D)).astype(np.float32)).to(dev)
    offsets = torch.from_numpy(b.offsets).to(dev)
    dst = torch.empty((B * K, D), dtype=torch.float32, device=dev)
    doc = torch.empty(B * K, dtype=torch.int32, device=dev)
    tok = torch.empty(B + 1, dtype=torch.int64, device=dev)
    ws = torch.empty(max(lib.fps_pack_workspace_bytes(), 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    vp = ctypes.c_void_p

    def call(strm):
        st = lib.fps_pack_tokens(vp(src.data_ptr()), D, vp(offsets.data_ptr()), None, B, K, vp(dst.data_ptr()),
                                 vp(doc.data_ptr()), vp(tok.data_ptr()), vp(ws.data_ptr()), ws.numel(),
                                 vp(strm.cuda_stream))
        if st != 0:
            raise RuntimeError(f"fps_pack_tokens failed: {st}")

    n_before = lib.fps_launch_count()
    for _ in range(3):
        call(stream)
    torch.cuda.synchronize(dev)
    per_call = (lib.fps_launch_count() - n_before) / 3
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(g, stream=cap):
        call(cap)
    torch.cuda.synchronize(dev)
    st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        st_ev[i].record(stream)
        g.replay()
        en_ev[i].record(stream)
    torch.cuda.synchronize(dev)
    ms = float(np.mean([a.elapsed_time(c) for a, c in zip(st_ev, en_ev)]))
    del g
    byts = 8 * (B + 1) + 2 * 4 * D * n_tok + 4 * n_tok + 8 * (B + 1)
    achieved = byts / (ms / 1e3) / 1e9
    return {"workload": f"c4 shapes: B={B}, K={K}, D={D}, {n_tok} tokens", "us_per_call": ms * 1e3,
            "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "algorithmic_bytes": byts,
            "algorithmic": "8(B+1) offsets read + 4*D*N_tok rows read and written + 4*N_tok doc ids "
                           "+ 8(B+1) token offsets",
            "kernels_per_call": per_call, "note": "scan (one CTA) + per-event copy"}


def e2e(fps, batch, kw, dev, steps):
    """Same metric through the host-pointer C entry point (H2D + compute + D2H)."""
    import torch

    c = torch.from_numpy(batch.coords).pin_memory()
    f = torch.from_numpy(batch.feats).pin_memory()
    o = torch.from_numpy(batch.offsets).pin_memory()
    kw2 = {k: v for k, v in kw.items() if k not in ("max_event_hint",)}
    out = fps.fps_tokenize_host(c, f, o, device=dev, **kw2)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        fps.fps_tokenize_host(c, f, o, device=dev, out=out, **kw2)
    tot = 0.0
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fps.fps_tokenize_host(c, f, o, device=dev, out=out, synchronize=False, **kw2)
        b.record(stream)
        b.synchronize()
        tot += a.elapsed_time(b)
    h2d = batch.coords.nbytes + batch.feats.nbytes + batch.offsets.nbytes
    d2h = sum(v.numel() * v.element_size() for v in out.values())
    return {"value": batch.B * steps / (tot / 1e3), "unit": "events/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": tot / steps}


if __name__ == "__main__":
    sys.exit(main())
