#!/usr/bin/env python
"""Benchmark of the Muon / DMuon optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the library's ``dmuon_step`` over a whole parameter set
(momentum, normalisation, 5 quintic Newton-Schulz steps, scale, decay and the
parameter write for every matrix).  Default workload: the matrix set of a
Llama-style 8B model (32 layers of q 4096^2, k and v 4096 x 1024, o 4096^2,
gate and up 4096 x 14336, down 14336 x 4096; 224 matrices, 6.98 G elements),
bf16 weights and grads ~ N(0, 1e-3^2), fp32 momenta.  Inputs are resident in
HBM before the timed region; they total 56 GB (> 126 MB of L2), so no L2
flush is needed between steps.

Prints one JSON line (rank 0).  N > 1 runs independent replicas, one per
rank (the step has no exchange on one parameter set); timing is the max over
ranks of the device-timed region.  ``--impl reference`` times the fp64 CPU
oracle on bounded samples of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "Muon step ms per param set; NS TFLOPS as % of B200 bf16 dense peak"
DEFAULT_WORKLOAD = "llama8b-matrices-bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 10 ** 6
# fp32 FFMA peak from unit counts and clock: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz
FP32_FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def measured_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def ns_flops(rows, cols, steps, variant):
    m, n = min(rows, cols), max(rows, cols)
    if steps == 0:
        return 0.0
    if variant == "gram":
        return 2.0 * (2 * m * m * n + (1 + 4 * (steps - 1)) * m ** 3)
    return 2.0 * steps * (2 * m * m * n + m ** 3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 100 ms in a background process; samples are
    kept with host timestamps so only those inside the timed window count."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for t, s in self.samples if t0 <= t <= t1]
        if not rows:  # a short window: take the nearest samples around it
            rows = [s for t, s in self.samples if t0 - 0.3 <= t <= t1 + 0.3]
        mhz, maxmhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                maxmhz = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxmhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ------------------------------------------------------------------ CPU baseline (oracle)
# A parameter set whose direct-form Newton-Schulz work is at most this many
# FLOPs is timed in full by the fp64 oracle (the fp32 256 x 512 set and the
# 64 x 1024^2 set: a few seconds on a many-core host).  Larger sets time one
# matrix of every distinct shape and scale each by its count ("extrapolated").
FULL_ORACLE_FLOPS = 4.0e12


def oracle_sample(w):
    """Matrix indices the oracle times and whether they are the whole set."""
    shapes = w.shapes()
    if sum(ns_flops(r, c, w.ns_steps, "direct") for r, c in shapes) <= FULL_ORACLE_FLOPS:
        return list(range(len(shapes))), False
    first = {}
    for i, s in enumerate(shapes):
        first.setdefault(s, i)
    return sorted(first.values()), True


def oracle_inputs(w, indices):
    """fp64 host copies of (W, G, M) for the given matrices (CPU generator:
    same shapes and distributions as the device draw; values do not affect
    the oracle's time)."""
    from newton_schulz_normalise_b200 import workloads as wl
    Ws, Gs, Ms = wl.generate(w, device="cpu", indices=indices)
    return [(a.double().numpy(), b.double().numpy(), c.double().numpy()) for a, b, c in zip(Ws, Gs, Ms)]


def oracle_seconds(w, inp):
    """Wall time of oracle.muon_step (as it stands) on one matrix."""
    import oracle.muon_oracle as ora
    W, G, M = inp
    t0 = time.perf_counter()
    ora.muon_step(W, G, M, w.lr, w.wd, w.mu, w.ns_steps)
    return time.perf_counter() - t0


def oracle_set_ms(w, per_shape_s):
    """ms per parameter set from mean seconds per matrix of each shape."""
    return 1e3 * sum(statistics.mean(per_shape_s[s]) for s in w.shapes())


def _threads():
    import torch
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    return cores


def cpu_baseline(w):
    """The fp64 oracle as it stands on the host cores: the whole parameter set
    when it is small (FULL_ORACLE_FLOPS), else one matrix of every distinct
    shape, each scaled by its count."""
    cores = _threads()
    idx, extrapolated = oracle_sample(w)
    shapes = w.shapes()
    inputs = oracle_inputs(w, idx)
    per_shape = {}
    for i, inp in zip(idx, inputs):
        per_shape.setdefault(shapes[i], []).append(oracle_seconds(w, inp))
    val = oracle_set_ms(w, per_shape)
    how = ("one matrix of each of the %d shapes, scaled by its count" % len(per_shape) if extrapolated
           else "the whole set")
    return {
        "value": val, "unit": "ms", "cores": cores, "kind": "oracle",
        "sample": f"{len(idx)} of {len(shapes)} matrices timed one by one ({how}); fp64 numpy, "
                  f"BLAS on {cores} threads",
        "extrapolated": extrapolated, "matrices_timed": len(idx),
        "per_shape_ms": {f"{r}x{c}": round(1e3 * statistics.mean(t), 3) for (r, c), t in per_shape.items()},
        "cpu": _cpu_model(),
        "adamw": adamw_oracle_time(),
    }


def adamw_oracle_time():
    """The fp64 AdamW oracle on 1/16 of the bench's AdamW set (3144 rows of
    the 50304 x 1024 table plus 6 of the 96 vectors), scaled to the whole set."""
    import numpy as np
    import oracle.adamw_oracle as aora
    rng = np.random.default_rng(5)
    parts = [rng.standard_normal((3144, 1024)) * 0.02] + [rng.standard_normal(1024) * 0.02 for _ in range(6)]
    t0 = time.perf_counter()
    for p in parts:
        g = p * 0.05
        aora.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), 1e-3, 0.9, 0.95, 1e-8, 0.1, 4)
    dt = time.perf_counter() - t0
    return {"value": dt * 16 * 1e3, "unit": "ms", "kind": "oracle",
            "sample": "1/16 of the 50304x1024 + 96x1024 set (fp64 numpy), scaled by 16"}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------ distributed
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(values, world_size, device="cpu"):
    """Element-wise max of per-rank timings over the process group (the
    step is timed on every rank; the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world_size > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_value(ms_max, steps, world_size):
    """ms per parameter set for the whole job: every rank (replica) updates
    one parameter set per step, so N ranks finish N sets in ms_max / steps."""
    return ms_max / steps / world_size


def run_reference(args, w):
    """The oracle arm.  A step times one bounded sample: the whole parameter
    set when it is small, else one matrix, taking the distinct shapes in turn.
    ms_per_step is the mean time of the timed samples as they ran; value is
    the ms per parameter set they imply (scaled by each shape's count when the
    samples are single matrices, and then marked extrapolated)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    cores = _threads()
    idx, extrapolated = oracle_sample(w)
    shapes = w.shapes()
    inputs = oracle_inputs(w, idx)
    per_shape, step_s = {}, []
    t_run0 = time.perf_counter()
    for k in range(args.warmup + args.steps):
        if extrapolated:
            j = k % len(idx)
            dt = oracle_seconds(w, inputs[j])
            if k >= args.warmup or len(idx) > args.steps:
                per_shape.setdefault(shapes[idx[j]], []).append(dt)
        else:
            dt = 0.0
            for i, inp in zip(idx, inputs):
                t = oracle_seconds(w, inp)
                dt += t
                if k >= args.warmup:
                    per_shape.setdefault(shapes[i], []).append(t)
        if k >= args.warmup:
            step_s.append(dt)
    for i, inp in zip(idx, inputs):  # a run too short to meet every shape: time the rest once
        if shapes[i] not in per_shape:
            per_shape[shapes[i]] = [oracle_seconds(w, inp)]
    run_s = time.perf_counter() - t_run0
    val = oracle_set_ms(w, per_shape)
    sample = (f"step k times matrix {{{', '.join(str(i) for i in idx)}}}[k mod {len(idx)}] (one of each shape); "
              f"value = sum over shapes of count x mean time" if extrapolated
              else f"every step times all {len(shapes)} matrices one by one")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "ms", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(step_s) if step_s else None,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "matrices": len(shapes),
                   "shapes": sorted({f"{r}x{c}" for r, c in shapes}), "ns_steps": w.ns_steps,
                   "lr": w.lr, "wd": w.wd, "mu": w.mu, "parallelism": "fp64 oracle on rank 0's host cores"},
        "extrapolated": extrapolated,
        "cpu_baseline": {"value": val, "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample,
                         "extrapolated": extrapolated,
                         "per_shape_ms": {f"{r}x{c}": round(1e3 * statistics.mean(t), 3)
                                          for (r, c), t in per_shape.items()},
                         "run_s": round(run_s, 2)},
        "e2e": {"value": val, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ncu summaries of the CTA-pair GEMM per bench workload; each holds the
# per-launch DRAM traffic of the bench's launches and the hash of the kernel
# source it was taken on.
PAIR_PROFILES = {"batch64-1024x1024-bf16": "tc_gemm_pair_batch64-1024x1024.md",
                 "llama8b-matrices-bf16": "tc_gemm_pair_llama8b-matrices.md"}


def host_memory_short(bytes_per_rank: int, local_ranks: int):
    """None when the host can pin bytes_per_rank for every rank of the node
    (with a quarter of the available memory to spare), else the reason."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:  # no way to tell: try it
        return None
    need = bytes_per_rank * max(1, local_ranks)
    if need * 1.25 <= avail:
        return None
    return (f"host memory: {need / 1e9:.1f} GB of pinned buffers for {local_ranks} rank(s), "
            f"{avail / 1e9:.1f} GB available")


def profile_traffic(kernel_file: Path, workload: str):
    """Per-launch DRAM traffic of the dominant kernel from the committed ncu
    summary of this workload, if it was taken on the current kernel source."""
    import hashlib
    name = PAIR_PROFILES.get(workload)
    summ = ROOT / "profiles" / name if name else None
    if summ is None or not summ.exists():
        return None
    sha = hashlib.sha256(kernel_file.read_bytes()).hexdigest()[:16]
    src, traffic = None, None
    for line in summ.read_text().splitlines():
        if line.startswith("kernel_source_sha256_16:"):
            src = line.split(":", 1)[1].strip()
        if line.startswith("traffic_bytes_per_launch:"):
            traffic = float(line.split(":", 1)[1].strip())
    return traffic if src == sha else None


def adamw_measure(dev, stream, torch_dtype, iters=20):
    """Device time of one dmuon_adamw_step over an embedding-sized set of
    non-matrix parameters; returns ms, GB/s of algorithmic bytes, element
    count and bytes per element."""
    import torch
    from newton_schulz_normalise_b200 import binding as B
    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    shapes = [(50304, 1024)] + [(1024,)] * 96
    P = [(torch.randn(s, device=dev, generator=gen) * 0.02).to(torch_dtype) for s in shapes]
    G = [(torch.randn(s, device=dev, generator=gen) * 1e-3).to(torch_dtype) for s in shapes]
    M = [torch.zeros(s, device=dev) for s in shapes]
    V = [torch.zeros(s, device=dev) for s in shapes]
    tP, tG, tM, tV = B.TensorList(P), B.TensorList(G), B.TensorList(M), B.TensorList(V)
    for t in range(1, 4):
        B.dmuon_adamw_step(tP, tG, tM, tV, 1e-3, 0.9, 0.95, 1e-8, 0.1, t, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for t in range(4, 4 + iters):
        B.dmuon_adamw_step(tP, tG, tM, tV, 1e-3, 0.9, 0.95, 1e-8, 0.1, t, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    n = sum(p.numel() for p in P)
    bpe = 22 if torch_dtype == torch.bfloat16 else 32
    return {"ms": ms, "gbs": n * bpe / (ms * 1e-3) / 1e9, "elements": n, "bpe": bpe}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", default="auto", choices=["auto", "direct", "gram", "batched"],
                    help="Newton-Schulz form for every shape group (default: the autotuner's choice)")
    ap.add_argument("--step-only", action="store_true",
                    help="time the step alone: no per-kernel pass, end-to-end, AdamW or CPU baseline "
                         "(profiler runs)")
    ap.add_argument("--cache-file", default=None,
                    help="autotune cache: loaded before the warm-up if present, saved after it "
                         "(lets a profiled run replay the plans of an unprofiled one)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from newton_schulz_normalise_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    from newton_schulz_normalise_b200 import binding as B

    ws, rank, local = dist_env()
    if ws != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={ws}", file=sys.stderr)
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", init_method="env://", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    Ws, Gs, Ms = wl.generate(w, device=dev)
    shapes = w.shapes()
    pdt = B.DMUON_BF16 if w.param_dtype == "bf16" else B.DMUON_F32
    opts = B.options(pdt, pdt, variant=args.variant)
    # the parameter lists are marshalled once, as an optimiser loop would
    tW, tG, tM = B.TensorList(Ws), B.TensorList(Gs), B.TensorList(Ms)

    def step():
        B.dmuon_step_ex(tW, tG, tM, w.lr, w.wd, w.mu, w.ns_steps, opts=opts, stream=stream)

    def barrier():
        if ws > 1:
            dist.barrier()

    # warm-up (first call tunes each shape group and fills the cache); the
    # first and second calls are timed on the host around a synchronize, so
    # the line reports the autotune cost separately from the timed steps
    cache_loaded = bool(args.cache_file and os.path.exists(args.cache_file))
    if cache_loaded:
        B.dmuon_cache_load(args.cache_file)
    warm_s = []
    for k in range(args.warmup):
        t0 = time.perf_counter()
        step()
        if k < 2:
            torch.cuda.synchronize()
            warm_s.append(time.perf_counter() - t0)
    torch.cuda.synchronize()
    autotune = {"first_call_ms": round(warm_s[0] * 1e3, 1), "second_call_ms": round(warm_s[1] * 1e3, 1),
                "cache_loaded": cache_loaded,
                "note": "wall time of the first call (tunes every shape group when the cache is cold) "
                        "and of the second (tuned), each synchronised"}
    if args.cache_file and rank == 0:
        B.dmuon_cache_save(args.cache_file)
    plans = B.dmuon_cache_entries()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    # ---------------- device-timed region: K steps
    # Inputs larger than L2 are timed back to back.  Smaller parameter sets
    # would stay in L2 from one step to the next, so each step is preceded by
    # a 256 MB write (flushing the 126 MB L2) and timed by its own events.
    in_bytes = sum(t.numel() * t.element_size() for t in Ws + Gs + Ms)
    flush = in_bytes <= L2_BYTES
    fbuf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    barrier()
    torch.cuda.synchronize()
    l0 = B.dmuon_launch_count()
    t_host0 = time.time()
    if not flush:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1)
        l2_note = f"inputs {in_bytes / 1e6:.0f} MB > 126 MB L2, no flush between steps"
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            fbuf.fill_(i & 255)
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs)
        l2_note = (f"inputs {in_bytes / 1e6:.1f} MB fit in L2: a 256 MB write before every step, "
                   f"each step timed by its own events")
    t_host1 = time.time()
    barrier()
    launches = (B.dmuon_launch_count() - l0) // args.steps
    time.sleep(0.2)
    clocks.stop()
    clk = clocks.summary(t_host0, t_host1)
    if args.step_only:
        ms_max = reduce_max([ms], ws, device=dev)[0]
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": round(job_value(ms_max, args.steps, ws), 4), "unit": "ms",
                              "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": False,
                              "dtype": w.param_dtype, "config": {"workload": w.name, "l2": l2_note, "plans": plans},
                              "gpu_launches_per_step": launches, "clocks": clk, "step_only": True}), flush=True)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    # ---------------- per-kernel timing pass: the same steps again, the
    # Newton-Schulz products of every chunk bracketed by one pair of events
    # (no event between two products), other launches by their own pair;
    # about 3 s of steps
    B.dmuon_timing_reset()
    B.dmuon_timing_enable(True)
    kt_steps = max(1, min(args.steps, 50, int(3000.0 / max(ms / args.steps, 1e-3))))
    for _ in range(kt_steps):
        step()
    torch.cuda.synchronize()
    B.dmuon_timing_enable(False)
    kinds = {k: B.dmuon_timing_get(k) for k in (B.KIND_TC_GEMM, B.KIND_EW, B.KIND_SIMT_GEMM, B.KIND_OTHER,
                                                 B.KIND_TC_GEMM_PAIR)}
    B.dmuon_timing_reset()

    # ---------------- end to end through the C ABI with host buffers
    # dmuon_step_host_io: each step's gradients come from pinned host memory
    # and the updated parameters go back to pinned host memory; the library
    # pipelines both copies with the computation, chunk by chunk.
    # The pinned buffers are filled straight from the device (no pageable
    # copy on the way); every rank of the node needs its own, so the leg is
    # skipped, with the reason, when the host cannot hold them all.
    h2d = sum(g.numel() * g.element_size() for g in Gs)
    d2h = sum(x.numel() * x.element_size() for x in Ws)
    e2e_skip = host_memory_short(h2d + d2h, int(os.environ.get("LOCAL_WORLD_SIZE", "1")))
    if reduce_max([0.0 if e2e_skip is None else 1.0], ws, device=dev)[0] > 0 and e2e_skip is None:
        e2e_skip = "host memory short on another rank of the node"  # every rank takes the same branch
    e2e_ms = 0.0
    if e2e_skip is None:
        hG = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in Gs]
        for hg, g in zip(hG, Gs):
            hg.copy_(g)
        hW = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in Ws]
        thG, thW = B.TensorList(hG), B.TensorList(hW)

        def step_io():
            B.dmuon_step_host_io(tW, thG, tM, w.lr, w.wd, w.mu, w.ns_steps, params_host_out=thW, opts=opts,
                                 stream=stream)

        for _ in range(2):  # plans of the host-I/O chunking
            step_io()
    e2e_steps = max(3, min(args.steps, 20))
    barrier()
    torch.cuda.synchronize()
    if e2e_skip is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            step_io()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
        del hG, hW, thG, thW

    # ---------------- AdamW on the non-matrix parameters that train beside Muon
    # (a separate measurement, outside the step above): one 50304 x 1024
    # embedding table plus 96 vectors of 1024, in the workload's dtype, fp32
    # moments; 1.2 GB per launch (bf16) > L2.  Times dmuon_adamw_step alone.
    aw = adamw_measure(dev, stream, torch_dtype=wl.torch_dtype(w.param_dtype))

    # ---------------- reduce over ranks (max), report on rank 0
    ms_max, e2e_max = reduce_max([ms, e2e_ms], ws, device=dev)
    ms_per_step = ms_max / args.steps
    value = job_value(ms_max, args.steps, ws)

    peaks = measured_peaks()
    variants = {}
    for e in plans:  # "rows cols dtype steps variant bn cnt cost"
        f = e.split()
        variants[(int(f[0]), int(f[1]))] = f[4]
    gemm = kinds[B.KIND_TC_GEMM]
    pairk = kinds[B.KIND_TC_GEMM_PAIR]
    simt = kinds[B.KIND_SIMT_GEMM]
    # executed NS FLOPs per step (symmetric products count their computed tiles only)
    flops = (gemm["flops"] + simt["flops"]) / kt_steps
    # plans are keyed by the iterate's shape (min, max): a weight and its transpose share one
    dense = sum(ns_flops(r, c, w.ns_steps, variants.get((min(r, c), max(r, c)), "direct")) for r, c in shapes)
    tflops = flops / (ms_per_step * 1e-3) / 1e12
    peak_tc = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    variants_used = {e.split()[4] for e in plans}
    # the dominant kernel: the CTA-pair GEMM when its chains hold most of the
    # tensor-core time, else the tensor-core GEMMs together (one-CTA tiles,
    # resident kernel), else the fp32 SIMT GEMM
    if pairk["launches"] > 0 and pairk["ms"] >= 0.5 * gemm["ms"]:
        dom, dom_kernel, prof = pairk, "tc_gemm2_kernel (CTA pair)", "pair"
    elif gemm["launches"] > 0:
        dom, prof = gemm, None
        # a resident plan runs the small-matrix kernel (m <= 128, n <= 512),
        # the medium one (one CTA pair per matrix), or for an fp32 iterate
        # (iterates of at most 5 rows) the fp32 one
        def resident_kernel(e):
            f = e.split()
            if f[2] == "f32":
                return "ns_f32_kernel"
            return "ns_small_kernel" if int(f[0]) <= 128 and int(f[1]) <= 512 else "ns_mid_kernel"

        resident = {resident_kernel(e) for e in plans if e.split()[4] == "batched"}
        if variants_used == {"batched"}:
            dom_kernel = " / ".join(sorted(resident)) + " (resident)"
        else:
            dom_kernel = " / ".join(["tc_gemm_kernel", "tc_gemm2_kernel"] + sorted(resident))
    else:
        dom, prof = simt, None
        dom_kernel = ("ns_f32_kernel (fp32 FFMA, every step in one cooperative launch)"
                      if variants_used == {"batched"} else "simt_gemm_kernel (fp32 FFMA)")
    ach = dom["flops"] / (dom["ms"] * 1e-3) / 1e12 if dom["ms"] > 0 else 0.0
    share = round(dom["ms"] / kt_steps / ms_per_step, 3) if ms_per_step else None
    per_launch_ms = dom["ms"] / dom["launches"] if dom["launches"] else None
    if dom is not simt:
        traffic = (profile_traffic(ROOT / "newton_schulz_normalise_b200" / "csrc" / "gemm_tc.cu", w.name)
                   if prof == "pair" else None)
        roofline = {"bound": "tensor", "kernel": dom_kernel, "achieved": round(ach, 1),
                    "peak": peak_tc, "unit": "TFLOP/s", "frac": round(ach / peak_tc, 4),
                    "traffic": traffic, "peak_source": f"{peaks['_source']} bf16_tflops (burst)",
                    "frac_of_sustained": round(ach / peak_sus, 4),
                    "launches": dom["launches"] // kt_steps,
                    "ms_per_launch": round(per_launch_ms, 4) if per_launch_ms else None,
                    "flops_per_launch": dom["flops"] / dom["launches"] if dom["launches"] else None,
                    "share_of_step": share}
        if dom is pairk:  # all tensor-core GEMMs together, for reference
            roofline["all_tc_gemms"] = {
                "achieved": round(gemm["flops"] / (gemm["ms"] * 1e-3) / 1e12, 1) if gemm["ms"] > 0 else 0.0,
                "launches": gemm["launches"] // kt_steps,
                "share_of_step": round(gemm["ms"] / kt_steps / ms_per_step, 3) if ms_per_step else None}
    else:  # fp32 path: Newton-Schulz on the CUDA cores (FFMA)
        roofline = {"bound": "alu", "kernel": dom_kernel, "achieved": round(ach, 2),
                    "peak": round(FP32_FFMA_TFLOPS, 1), "unit": "TFLOP/s", "frac": round(ach / FP32_FFMA_TFLOPS, 4),
                    "traffic": None,
                    "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz",
                    "launches": dom["launches"] // kt_steps,
                    "ms_per_launch": round(per_launch_ms, 4) if per_launch_ms else None,
                    "share_of_step": share}
    ew = kinds[B.KIND_EW]
    ew_gbs = ew["bytes"] / (ew["ms"] * 1e-3) / 1e9 if ew["ms"] > 0 else 0.0

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 4), "unit": "ms", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": w.param_dtype,
            "data": "synthetic (seeded N(0,0.02^2) weights, N(0,1e-3^2) grads, zero fp32 momenta)",
            "config": {"workload": w.name, "matrices": len(shapes),
                       "shapes": sorted({f"{r}x{c}" for r, c in shapes}), "ns_steps": w.ns_steps,
                       "lr": w.lr, "wd": w.wd, "mu": w.mu, "parallelism": f"replicas{ws}",
                       "l2": l2_note,
                       "plans": plans},
            "ns_tflops": round(tflops, 1),
            "ns_frac_of_peak": round(tflops / peak_tc, 4),
            "ns_tflops_dense_equivalent": round(dense / (ms_per_step * 1e-3) / 1e12, 1),
            "roofline": roofline,
            "elementwise": {"bound": "hbm", "kernel": "momentum", "achieved": round(ew_gbs, 1),
                            "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": round(ew_gbs / peaks["hbm_gbs"], 4)},
            "adamw": {"bound": "hbm", "kernel": "adamw_kernel", "achieved": round(aw["gbs"], 1),
                      "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(aw["gbs"] / peaks["hbm_gbs"], 4),
                      "ms": round(aw["ms"], 4), "elements": aw["elements"], "bytes_per_element": aw["bpe"],
                      "set": "50304x1024 embedding + 96 x 1024 vectors"},
            "e2e": ({"value": round(job_value(e2e_max, 1, ws), 4), "unit": "ms", "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h} if e2e_skip is None else
                    {"value": None, "unit": "ms", "skipped": e2e_skip, "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h}),
            "gpu_launches": launches * args.steps,
            "gpu_launches_per_step": launches,
            "autotune": autotune,
            "clocks": clk,
        }
        if not args.no_cpu_baseline and ws == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
