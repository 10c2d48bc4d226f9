#!/usr/bin/env python
"""Benchmark of batched speculative-decoding verification on B200.

One step = one spec_verify_run over a resident batch: row statistics and the
accept chain for every request, the residual / bonus sample, and the fp64
refinement of the samples the fp32 filter could not certify.

Default workload: stochastic verification, B=256 requests, k=5 drafted
tokens each, all 5 verified, V=151936, bf16 logits (target ~ N(0, 3^2),
draft = 0.8 target + 0.6 N(0, 3^2)), T=1.  Metric: verified draft positions
per second (sum of L_i over the batch / step time), plus the HBM bandwidth
the step sustains.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload headline|stochastic|greedy|conf|conf_budget|sweep:B|lmhead]

``--workload lmhead`` times verification fused into the shared LM head
instead: the inputs are the two models' last hidden states (B=256, k=5,
H=2560, bf16) and the output head W [151936, 2560] bf16; one step is the
tcgen05 GEMM with the statistics epilogue, the accept chains, the GEMM of the
sampled rows and the sample.  Its roofline is the tensor-core one.

With N > 1 (launched by torch.distributed.run) every rank verifies its own
batch of the same shape (weak scaling, no collective on the data path); the
step time is the max over ranks.  ``--impl reference`` times the fp64 CPU
oracle instead, on the host's cores, one bounded sample of requests per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified draft positions/s and HBM GB/s (% of B200 peak), B=256 k=5 V=151936"
UNIT = "positions/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks (one per GPU, launched by torch.distributed.run when N > 1); "
                         "each verifies its own batch (weak scaling)")
    ap.add_argument("--steps", type=int, default=2000, help="timed steps")
    ap.add_argument("--warmup", type=int, default=20, help="untimed warm-up steps (at least 3)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"],
                    help="ours: the CUDA library; reference: the fp64 CPU oracle on the host "
                         "cores, on a bounded sample of the same workload")
    ap.add_argument("--workload", default="headline",
                    help="headline | stochastic | greedy | conf | conf_budget | sweep:B | lmhead")
    ap.add_argument("--timed-seconds", type=float, default=1.0,
                    help="repeat the timed block of --steps steps until this much time has "
                         "elapsed (0: one block, e.g. under a profiler)")
    ap.add_argument("--e2e-steps", type=int, default=5,
                    help="steps of the end-to-end measurement through host buffers (0: skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the oracle beside the GPU run")
    ap.add_argument("--mode", default="prefix", choices=["prefix", "dense", "auto"],
                    help="order of the statistics passes in the verification kernel")
    ap.add_argument("--prefix-tail", type=int, default=None,
                    help="prefix order: read a request's remaining positions together from "
                         "this position on (1..17; default: the library's)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a 512 MB buffer before every step (cold L2) and report the "
                         "kernel time of each launch")
    ap.add_argument("--lm-cta-pairs", type=int, default=2, choices=[0, 1, 2],
                    help="lmhead: GEMM tile form (0 one CTA per tile, 1 CTA pairs for both "
                         "GEMMs, 2 CTA pairs for the row-writing GEMM only)")
    ap.add_argument("--vocab-shards", type=int, default=1,
                    help="N > 1: time the vocabulary-parallel protocol with N ranks emulated "
                         "on this one GPU (one rank per context, exchanges as copies)")
    return ap.parse_args()


# ------------------------------------------------------------- workloads ----

def make_workload(name, device, rank):
    from speculative_decoding_verification_86_b200 import workloads as W
    if name == "headline":
        w = W.headline(device, seed=1)
    elif name == "stochastic":
        w = W.stochastic(device, seed=1)
    elif name == "greedy":
        w = W.greedy(device, seed=2)
    elif name == "conf":
        w = W.confidence(device, seed=3)
    elif name == "conf_budget":
        w = W.confidence_batch_budget(device, seed=3)
    elif name.startswith("sweep:"):
        w = W.sweep(device, seed=4, B=int(name.split(":")[1]))
    else:
        raise SystemExit("unknown workload %r" % name)
    return w


def effective_lengths(w, ver=None):
    """L_i after clamping and, with a confidence head, after its budgets: the
    lengths the run verifies (computed by the library when a verifier is
    given, else from verify_len alone)."""
    import torch
    B, kp1, _ = w["target"].shape
    k = kp1 - 1
    if w.get("conf") is not None and ver is not None:
        L, _ = ver.lengths(w["conf"], k, verify_len=w.get("verify_len"))
        torch.cuda.synchronize()
        return L
    L = (w["verify_len"].clamp(0, k) if w.get("verify_len") is not None
         else torch.full((B,), k, dtype=torch.int32, device=w["target"].device))
    return L


def dense_row_bytes(w, L):
    """Algorithmic bytes of the statistics pass: (L_i + 1) target rows and, for
    sampled requests, L_i draft rows, each V logits."""
    import torch
    V = w["target"].shape[2]
    es = w["target"].element_size()
    T = w.get("temperature")
    sampled = (T > 0) if T is not None else torch.ones_like(L, dtype=torch.bool)
    rows = (L + 1) + torch.where(sampled, L, torch.zeros_like(L))
    return int(rows.sum().item()) * V * es


def prefix_row_bytes(w, L, accepted):
    """Algorithmic bytes in prefix order: rows up to and including the first
    rejection (or the bonus row): n_i + 1 target rows and, for sampled
    requests, min(n_i + 1, L_i) draft rows."""
    import torch
    V = w["target"].shape[2]
    es = w["target"].element_size()
    T = w.get("temperature")
    sampled = (T > 0) if T is not None else torch.ones_like(L, dtype=torch.bool)
    n = accepted.clamp(min=0)
    rows = (n + 1) + torch.where(sampled, torch.minimum(n + 1, L), torch.zeros_like(L))
    return int(rows.sum().item()) * V * es


def config_dict(w, name, n, L):
    B, kp1, V = w["target"].shape
    return {
        "workload": w["name"],
        "B": int(B), "k": int(kp1 - 1), "V": int(V),
        "logits": "bf16" if w["target"].element_size() == 2 else "fp32",
        "mean_L": float(L.float().mean().item()),
        "temperature": "per-request" if w.get("temperature") is not None else 1.0,
        "confidence_head": w.get("conf") is not None,
        "l2": "no flush: the step reads %.0f MB of logits, more than the 126 MB L2"
              % (w["target"].numel() * w["target"].element_size() / 1e6
                 + (0 if w.get("draft") is None else w["draft"].numel() * w["draft"].element_size() / 1e6)),
        "parallelism": "replicas%d" % n if n > 1 else "single",
        "global_batch": int(B) * n,
    }


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        self.marks.append(time.time())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        t0, t1 = (self.marks + [0, 0])[:2]
        inside = [l for (t, l) in self.lines if t0 <= t <= t1 + 0.05]
        rows = [r.split(", ") for r in (inside or [l for _, l in self.lines[-3:]])]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[c - 5] for r in rows if len(r) >= 9 for c in range(5, 9)
                          if r[c].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows), "samples_in_timed_region": len(inside)}


# ---------------------------------------------------------------- timing ----

def timed_blocks(step, steps, stream, dev, world, seconds=1.0):
    """Time blocks of `steps` steps with CUDA events on the launching stream,
    a barrier and a device synchronisation on both sides of each, until about
    `seconds` have elapsed; each block's time is the max over ranks.
    Returns the per-block milliseconds (every rank gets the same list)."""
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_86_b200 import ranks
    out = []
    t0 = time.perf_counter()
    while True:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        out.append(ranks.max_over_ranks(e0.elapsed_time(e1), dev))
        elapsed = ranks.max_over_ranks((time.perf_counter() - t0) * 1e3, dev) / 1e3
        if elapsed >= seconds:
            return out


# -------------------------------------------------------------- roofline ----

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return None


# The device sources each profiled kernel is compiled from (host code, the C
# header and the other kernels' files do not change its machine code).
KERNEL_SOURCES = {
    "k_engine": ["common.cuh", "conf.cuh", "engine.cuh", "fp64.cuh", "philox.cuh", "refine.cuh",
                 "sample.cuh", "stage.cuh", "stats.cuh"],
    "k_lmhead": ["common.cuh", "philox.cuh", "stage.cuh", "stats.cuh", "lmhead.cuh"],
}


def _code_only(text):
    """Source text without comments and with whitespace collapsed: a change of
    comments alone does not change the machine code the counters describe."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel):
    from speculative_decoding_verification_86_b200 import build
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(build.CSRC, name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (same source hash); else None."""
    path = os.path.join(ROOT, "profiles", "%s_%s.md" % (kernel, workload))
    try:
        text = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            key, _, val = line.strip()[2:].partition(":")
            vals[key.strip()] = val.strip().strip("`")
    if vals.get("source_hash") != kernel_source_hash(kernel):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- oracle ----

def oracle_sample(w, n_requests, threads):
    """Run the fp64 oracle on the first n_requests of the batch; returns (seconds, positions)."""
    import oracle
    from speculative_decoding_verification_86_b200 import workloads as W
    sub = {k: (v[:n_requests] if hasattr(v, "shape") and v.dim() > 0 and v.shape[0] == w["target"].shape[0] else v)
           for k, v in w.items()}
    if w.get("conf") is not None:
        sub["conf"] = dict(w["conf"], hidden=w["conf"]["hidden"][:n_requests])
    h = W.to_numpy_inputs(sub)
    t0 = time.perf_counter()
    res = oracle.verify(h["target"], h["draft"], h["tokens"], dtype=h["dtype"], verify_len=h["verify_len"],
                        temperature=h["temperature"], conf=h["conf"], seed=h["seed"], threads=threads)
    dt = time.perf_counter() - t0
    return dt, int(res["verify_len_used"].sum()), h


def run_reference(args):
    """The fp64 CPU oracle, timed on the host's cores (reference arm)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import torch
    oracle.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = make_workload(args.workload, dev, 0)
    L = effective_lengths(w)
    cores = os.cpu_count() or 1
    B = int(w["target"].shape[0])
    per_step = max(1, min(B, cores))
    for _ in range(max(0, args.warmup)):
        oracle_sample(w, per_step, per_step)
    tot_t, tot_pos = 0.0, 0
    for _ in range(args.steps):
        dt, pos, _ = oracle_sample(w, per_step, per_step)
        tot_t += dt
        tot_pos += pos
    value = tot_pos / tot_t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": max(0, args.warmup),
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args.workload, 1, L),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": per_step, "kind": "oracle",
                         "sample": "first %d requests of the batch per step, one per thread" % per_step},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours ----

def run_ours(args):
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_86_b200 import binding, build, ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    build.build()
    w = make_workload(args.workload, dev, rank)
    B, kp1, V = w["target"].shape
    k = kp1 - 1
    ver = binding.SpecVerifier(dev, max_batch=max(B, 1), max_k=max(k, 1), max_vocab=V, mode=args.mode)
    if args.prefix_tail is not None:
        ver.set_prefix_tail(args.prefix_tail)
    L = effective_lengths(w, ver)
    positions = int(L.sum().item())
    step_bytes = dense_row_bytes(w, L)
    out = ver._outputs(B, k, True)
    stream = torch.cuda.current_stream(dev)

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None

    def step():
        if flush is not None:
            flush.fill_(1)  # evicts the 126 MB L2 before the verification
        ver.run(w["target"], w.get("draft"), w["tokens"], verify_len=w.get("verify_len"),
                temperature=w.get("temperature"), conf=w.get("conf"), seed=w["seed"],
                request_offset=ranks.weak_offset(B, rank), out=out)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    phys = int(visible.split(",")[local]) if visible else local
    clocks = ClockSampler(phys)
    clocks.start()
    time.sleep(0.2)
    ver.timing_enable([binding.TIMING_STATS, binding.TIMING_CONF])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark()
    block_ms = timed_blocks(step, args.steps, stream, dev, world, args.timed_seconds)
    clocks.mark()
    n_stats, ms_stats = ver.timing_read(binding.TIMING_STATS)
    n_conf, ms_conf = ver.timing_read(binding.TIMING_CONF)
    ver.timing_enable([])
    clk = clocks.stop()
    counters = ver.last_counters()
    # the other statistics order, timed the same way on the same batch
    other = "prefix" if ver.mode == "dense" else "dense"
    ver.set_mode(other)
    for _ in range(3):
        step()
    nb = min(args.steps, 500)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    o0 = torch.cuda.Event(enable_timing=True)
    o1 = torch.cuda.Event(enable_timing=True)
    o0.record(stream)
    for _ in range(nb):
        step()
    o1.record(stream)
    torch.cuda.synchronize(dev)
    other_ms = ranks.max_over_ranks(o0.elapsed_time(o1), dev) / nb
    other_line = {"mode": other, "ms_per_step": other_ms,
                  "value": positions * world / (other_ms / 1e3),
                  "hbm_gbs": dense_row_bytes(w, L) / (other_ms * 1e-3) / 1e9 if other == "dense" else None}
    ver.set_mode(args.mode)
    ms_per_step = statistics.median(block_ms) / args.steps
    if flush is not None and n_stats:
        # the step includes the flush: report the verification launches alone
        ms_per_step = ranks.max_over_ranks(ms_stats / n_stats + (ms_conf / n_conf if n_conf else 0.0), dev)
    value = positions * world / (ms_per_step / 1e3)
    # k_engine; with a confidence head in the dense order, k_conf before it
    # (the benchmark's confidence workloads are large enough for "auto" to
    # resolve to the prefix order)
    launches_per_step = 1 + (1 if (w.get("conf") is not None and ver.mode == "dense") else 0)

    # end to end: host buffers in, host results out, through the C ABI
    e2e = None
    if args.e2e_steps > 0:
        host = {key: (v.detach().cpu().pin_memory() if isinstance(v, torch.Tensor) else v)
                for key, v in w.items()}
        hconf = None
        if w.get("conf") is not None:
            hconf = dict(w["conf"], hidden=w["conf"]["hidden"].cpu().pin_memory(),
                         w=w["conf"]["w"].cpu().pin_memory())
        hout = dict(accepted=torch.empty(B, dtype=torch.int32).pin_memory(),
                    tokens=torch.empty((B, k + 1), dtype=torch.int32).pin_memory(),
                    p=torch.empty((B, k), dtype=torch.float32).pin_memory(),
                    q=torch.empty((B, k), dtype=torch.float32).pin_memory(),
                    status=torch.empty(B, dtype=torch.int32).pin_memory())

        def hstep():
            ver.run_host(host["target"], host.get("draft"), host["tokens"], verify_len=host.get("verify_len"),
                         temperature=host.get("temperature"), conf=hconf, seed=w["seed"],
                         request_offset=ranks.weak_offset(B, rank), out=hout)

        hstep()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            hstep()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = ranks.max_over_ranks(a0.elapsed_time(a1), dev) / args.e2e_steps
        h2d = sum(v.numel() * v.element_size() for key, v in host.items()
                  if isinstance(v, torch.Tensor) and key in ("target", "draft", "tokens", "verify_len", "temperature"))
        if hconf is not None:
            h2d += hconf["hidden"].numel() * 2 + hconf["w"].numel() * 2
        d2h = sum(v.numel() * v.element_size() for v in hout.values())
        e2e = {"value": positions * world / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    # CPU baseline: the fp64 oracle on this host, rank 0 at N = 1 only
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        t1, pos1, _ = oracle_sample(w, 1, 1)
        n = int(max(1, min(B, round(cores * 10.0 / max(t1, 1e-3)))))
        threads = min(cores, n)
        # repeat the sample until about 10 s of CPU time have been measured
        dt, pos, reps = 0.0, 0, 0
        while reps == 0 or (dt < 10.0 and reps < 64):
            d1, p1, _ = oracle_sample(w, n, threads)
            dt, pos, reps = dt + d1, pos + p1, reps + 1
        cpu = {"value": pos / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "first %d of %d requests of this batch, %d times, fp64 C oracle, %d threads, %.1f s"
                         % (n, B, reps, threads, dt)}

    peaks = measured_peaks()
    if peaks and peaks.get("hbm_gbs"):
        peak, peak_src = float(peaks["hbm_gbs"]), "measured"
    else:
        peak, peak_src = FALLBACK_HBM_GBS, "fallback"
    ms_stats_avg = ms_stats / max(n_stats, 1)
    algo_bytes = step_bytes if args.mode == "dense" else prefix_row_bytes(w, L, out["accepted"])
    achieved = algo_bytes / (ms_stats_avg * 1e-3) / 1e9 if n_stats else None
    traffic = profiled_traffic("k_engine", "%s_%s" % (args.workload.replace(":", ""), args.mode))
    step_gbs = algo_bytes / (ms_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w["target"].element_size() == 2 else "f32",
        "data": "synthetic", "config": dict(config_dict(w, args.workload, world, L), **(
            {"l2": "flushed (512 MB write) before every step; kernel time per launch"} if flush is not None else {})),
        "hbm_gbs": step_gbs, "hbm_frac_measured": step_gbs / peak, "hbm_frac_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "kernel": "k_engine", "achieved": achieved, "peak": peak,
                     "peak_source": peak_src, "unit": "GB/s",
                     "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                     "algorithmic_bytes_per_launch": algo_bytes,
                     "algorithmic_bytes_dense": step_bytes,
                     "launch_ms": ms_stats_avg, "launches_timed": n_stats},
        "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps * len(block_ms),
        "timed_blocks": {"blocks": len(block_ms), "steps_per_block": args.steps,
                         "ms_per_block_min": min(block_ms), "ms_per_block_median": statistics.median(block_ms),
                         "ms_per_block_max": max(block_ms)},
        "fp64_paths": counters,
        "conf_launch_ms": (ms_conf / n_conf) if n_conf else None,
        "mode": args.mode,
        "prefix_tail": args.prefix_tail,
        "other_mode": other_line,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ver.close()
    if world > 1:
        dist.destroy_process_group()


def run_vocab_parallel(args):
    """The vocabulary-parallel protocol with N ranks emulated on one GPU.  Every
    rank's phases are timed with events on the stream; a step on N GPUs would
    take the slowest rank's phases plus three small collectives (not timed
    here: no run of this build has more than one GPU)."""
    import torch
    from speculative_decoding_verification_86_b200 import binding, build
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = make_workload(args.workload, dev, 0)
    B, kp1, V = w["target"].shape
    k = kp1 - 1
    n = args.vocab_shards
    bounds, b1, b2, b3 = binding.shard_layout(B, k, V, w["target"].dtype, n)
    ranks = [binding.ShardRank(dev, r, n, max_batch=B, max_k=max(k, 1), max_vocab=V) for r in range(n)]
    shards = [(w["target"][:, :, bounds[r]:bounds[r + 1]].contiguous(),
               None if w.get("draft") is None else w["draft"][:, :, bounds[r]:bounds[r + 1]].contiguous())
              for r in range(n)]
    kw = dict(verify_len=w.get("verify_len"), temperature=w.get("temperature"), conf=w.get("conf"))
    all1 = torch.empty(n * b1, dtype=torch.uint8, device=dev)
    all2 = torch.empty(n * b2, dtype=torch.uint8, device=dev)
    all3 = torch.empty(n * b3, dtype=torch.uint8, device=dev)
    votes = torch.empty((n, B), dtype=torch.int32, device=dev)
    outs = [rk.ver._outputs(B, k, True) for rk in ranks]
    ev = lambda: torch.cuda.Event(enable_timing=True)
    phase_ms = [[0.0, 0.0, 0.0, 0.0] for _ in range(n)]
    redo_counts = []

    def step(timed):
        marks = []
        for r, rk in enumerate(ranks):
            e0, e1 = ev(), ev()
            e0.record()
            rk.stats(shards[r][0], shards[r][1], w["tokens"], V, all1[r * b1:(r + 1) * b1], **kw)
            e1.record()
            marks.append((r, 0, e0, e1))
        for r, rk in enumerate(ranks):
            e0, e1 = ev(), ev()
            e0.record()
            rk.decide(all1, shards[r][0], shards[r][1], w["tokens"], V, outs[r],
                      all2[r * b2:(r + 1) * b2], seed=w["seed"], **kw)
            e1.record()
            marks.append((r, 1, e0, e1))
        for r, rk in enumerate(ranks):
            e0, e1 = ev(), ev()
            e0.record()
            rk.locate(all2, shards[r][0], shards[r][1], w["tokens"], V, votes[r], **kw)
            e1.record()
            marks.append((r, 2, e0, e1))
        vmax = votes.max(dim=0).values.contiguous()
        redo = [rk.finish(vmax, outs[r]) for r, rk in enumerate(ranks)][0]
        if bool((redo == 2).any()):
            for r, rk in enumerate(ranks):
                e0, e1 = ev(), ev()
                e0.record()
                rk.refine_partials(shards[r][0], shards[r][1], w["tokens"], V,
                                   all3[r * b3:(r + 1) * b3], **kw)
                rk.refine_locate(all3, shards[r][0], shards[r][1], w["tokens"], V, votes[r], **kw)
                e1.record()
                marks.append((r, 3, e0, e1))
            vmax = votes.max(dim=0).values.contiguous()
            redo = [rk.refine_finish(vmax, outs[r]) for r, rk in enumerate(ranks)][0]
        torch.cuda.synchronize()
        if timed:
            for r, ph, e0, e1 in marks:
                phase_ms[r][ph] += e0.elapsed_time(e1)
            redo_counts.append(int((redo == 1).sum().item()))

    for _ in range(max(args.warmup, 3)):
        step(False)
    steps = min(args.steps, 200)
    for _ in range(steps):
        step(True)
    per_rank = [[x / steps for x in ph] for ph in phase_ms]
    slowest = max(sum(ph) for ph in per_rank)
    L = effective_lengths(w, ranks[0].ver)
    positions = int(L.sum().item())
    line = {
        "metric": "vocabulary-parallel verification, %d ranks emulated on one GPU" % n,
        "value": positions / (slowest * 1e-3), "unit": "positions/s (slowest rank's phases)",
        "n_gpus": 1, "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step_slowest_rank": slowest,
        "higher_is_better": True, "data": "synthetic", "dtype": "bf16" if w["target"].element_size() == 2 else "f32",
        "config": {"workload": w["name"], "vocab_bounds": bounds},
        "per_rank_ms": [{"stats": a, "decide_and_masses": b, "locate": c, "fp64_refinement": d}
                        for a, b, c, d in per_rank],
        "exchange_bytes_per_rank": {"block1": b1, "block2": b2, "block3": b3, "votes": 4 * B},
        "requests_redone_per_step": sum(redo_counts) / max(len(redo_counts), 1),
        "note": "excludes the collectives (3, or 5 with a refinement) and whole redos",
    }
    print(json.dumps(line), flush=True)
    for rk in ranks:
        rk.close()


LM_METRIC = ("verified draft positions/s, verification fused into the shared LM head "
             "(B=256 k=5 V=151936 H=2560)")
LM_LAUNCHES_PER_STEP = 16  # kernels spec_lmhead_verify launches (no confidence head)


def lm_config(w, n):
    B, kp1, H = w["hidden_target"].shape
    return {"workload": w["name"], "B": int(B), "k": int(kp1 - 1), "V": int(w["head"].shape[0]),
            "H": int(H), "hidden": "bf16", "logits": "fp32 accumulators (never stored)",
            "temperature": 1.0, "mean_L": float(kp1 - 1),
            "l2": "no flush: the head alone is %.0f MB, more than the 126 MB L2"
                  % (w["head"].numel() * 2 / 1e6),
            "parallelism": "replicas%d" % n if n > 1 else "single", "global_batch": int(B) * n}


def lm_oracle_sample(w, n_requests, threads):
    """fp64 oracle on the first n_requests: the head's logits of their rows, then
    the verification; returns (seconds, positions)."""
    import numpy as np
    import oracle

    def bits(t):
        return t.detach().cpu().contiguous().view(torch_int16()).numpy().view(np.uint16)

    hs = bits(w["hidden_target"][:n_requests])
    hd = bits(w["hidden_draft"][:n_requests])
    W = bits(w["head"])
    tok = w["tokens"][:n_requests].cpu().numpy()
    t0 = time.perf_counter()
    res = oracle.verify_lmhead(hs, hd, W, tok, seed=w["seed"], threads=threads)
    dt = time.perf_counter() - t0
    return dt, int(res["verify_len_used"].sum())


def blas_threads():
    """Threads numpy's BLAS runs the oracle's matmul on."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def torch_int16():
    import torch
    return torch.int16


def run_lmhead(args):
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_86_b200 import binding, build, ranks, workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    build.build()
    w = W.lmhead(dev, seed=5)
    ht, hd, head, tok = w["hidden_target"], w["hidden_draft"], w["head"], w["tokens"]
    B, kp1, H = ht.shape
    k = kp1 - 1
    V = head.shape[0]
    ver = binding.SpecVerifier(dev, max_batch=B, max_k=k, max_vocab=V, mode="dense")
    lm = binding.LmHeadVerifier(ver, max_hidden=H, cta_pairs=args.lm_cta_pairs)
    positions = B * k
    out = ver._outputs(B, k, True)
    stream = torch.cuda.current_stream(dev)
    off = ranks.weak_offset(B, rank)

    def step():
        lm.verify(ht, hd, head, tok, seed=w["seed"], request_offset=off, out=out, redo_whole=False)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    redo_warm = int(out["redo"].sum().item())
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    phys = int(visible.split(",")[local]) if visible else local
    clocks = ClockSampler(phys)
    clocks.start()
    time.sleep(0.2)
    ver.timing_enable([binding.TIMING_LM_STATS, binding.TIMING_LM_ROWS])
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark()
    block_ms = timed_blocks(step, args.steps, stream, dev, world, args.timed_seconds)
    clocks.mark()
    n_st, ms_st = ver.timing_read(binding.TIMING_LM_STATS)
    n_rw, ms_rw = ver.timing_read(binding.TIMING_LM_ROWS)
    ver.timing_enable([])
    clk = clocks.stop()
    redo_last = int(out["redo"].sum().item())
    ms_per_step = statistics.median(block_ms) / args.steps
    value = positions * world / (ms_per_step / 1e3)

    # the unfused pipeline on the same inputs (this GEMM writing fp32 logits,
    # then the verifier), and cuBLAS's bf16 GEMM of the same shape, for context
    tl = torch.empty((B, k + 1, V), dtype=torch.float32, device=dev)
    dl = torch.empty((B, k, V), dtype=torch.float32, device=dev)
    hall = torch.cat([ht.reshape(-1, H), hd.reshape(-1, H)]).contiguous()

    def timed(fn, n):
        # the same timed blocks as the fused pipeline above (median block), so
        # all three are compared at the same settled power state
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        return statistics.median(timed_blocks(fn, n, stream, dev, world, args.timed_seconds)) / n

    def unfused():
        lm.logits(ht, head, out=tl)
        lm.logits(hd, head, out=dl)
        ver.run(tl, dl, tok, seed=w["seed"], request_offset=off)

    nb = max(3, min(args.steps, 50))
    unfused_ms = timed(unfused, nb)
    cublas_ms = timed(lambda: torch.matmul(hall, head.T), nb)
    del tl, dl

    # end to end: hidden states and tokens from pinned host memory, outputs back
    e2e = None
    if args.e2e_steps > 0:
        h_ht, h_hd, h_tok = ht.cpu().pin_memory(), hd.cpu().pin_memory(), tok.cpu().pin_memory()
        d_ht, d_hd, d_tok = torch.empty_like(ht), torch.empty_like(hd), torch.empty_like(tok)
        hout = {key: torch.empty(v.shape, dtype=v.dtype).pin_memory() for key, v in out.items()}

        def hstep():
            d_ht.copy_(h_ht, non_blocking=True)
            d_hd.copy_(h_hd, non_blocking=True)
            d_tok.copy_(h_tok, non_blocking=True)
            o = lm.verify(d_ht, d_hd, head, d_tok, seed=w["seed"], request_offset=off, out=out)
            for key in hout:
                hout[key].copy_(o[key], non_blocking=True)

        hstep()
        torch.cuda.synchronize(dev)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            hstep()
        a1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = ranks.max_over_ranks(a0.elapsed_time(a1), dev) / args.e2e_steps
        h2d = sum(t.numel() * t.element_size() for t in (h_ht, h_hd, h_tok))
        d2h = sum(t.numel() * t.element_size() for t in hout.values())
        e2e = {"value": positions * world / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "note": "the public call with its whole-request redo check (one host sync per step)"}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        dt, pos = lm_oracle_sample(w, 1, 1)
        cpu = {"value": pos / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": "request 0 of %d: fp64 head logits of its 11 rows (numpy matmul on the "
                         "BLAS threads) then the fp64 C oracle on one thread, %.1f s" % (B, dt)}

    peaks = measured_peaks()
    if peaks and peaks.get("bf16_tflops"):
        peak, peak_src = float(peaks["bf16_tflops"]), "measured burst (cuBLAS bf16)"
    else:
        peak, peak_src = 1590.0, "fallback"
    import numpy as np
    rows = B * (2 * k + 1)
    flops = 2.0 * rows * V * H  # the whole head applied to every row: the unfused GEMM, cuBLAS
    # the rows the prefix-ordered statistics passes computed: position 0 of every
    # request, then the other rows of the requests that accepted position 0
    acc = out["accepted"].cpu().numpy()
    temp = w.get("temperature")
    tn = temp.cpu().numpy() if temp is not None else np.ones(B)
    vl = w.get("verify_len")
    lv = np.clip(vl.cpu().numpy(), 0, k) if vl is not None else np.full(B, k)
    cont = acc >= 1
    rows_done = B * (2 if k > 0 else 1) + int(np.sum(np.where(tn[cont] == 0, lv[cont], 2 * lv[cont] - 1)))
    flops_done = 2.0 * rows_done * V * H
    st_ms = ms_st / max(len(block_ms) * args.steps, 1)  # both statistics launches of a step
    achieved = flops_done / (st_ms * 1e-3) / 1e12
    line = {
        "metric": LM_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(lm_config(w, world), cta_pairs=args.lm_cta_pairs),
        "roofline": {"bound": "tensor", "kernel": "k_lmhead (statistics epilogue)",
                     "achieved": achieved, "peak": peak, "peak_source": peak_src,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_of_sustained": (achieved / float(peaks["bf16_tflops_sustained"])
                                           if peaks and peaks.get("bf16_tflops_sustained") else None),
                     "traffic": profiled_traffic("k_lmhead", "lmhead_stats_pairs" if args.lm_cta_pairs == 1
                                                  else "lmhead_stats"),
                     "flops_per_step": flops_done, "rows_per_step": rows_done, "rows_all": rows,
                     "ms_per_step": st_ms, "launches_timed": n_st},
        "timed_blocks": {"blocks": len(block_ms), "steps_per_block": args.steps,
                         "ms_per_block_min": min(block_ms), "ms_per_block_median": statistics.median(block_ms),
                         "ms_per_block_max": max(block_ms)},
        "rows_gemm_ms": ms_rw / max(n_rw, 1),
        "unfused_ms_per_step": unfused_ms,
        "unfused_value": positions * world / (unfused_ms / 1e3),
        "cublas_bf16_gemm_ms": cublas_ms,
        "cublas_bf16_gemm_tflops": flops / (cublas_ms * 1e-3) / 1e12,
        "requests_redone": {"warmup_last_step": redo_warm, "timed_last_step": redo_last},
        "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
        "gpu_launches": LM_LAUNCHES_PER_STEP * args.steps * len(block_ms),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    lm.close()
    ver.close()
    if world > 1:
        dist.destroy_process_group()


def run_lmhead_reference(args):
    """The fp64 oracle on the LM-head workload (reference arm), host cores."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle
    import torch
    from speculative_decoding_verification_86_b200 import workloads as W
    oracle.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = W.lmhead(dev, seed=5)
    for _ in range(max(0, min(args.warmup, 1))):
        lm_oracle_sample(w, 1, 1)
    tot_t, tot_pos = 0.0, 0
    for _ in range(args.steps):
        dt, pos = lm_oracle_sample(w, 1, 1)
        tot_t += dt
        tot_pos += pos
    value = tot_pos / tot_t
    line = {
        "impl": "reference", "metric": LM_METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": max(0, min(args.warmup, 1)),
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": lm_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": "one request per step: fp64 head logits of its rows (BLAS "
                                   "threads), then the oracle on one thread"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.workload == "lmhead":
        if args.impl == "reference":
            run_lmhead_reference(args)
        else:
            run_lmhead(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.vocab_shards > 1:
        run_vocab_parallel(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
