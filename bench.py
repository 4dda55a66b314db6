#!/usr/bin/env python
"""Prefill throughput of the STILL hybrid-attention layer on B200, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one still_hybrid_prefill over one batch of synthetic input: saliency,
per-chunk top-k + gather, NP-Map of the keys, linear state, softmax/linear
merge (every step of the layer).  Prints ONE JSON line (rank 0).

* value: tokens/s of the whole job (B*N tokens per step per GPU), inputs resident
  in HBM, L2 flushed (a 512 MiB write) before every step outside the timed
  events; per-step CUDA events on the launching stream, max over ranks.
* e2e: the same metric through the same call with pinned HOST buffers, the
  host->device copies of q, k, v, Wq, Wk and the device->host copy of o inside
  the timed region.
* roofline: the merge kernel (dominant), algorithmic FLOPs per launch over its
  event-timed duration, against the measured bf16 dense peak.
* cpu_baseline: the fp64 oracle on the host cores, on a bounded sample of the
  same workload (whole (batch, KV-group) slices, every query row or a stride
  of them, about 15 s of CPU work), scaled to the whole layer.
* --impl reference: that oracle arm alone, as the line's value.
Multi-GPU: independent replicas (the layer has no cross-GPU exchange), weak scaling.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_still_b200.synth import WORKLOADS, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "llama32_1b_layer_n16k"
METRIC = "STILL hybrid-attn prefill tokens/s per layer at 16K/64K; % of roofline"
METRIC_DECODE = "STILL chunk-delayed decode tokens/s per layer (one token per sequence per step)"
METRIC_BACKWARD = "STILL hybrid-attn backward tokens/s per layer (gradients of q, k, v, Wq, Wk)"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=None, choices=sorted(WORKLOADS))
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="target oracle time of the CPU baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--keep", choices=["config", "all", "none", "window"], default="config",
                   help="tokens kept per chunk: the workload's k, all of them (k = C: exact causal softmax "
                        "attention through the same kernels, a same-box dense comparator), none (k = 0: "
                        "window + linear branch only), or window (k = 0 with a window of the whole sequence: "
                        "exact causal softmax attention in the window phase alone, flash-style, with no "
                        "selection, kept cache or linear state)")
    p.add_argument("--pass", dest="pass_", choices=["forward", "backward"], default="forward",
                   help="prefill workloads: time the forward layer (default) or its backward pass "
                        "(gradients of q, k, v, Wq, Wk with the selection held fixed)")
    p.add_argument("--bwd-stats", choices=["saved", "recompute"], default="saved",
                   help="backward pass: take each row's normaliser and D_i from the forward's output and "
                        "normaliser (saved, what a training step has at hand) or form them again (recompute)")
    p.add_argument("--workloads", choices=["auto", "none"], default="auto",
                   help="auto: a default single-GPU run (no --workload, forward pass, default router and keep) "
                        "also measures the other layer configurations (8B-shaped prefill at B4 x 16K and "
                        "1 x 64K, the B16 x 64K decode) and reports each under `workloads`")
    p.add_argument("--router", choices=["saliency", "diagonal"], default="saliency",
                   help="prefill token router: the Self-Saliency Score, or the diagonal-only ablation "
                        "(score -> per-chunk top-k -> prefill with that selection)")
    a = p.parse_args()
    a.workload_given = a.workload is not None
    if a.workload is None:
        a.workload = DEFAULT_WORKLOAD
    return a


# ----------------------------------------------------------------------------- algorithmic counts

def soft_sizes(shape, N=None):
    """|Soft(i)| for every query position i (same for every (b, h))."""
    import numpy as np
    N = shape.N if N is None else N
    i = np.arange(N, dtype=np.int64)
    if shape.w == 0:
        return np.zeros(N, dtype=np.int64)
    m = shape.w // shape.C
    t = i // shape.C
    lo = np.maximum(0, (t - m) * shape.C)
    return (i - lo + 1) + shape.k * np.maximum(0, t - m)


def merge_flops(shape):
    """Algorithmic FLOPs of the merge kernel per launch: 4d per (query-head, softmax key) for QK^T and
    PV, plus 2dD for phi(q) = NP-Map GEMV and 2dD + 2D for phi(q)^T S and phi(q)^T z per query-head."""
    rows = shape.B * shape.H
    return rows * (4 * shape.d * int(soft_sizes(shape).sum()) + shape.N * (4 * shape.d * shape.D + 2 * shape.D))


EX2_PER_CLOCK_PER_SM = 16  # ex2.approx: one warp instruction per 8 cycles on each of the 4 SMSPs (microbenchmarked)


def merge_exps(shape):
    """Exponentials of the merge kernel per step: one per (query-head, softmax key)."""
    return shape.B * shape.H * int(soft_sizes(shape).sum())


def exp_pipe_diag(shape, merge_ms_per_step, clocks=None, sms: int = 148):
    """The merge's exponential rate against the MUFU ceiling (EX2_PER_CLOCK_PER_SM x SMs x the median
    SM clock seen during the timed region, else the 1965 MHz maximum): a diagnostic beside the
    tensor roofline, the tighter of the two at d = 64.  None without a merge time."""
    if not merge_ms_per_step:
        return None
    mhz = (clocks or {}).get("sm_mhz") or 1965.0
    peak = EX2_PER_CLOCK_PER_SM * sms * mhz * 1e6
    exps = merge_exps(shape)
    achieved = exps / (merge_ms_per_step / 1e3)
    flop_s = merge_flops(shape) / (merge_ms_per_step / 1e3)
    return {"exps_per_step": exps, "achieved": achieved, "peak": peak, "unit": "ex2/s", "frac": achieved / peak,
            "sm_mhz": mhz, "sms": sms, "ms_at_exp_peak": exps / peak * 1e3,
            "flops_per_exp": merge_flops(shape) / max(exps, 1), "achieved_tflops": flop_s / 1e12}


def nowin_flops(shape):
    """Algorithmic FLOPs of a w = 0 step (pure chunked linear attention): per (query-head, key of the
    query's own chunk up to the query) 2D for <phi(q), phi(k)> and 2d for the weighted value; per
    query-head 2dD for phi(q), 2dD + 2D for phi(q)^T S_t and phi(q)^T z_t; per key of a KV head 2dD
    for phi(k) and 2dD for its outer product with v."""
    import numpy as np
    N, d, D, C = shape.N, shape.d, shape.D, shape.C
    i = np.arange(N, dtype=np.int64)
    intra = int((i - (i // C) * C + 1).sum())
    return shape.B * shape.H * (2 * (D + d) * intra + N * (4 * d * D + 2 * D)) + shape.B * shape.Hkv * N * 4 * d * D


def layer_flops(shape):
    """Algorithmic FLOPs of one whole step (all kernels)."""
    import numpy as np
    N, d, D = shape.N, shape.d, shape.D
    band = np.minimum(np.arange(N) + 1, shape.w) if shape.w > 0 else np.zeros(N)
    sal = shape.B * shape.H * 2 * d * float(band.sum()) if shape.k > 0 else 0.0
    phik = shape.B * shape.Hkv * N * 2 * d * D
    lin = shape.B * shape.Hkv * N * 2 * D * d
    if shape.w == 0:
        return nowin_flops(shape)
    return merge_flops(shape) + sal + phik + lin


# ----------------------------------------------------------------------------- clocks

def profiled_traffic(workload: str, prefix: str = "merge_"):
    """DRAM bytes per step of the profiled launches (the merge pair; with prefix "bwd_", the
    backward's dq kernel) from a committed ncu summary under profiles/<prefix>*.md (a block of
    `workload:`, `traffic_bytes_per_step:` and `source_sha256:` lines), or None when there is none
    for this workload or the kernel sources changed since the capture."""
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", prefix + "*.md"))):
        blocks, kv = [], {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("    ") and not line.startswith("     "):
                    k_, _, v_ = line.strip().partition(": ")
                    if k_ == "workload" and kv:
                        blocks.append(kv)
                        kv = {}
                    kv[k_] = v_
        if kv:
            blocks.append(kv)
        for kv in blocks:
            if kv.get("workload") != workload or "traffic_bytes_per_step" not in kv:
                continue
            fresh = True
            for item in kv.get("source_sha256", "").split():
                name, _, digest = item.partition("=")
                src = os.path.join(ROOT, "linear_attention_still_b200", "csrc", name)
                try:
                    with open(src, "rb") as f:
                        fresh = fresh and hashlib.sha256(f.read()).hexdigest().startswith(digest)
                except OSError:
                    fresh = False
            if fresh:
                return int(kv["traffic_bytes_per_step"])
    return None


class ClockSampler:
    """SM clock, power and clock-event reasons sampled DURING a timed region (reads only).

    In-process NVML queries every `period_s` (2 ms) from a thread, so that even a timed region of a
    few tens of milliseconds gets samples of its own; falls back to an `nvidia-smi -lms 20` child
    when NVML cannot be loaded."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                   "sw_power_cap": 0x4}

    def __init__(self, gpu_id: str | None, period_s: float = 0.002, nvml=None):
        self.rows = []          # (sm_mhz, sm_max_mhz, power_w, set of reason names)
        self.proc = None
        self.thread = None
        self.gpu_id = gpu_id
        self.period_s = period_s
        self.source = None
        self._nvml = nvml
        self._stop = threading.Event()

    def _nvml_handle(self):
        nv = self._nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        if self.gpu_id:
            h = nv.nvmlDeviceGetHandleByUUID(self.gpu_id)
        else:
            h = nv.nvmlDeviceGetHandleByIndex(0)
        return nv, h

    def _nvml_sample(self, nv, h):
        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        try:
            pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            pw = None
        bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
        self.rows.append((sm, smax, pw, {n for n, b in self.REASON_BITS.items() if bits & b}))

    def _nvml_loop(self, nv, h):
        while not self._stop.is_set():
            try:
                self._nvml_sample(nv, h)
            except Exception:
                return
            self._stop.wait(self.period_s)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self._nvml_sample(nv, h)  # fails here, not in the thread, when a query is unsupported
            self.rows.clear()
            self.source = f"nvml, every {self.period_s * 1e3:g} ms"
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            self.rows.clear()
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits", "-lms", "20"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi -lms 20"
        self.thread = threading.Thread(target=self._smi_read, daemon=True)
        self.thread.start()
        # nvidia-smi takes a moment to start: wait for its first sample, then keep only later ones
        t_end = time.time() + 5.0
        while not self.rows and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)
        self.rows.clear()

    def _smi_read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == len(self.FIELDS) and num(parts[1]) is not None:
                self.rows.append((num(parts[1]), num(parts[2]), num(parts[3]),
                                  {names[j] for j in range(4) if parts[5 + j].lower() == "active"}))

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [r[0] for r in self.rows if r[0] is not None]
        smax = [r[1] for r in self.rows if r[1] is not None]
        pw = [r[2] for r in self.rows if r[2] is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(set().union(*(r[3] for r in self.rows))), "samples": len(self.rows),
                "power_w_max": max(pw) if pw else None, "source": self.source}


# ----------------------------------------------------------------------------- CPU baseline (oracle)

_ORACLE_CACHE: dict = {}


def _cached_inputs(shape, b: int):
    """Batch item b's inputs (drawn once per process)."""
    key = ("inputs", shape, b)
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE[key] = make_inputs(shape.replace(decode_steps=0) if shape.decode_steps == 0 else shape,
                                         batches=[b])
    return _ORACLE_CACHE[key]


def _row_runs(N: int, m: int):
    """m positions of [0, N) (m a multiple of min(64, m), m <= N) in runs of up to 64 consecutive
    ones whose centres are spread evenly: the oracle then walks them head-major with the position
    fastest, as it walks a whole slice, so each thread keeps reusing the prefix it just read; the
    mean position is (N - 1) / 2 up to rounding, so a cost linear in the position is estimated
    without bias."""
    import numpy as np
    run = min(64, m)
    nrun = m // run
    starts = ((np.arange(nrun) + 0.5) * (N / nrun) - run / 2).astype(np.int64).clip(0, N - run)
    return (starts[:, None] + np.arange(run)[None, :]).reshape(-1)


def oracle_sample(shape, seconds: float, nthreads: int | None = None, router: str = "saliency"):
    """Time the fp64 oracle on one (batch, KV group) slice of G heads over the whole sequence: the
    score and per-chunk top-k of every token, the NP-Map of every key, and the output rows of m
    positions spread evenly over [0, N) (all G heads each).  A row's cost in the oracle is a constant
    plus a term linear in its position (its linear branch and softmax set are built over its whole
    prefix), so the evenly spread rows scaled by N/m estimate all N rows without a fitted model.  The
    selection and the keys' NP-Map are each timed in full, every step unless one alone takes a
    quarter of the budget (then once per process); the rows call gets the keys' features ready-made,
    its fixed cost (routing masks, output buffer) and its cost per position are calibrated once per
    process, and m is sized from them so that a step takes about `seconds`.  Returns (tokens/s,
    seconds measured, description, threads)."""
    import numpy as np

    import oracle
    oracle.build()
    nth = nthreads or len(os.sched_getaffinity(0))
    N, G = shape.N, shape.G
    inp = _cached_inputs(shape, 0)
    q = np.ascontiguousarray(inp.q[:, :G])
    k, v = inp.k[:, :1], inp.v[:, :1]
    wq, wk = inp.wq[:G], inp.wk[:1]
    sl = shape.replace(B=1, H=G, Hkv=1)
    d = oracle.Dims.of(sl)
    selects = sl.w > 0 and sl.k > 0 and sl.T > 0

    def select():
        t0 = time.perf_counter()
        r = oracle.diagonal_score(d, q, k) if router == "diagonal" else oracle.saliency(d, q, k, nthreads=nth)[1]
        idx = oracle.topk(d, r)
        return idx, time.perf_counter() - t0

    def features():
        t0 = time.perf_counter()
        phik = oracle.npmap(k[0, 0], wk[0])[None, None]
        return phik, time.perf_counter() - t0

    def timed(key, fn):
        """fn() timed this step, or its result and time from an earlier step when it is costly."""
        if key in _ORACLE_CACHE and _ORACLE_CACHE[key][1] > 0.25 * seconds:
            return _ORACLE_CACHE[key][0], _ORACLE_CACHE[key][1], False
        _ORACLE_CACHE[key] = fn()
        return _ORACLE_CACHE[key][0], _ORACLE_CACHE[key][1], True

    def rows_call(idx, phik, m):
        pos = _row_runs(N, m)
        rows = np.array([(0, h, int(p_)) for h in range(G) for p_ in pos], dtype=np.int32)
        t0 = time.perf_counter()
        oracle.prefill(d, q, k, v, wq, None, idx_in=idx, rows=rows, nthreads=nth, phik=phik)
        return time.perf_counter() - t0

    idx, t_sel, sel_now = timed(("selection", shape, router, nth), select) if selects else (None, 0.0, False)
    phik, t_phi, phi_now = timed(("features", shape), features)
    cal_key = ("rows", shape, router, nth)
    if cal_key not in _ORACLE_CACHE:  # once per process: the fixed cost of a call and the cost per position
        t_call = min(rows_call(idx, phik, 1) for _ in range(3))
        m0 = min(N, 64)
        while True:  # grow the calibration sample until its rows outweigh the fixed cost
            t = rows_call(idx, phik, m0)
            if m0 >= N or t - t_call >= max(0.1, t_call):
                break
            m0 = min(N, 2 * m0)
        _ORACLE_CACHE[cal_key] = (t_call, m0, max(t - t_call, 1e-9) / m0)
    t_call, m0, per_pos = _ORACLE_CACHE[cal_key]
    left = seconds - (t_sel if sel_now else 0.0) - (t_phi if phi_now else 0.0) - t_call
    m = int(min(N, max(m0, left / per_pos)))
    m = N if m >= N else max(1, m // min(64, m)) * min(64, m)  # whole runs of 64
    t_rows = rows_call(idx, phik, m)
    t_slice = t_sel + t_phi + t_call + max(t_rows - t_call, 0.0) * N / m
    t_layer = t_slice * shape.B * shape.Hkv
    desc = (f"oracle fp64 on one (batch, KV group) slice of {G} heads and {N} tokens: {router} score + "
            f"top-k of every token ({t_sel:.2f} s), NP-Map of every key ({t_phi:.2f} s), output rows of {m} "
            f"positions in evenly spread runs x {G} heads ({t_rows - t_call:.2f} s, scaled x{N / m:.1f} to all "
            f"positions, plus the call's own {t_call:.2f} s); times {shape.B * shape.Hkv} slices")
    return shape.B * N / t_layer, (t_sel if sel_now else 0.0) + (t_phi if phi_now else 0.0) + t_rows, desc, nth


# ----------------------------------------------------------------------------- main arms

def dist_setup(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def run_reference(args):
    rank, world, _ = dist_setup(args)
    if rank != 0:
        return
    shape = workload_shape(args)
    per_step = max(0.25, 150.0 / max(1, args.steps + args.warmup))
    vals = []
    desc, nth = "", 1
    backward = shape.decode_steps == 0 and getattr(args, "pass_", "forward") == "backward"
    for i in range(args.warmup + args.steps):
        if shape.decode_steps > 0:
            v, t, desc, nth = oracle_decode_sample(shape, per_step)
        elif backward:
            v, t, desc, nth = oracle_backward_sample(shape, per_step)
        else:
            v, t, desc, nth = oracle_sample(shape, per_step, router=getattr(args, "router", "saliency"))
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals) if vals else None
    metric = METRIC_DECODE if shape.decode_steps > 0 else (METRIC_BACKWARD if backward else METRIC)
    config = config_of(shape, args)
    if backward:
        config["pass"] = "backward"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nth, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_shape(args, name=None):
    """The workload's shape with --keep applied (k = C keeps every token of a decided chunk)."""
    shape = WORKLOADS[name or args.workload]
    keep = getattr(args, "keep", "config")
    if keep == "all" and shape.w > 0:
        shape = shape.replace(k=shape.C)
    elif keep == "none":
        shape = shape.replace(k=0)
    elif keep == "window":
        shape = shape.replace(k=0, w=-(-shape.N // shape.C) * shape.C)
    return shape


def config_of(shape, args, name=None):
    return {"workload": name or args.workload, "B": shape.B, "H": shape.H, "Hkv": shape.Hkv, "N": shape.N, "d": shape.d,
            "D": shape.D, "w": shape.w, "C": shape.C, "k": shape.k, "global_batch": shape.B * args.gpus,
            "seq_len": shape.N, "parallelism": f"replicas{args.gpus}", "l2": "flushed before every step",
            "router": getattr(args, "router", "saliency"), "keep": getattr(args, "keep", "config")}


def max_over_ranks(value_ms: float, world: int, device=None) -> float:
    """Max of a per-rank time over all ranks (identity on one rank)."""
    if world <= 1:
        return value_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def pipelined_e2e(steps: int, h2d_fn, compute_fn, d2h_fn, nbuf: int = 2) -> float:
    """Elapsed ms of `steps` end-to-end steps, each with its host->device input copy and its
    device->host output copy inside the timed region, pipelined the way a caller would run it: the
    inputs of step n+1 go up on one copy stream and the output of step n comes down on another while
    step n+1 computes on the current stream, with `nbuf` device buffer sets and events ordering each
    buffer's reuse.  h2d_fn(n, b), compute_fn(n, b) and d2h_fn(n, b) enqueue step n's work on the
    current stream (the caller's callbacks run inside the right stream context); b = n % nbuf."""
    import torch
    main = torch.cuda.current_stream()
    cs, os_ = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_ev = [torch.cuda.Event() for _ in range(nbuf)]
    comp_ev = [torch.cuda.Event() for _ in range(nbuf)]
    d2h_ev = [torch.cuda.Event() for _ in range(nbuf)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(main)
    cs.wait_event(start)
    os_.wait_event(start)

    def issue_h2d(n):
        b = n % nbuf
        with torch.cuda.stream(cs):
            if n >= nbuf:
                cs.wait_event(comp_ev[b])  # step n - nbuf has finished reading buffer set b
            h2d_fn(n, b)
            h2d_ev[b].record(cs)

    issue_h2d(0)
    for n in range(steps):
        b = n % nbuf
        if n + 1 < steps:
            issue_h2d(n + 1)
        main.wait_event(h2d_ev[b])
        if n >= nbuf:
            main.wait_event(d2h_ev[b])  # output buffer b has been copied out
        compute_fn(n, b)
        comp_ev[b].record(main)
        with torch.cuda.stream(os_):
            os_.wait_event(comp_ev[b])
            d2h_fn(n, b)
            d2h_ev[b].record(os_)
    main.wait_stream(os_)
    end.record(main)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def job_throughput(tokens_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


def bench_prefill(args, name, rank, world, local, cpu_seconds):
    """One prefill workload on this rank: the timed steps, the end-to-end steps, the roofline and (rank 0,
    one GPU) the CPU baseline; returns the JSON line as a dict."""
    import numpy as np
    import torch

    from linear_attention_still_b200 import still

    shape = workload_shape(args, name)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    inp = make_inputs(shape.replace(seed=rank), threads=len(os.sched_getaffinity(0)))
    host = {n: to_host_tensor(getattr(inp, n)[:, :, :shape.N] if n in "qkv" else getattr(inp, n), tdt)
            for n in ("q", "k", "v", "wq", "wk")}
    del inp
    devt = {n: t.cuda() for n, t in host.items()}
    o = torch.empty_like(devt["q"])
    dims = still.dims_of(shape)
    ws = torch.empty(still.still_prefill_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    diag = args.router == "diagonal" and shape.w > 0 and shape.k > 0 and shape.T > 0
    if diag:
        r_sel = torch.empty(shape.B, shape.Hkv, shape.N, dtype=torch.float32, device="cuda")
        idx_sel = torch.empty(shape.B, shape.Hkv, shape.T, shape.k, dtype=torch.int32, device="cuda")

    def step(t, out=None):
        out = o if out is None else out
        if diag:  # diagonal-only router: score, per-chunk top-k, then the layer on that selection
            still.still_diagonal_score(dims, t["q"], t["k"], r_sel)
            still.still_select_topk(dims, r_sel, idx_sel)
            still.still_hybrid_prefill(dims, t["q"], t["k"], t["v"], t["wq"], t["wk"], out, idx_in=idx_sel,
                                       workspace=ws)
        else:
            still.still_hybrid_prefill(dims, t["q"], t["k"], t["v"], t["wq"], t["wk"], out, workspace=ws)

    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    free0, total_mem = torch.cuda.mem_get_info()
    for _ in range(args.warmup):
        flush.zero_()
        step(devt)
    torch.cuda.synchronize()
    if still.still_get_device_status() != 0:
        raise RuntimeError("device-side check failed during warm-up")
    # every byte the layer touches is a torch allocation made above (inputs, output, workspace; the
    # library allocates nothing), so the allocator's high-water mark minus the L2-flush buffer is the
    # layer's peak device memory
    peak_layer = torch.cuda.max_memory_allocated() - flush.numel()
    es = 2 if shape.dtype == "bf16" else 4
    memory = {
        "peak_device_bytes": int(peak_layer),
        "workspace_bytes": int(ws.numel()),
        "io_bytes": int(sum(t.numel() * t.element_size() for t in devt.values()) + o.numel() * o.element_size()),
        # dense causal softmax attention of the same layer, for comparison (analytic):
        "dense_flash_bytes": int((2 * shape.B * shape.H + 2 * shape.B * shape.Hkv) * shape.N * shape.d * es
                                 + shape.B * shape.H * shape.N * 4),  # Q, K, V, O + row LSE
        "dense_scores_bytes": int(shape.B * shape.H * shape.N * shape.N * es),  # materialised N x N scores
        "free_before_bytes": int(free0), "total_bytes": int(total_mem),
    }

    gpu_id = None
    try:
        gpu_id = f"GPU-{torch.cuda.get_device_properties(local).uuid}"
    except Exception:
        gpu_id = None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    sampler.start()
    n0 = still.still_launch_count()
    still.still_timing_read()
    still.still_timing_enable(True)
    for s_, e_ in evs:
        flush.zero_()
        s_.record(stream)
        step(devt)
        e_.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    still.still_timing_enable(False)
    launches = still.still_launch_count() - n0
    clocks = sampler.stop()
    kern = still.still_timing_read()
    total_ms = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in evs), world, "cuda")
    ms_per_step = total_ms / args.steps
    tokens = shape.B * shape.N
    value = job_throughput(tokens, args.steps, world, total_ms)

    # end to end through the same call with pinned host buffers: every step copies its inputs up and
    # its output down inside the timed region, pipelined across two buffer sets (pipelined_e2e)
    pinned = {n: t.pin_memory() for n, t in host.items()}
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = o_host.numel() * o_host.element_size()
    dev_sets = [devt, {n: torch.empty_like(t) for n, t in devt.items()}]
    o_sets = [o, torch.empty_like(o)]

    def e2e_h2d(n, b):
        for nm in dev_sets[b]:
            dev_sets[b][nm].copy_(pinned[nm], non_blocking=True)

    def e2e_compute(n, b):
        flush.zero_()
        step(dev_sets[b], o_sets[b])

    def e2e_d2h(n, b):
        o_host.copy_(o_sets[b], non_blocking=True)

    e2e_ms = max_over_ranks(pipelined_e2e(args.e2e_steps, e2e_h2d, e2e_compute, e2e_d2h), world, "cuda")
    e2e_value = job_throughput(tokens, args.e2e_steps, world, e2e_ms)
    del dev_sets, o_sets
    status = still.still_get_device_status()

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    # the merge runs as one kernel (SIMT path) or as two tensor-core phases (window part with the fused
    # saliency, then the kept prefix + linear branch); achieved = algorithmic FLOPs of one step's merge
    # over the summed device time of its launches
    merge_ms = kern["merge"][0] + kern["merge_prefix"][0]
    merge_n = args.steps if merge_ms > 0 else 0
    mflops = nowin_flops(shape) if shape.w == 0 else merge_flops(shape)
    achieved = mflops / (merge_ms / merge_n / 1e3) / 1e12 if merge_n else None
    peak = peaks.get("bf16_tflops", 1590.0) if shape.dtype == "bf16" else None
    roofline = {
        "kernel": "merge (window phase + kept-prefix phase)" if shape.w > 0 else
                  "no-window merge (phi(K) once, intra-chunk tile + phi(q)^T S_t, with the W^T transpose)",
        "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": (achieved / peak) if (achieved and peak) else None,
        "peak_source": "measured bf16_tflops" if "bf16_tflops" in peaks else "fallback 1.59 PFLOP/s",
        "traffic": profiled_traffic(name),
        "traffic_unit": "DRAM bytes per step (both merge launches, ncu)" if shape.w > 0 else
                        "DRAM bytes per step (the three no-window launches, ncu)",
        "flops_per_step": mflops, "ms_per_step": merge_ms / merge_n if merge_n else None,
    }
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic", "config": config_of(shape, args, name),
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipelined": "inputs of step n+1 up and output of step n down on two copy streams, overlapping "
                             "the compute of step n+1"},
        "gpu_launches": launches, "clocks": clocks,
        "kernel_ms_per_step": {k_: v_[0] / args.steps for k_, v_ in kern.items() if v_[1]},
        "layer_tflops": layer_flops(shape) / (ms_per_step / 1e3) / 1e12, "device_status": status,
        "memory": memory,
        "exp_pipe": exp_pipe_diag(shape, roofline["ms_per_step"], clocks,
                                  torch.cuda.get_device_properties(local).multi_processor_count)
        if shape.w > 0 else None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, t, desc, nth = oracle_sample(shape, cpu_seconds, router=args.router)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": nth, "kind": "oracle", "sample": desc}
    del devt, o, ws, flush, host
    return line


# ----------------------------------------------------------------------------- decode workload

def decode_step_bytes(shape, pos: int) -> int:
    """Algorithmic HBM bytes of one decode step at position pos (one token for each of the B
    sequences): per (b, g) the kept rows and the window rows of K and V, S [D,d] and z [D] in fp32;
    per (b, h) q and o."""
    es = 2 if shape.dtype == "bf16" else 4
    m, t = shape.w // shape.C, pos // shape.C
    lo = max(0, (t - m) * shape.C)
    rows = shape.k * max(0, t - m) + (pos - lo + 1)
    per_bg = rows * 2 * shape.d * es + shape.D * shape.d * 4 + shape.D * 4
    return shape.B * shape.Hkv * per_bg + shape.B * shape.H * 2 * shape.d * es


def _causal_pairs(n: int) -> float:
    """(query, key) pairs of n causal rows, keys up to and including the row itself."""
    return n * (n + 1) / 2.0


def oracle_backward_sample(shape, seconds: float):
    """fp64 oracle backward (oracle/backward.py, one process) on the first n tokens of one (batch,
    KV group) slice, n grown once per process until about `seconds` are spent, scaled to the layer by
    the ratio of causal (query, key) pairs n(n+1)/2: the numpy oracle visits every earlier token of
    a row once, in its softmax or its linear set, at about the same cost either way.  Returns
    (tokens/s, seconds, description, threads)."""
    import numpy as np

    from oracle import backward
    import oracle
    oracle.build()
    inp = _cached_inputs(shape, 0)
    q = np.ascontiguousarray(inp.q[:, :shape.G])
    k, v = inp.k[:, :1], inp.v[:, :1]
    wq, wk = inp.wq[:shape.G], inp.wk[:1]
    prepared: dict = _ORACLE_CACHE.setdefault(("backward-sets", shape), {})

    def run(n):
        sl = shape.replace(B=1, H=shape.G, Hkv=1, N=n)
        if n not in prepared:  # the gradient and the forward's selection are inputs, built untimed
            d = oracle.Dims.of(sl)
            do = np.random.default_rng(0).standard_normal(q[:, :, :n].shape)
            idx = oracle.prefill(d, q[:, :, :n], k[:, :, :n], v[:, :, :n], wq, wk)["idx"] \
                if (sl.k > 0 and sl.T > 0) else None
            prepared[n] = (do, idx)
        do, idx = prepared[n]
        t0 = time.perf_counter()
        backward.layer_backward(q[:, :, :n], k[:, :, :n], v[:, :, :n], wq, wk, do, idx, sl.w, sl.C)
        return time.perf_counter() - t0

    key = ("backward", shape, round(seconds, 3))
    if key in _ORACLE_CACHE:
        n = _ORACLE_CACHE[key]
        t_last = run(n)
    else:  # grow the sample while the next one (work ~ softmax pairs) still fits the budget
        n = min(shape.N, max(shape.C, 256))
        t_last = run(n)
        spent = t_last
        while n < shape.N:
            n2 = min(shape.N, n * 2)
            t_next = t_last * _causal_pairs(n2) / _causal_pairs(n)
            if spent + t_next > seconds:
                break
            n = n2
            t_last = run(n)
            spent += t_last
        _ORACLE_CACHE[key] = n
    scale = _causal_pairs(shape.N) / _causal_pairs(n) * shape.B * shape.Hkv
    t_layer = t_last * scale
    desc = (f"oracle backward fp64 (numpy, 1 process) on the first {n} tokens of one (batch, KV group) slice "
            f"of {shape.G} heads ({t_last:.1f} s), scaled to the layer by causal (query, key) pairs "
            f"(x{scale:.0f})")
    return shape.B * shape.N / t_layer, t_last, desc, 1


def oracle_decode_sample(shape, seconds: float):
    """fp64 oracle cost of decode rows: one (batch 0, KV group 0) slice of N + steps tokens, the output
    rows (G heads each) of m decode positions spread evenly over the decode steps, evaluated by the
    same definition as a prefill row.  The slice, its selection and the NP-Map of its keys are set
    up once per process and handed to every call (a decode token maps only its own key); the call's
    remaining fixed cost (routing masks, output buffer) is measured once (the fastest of three
    one-position calls) and taken off, and the cost per position calibrated with it; m is sized to
    the budget (eight at least).  Returns tokens/s of one sequence over all KV groups, seconds
    measured, description, threads."""
    import numpy as np

    import oracle
    oracle.build()
    nth = len(os.sched_getaffinity(0))
    key = ("decode", shape, nth)
    if key not in _ORACLE_CACHE:
        full = shape.replace(B=1, H=shape.G, Hkv=1, N=shape.N + shape.decode_steps, decode_steps=0)
        inp = make_inputs(shape.replace(B=1, H=shape.G, Hkv=1))
        d = oracle.Dims.of(full)
        _, r = oracle.saliency(d, inp.q, inp.k, nthreads=nth)
        phik = oracle.npmap(inp.k[0, 0], inp.wk[0])[None, None]
        _ORACLE_CACHE[key] = [inp, d, oracle.topk(d, r), phik, None]
    inp, d, idx, phik, cal = _ORACLE_CACHE[key]

    def run(m):
        pos = shape.N + (np.arange(m) + 0.5) * (shape.decode_steps / m)
        rows = np.array([(0, h, int(p_)) for h in range(shape.G) for p_ in pos], dtype=np.int32)
        t0 = time.perf_counter()
        oracle.prefill(d, inp.q, inp.k, inp.v, inp.wq, None, idx_in=idx, rows=rows, nthreads=nth, phik=phik)
        return time.perf_counter() - t0

    if cal is None:
        t_fixed = min(run(1) for _ in range(3))
        m0 = 8
        while True:  # grow the calibration sample until its rows outweigh the fixed cost
            t = run(m0)
            if m0 >= shape.decode_steps or t - t_fixed >= max(0.05, 0.5 * t_fixed):
                break
            m0 = min(shape.decode_steps, 2 * m0)
        cal = _ORACLE_CACHE[key][4] = (t_fixed, max(t - t_fixed, 1e-9) / m0)
    t_fixed, per_pos = cal
    m = int(min(shape.decode_steps, max(8, (seconds - t_fixed) / per_pos)))
    t_call = run(m)
    t_rows = max(t_call - t_fixed, 1e-9)
    per_token = t_rows / m * shape.Hkv  # one token of one sequence, every KV group
    desc = (f"oracle fp64: rows of {m} decode positions x {shape.G} heads of one KV group at context "
            f"{shape.N} ({t_rows:.2f} s, after the call's fixed {t_fixed:.2f} s; keys' NP-Map and selection "
            f"prepared once), scaled to all {shape.Hkv} KV groups")
    return 1.0 / per_token, t_call, desc, nth


def bench_decode(args, name, rank, world, local, cpu_seconds, all_steps=False):
    """One decode workload on this rank (prefill of the context, then timed decode steps); returns the
    JSON line as a dict.  all_steps: time every decode step left after the warm-up and end-to-end ones
    (about one chunk cycle: C - 1 ordinary steps and the one that closes a chunk) instead of --steps."""
    import numpy as np
    import torch

    from linear_attention_still_b200 import still
    shape = workload_shape(args, name)
    N, steps, B = shape.N, shape.decode_steps, shape.B
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    e2e_steps = min(args.e2e_steps, 20)
    K = steps - args.warmup - e2e_steps if all_steps else min(args.steps, steps - args.warmup - e2e_steps)
    cap = N + steps
    dims = still.dims_of(shape)
    q = torch.empty(B, shape.H, N, shape.d, dtype=tdt, device="cuda")
    k = torch.empty(B, shape.Hkv, N, shape.d, dtype=tdt, device="cuda")
    v = torch.empty_like(k)
    qd = torch.empty(steps, B, shape.H, shape.d, dtype=tdt)   # decode tokens, host
    kd = torch.empty(steps, B, shape.Hkv, shape.d, dtype=tdt)
    vd = torch.empty_like(kd)
    wq = wk = None
    # a few batch items at a time (drawn concurrently) keeps the host footprint bounded; the prefix
    # goes to the device in fp32 and is converted there
    group = max(1, min(8, len(os.sched_getaffinity(0))))
    for b0 in range(0, B, group):
        bs = list(range(b0, min(B, b0 + group)))
        inp = make_inputs(shape.replace(seed=shape.seed + rank), batches=bs, threads=len(bs))
        for n, b in enumerate(bs):
            for dst, src_ in ((q, inp.q), (k, inp.k), (v, inp.v)):
                dst[b].copy_(torch.from_numpy(np.ascontiguousarray(src_[n, :, :N])).cuda().to(tdt))
            qd[:, b] = torch.from_numpy(np.ascontiguousarray(inp.q[n, :, N:].transpose(1, 0, 2))).to(tdt)
            kd[:, b] = torch.from_numpy(np.ascontiguousarray(inp.k[n, :, N:].transpose(1, 0, 2))).to(tdt)
            vd[:, b] = torch.from_numpy(np.ascontiguousarray(inp.v[n, :, N:].transpose(1, 0, 2))).to(tdt)
        wq, wk = torch.from_numpy(inp.wq).to(tdt).cuda(), torch.from_numpy(inp.wk).to(tdt).cuda()
        del inp
    state = torch.empty(still.still_decode_state_bytes(dims, cap), dtype=torch.uint8, device="cuda")
    still.still_decode_init(dims, cap, state)
    o = torch.empty_like(q)
    ws = torch.empty(still.still_prefill_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    still.still_hybrid_prefill(dims, q, k, v, wq, wk, o, workspace=ws, state=state, state_capacity=cap)
    del ws, o, q, k, v
    torch.cuda.synchronize()
    qdd, kdd, vdd = qd.cuda(), kd.cuda(), vd.cuda()
    o_t = torch.empty(B, shape.H, shape.d, dtype=tdt, device="cuda")
    stream = torch.cuda.current_stream()
    pos = N
    for _ in range(args.warmup):
        still.still_decode_step(dims, state, cap, pos, wq, wk, qdd[pos - N], kdd[pos - N], vdd[pos - N], o_t)
        pos += 1
    torch.cuda.synchronize()
    if still.still_get_device_status() != 0:
        raise RuntimeError("device-side check failed during warm-up")
    # end to end: each step's token goes up from pinned host memory and its output comes down inside
    # the timed region, pipelined across two buffer sets (pipelined_e2e)
    pins = [t_.pin_memory() for t_ in (qd, kd, vd)]
    o_host = torch.empty(o_t.shape, dtype=tdt).pin_memory()
    tok_sets = [[torch.empty_like(t_[0], device="cuda") for t_ in (qd, kd, vd)] for _ in range(2)]
    ot_sets = [o_t, torch.empty_like(o_t)]
    pos0 = pos

    def e2e_h2d(n, b):
        for x_, src_ in zip(tok_sets[b], pins):
            x_.copy_(src_[pos0 + n - N], non_blocking=True)

    def e2e_compute(n, b):
        still.still_decode_step(dims, state, cap, pos0 + n, wq, wk, *tok_sets[b], ot_sets[b])

    def e2e_d2h(n, b):
        o_host.copy_(ot_sets[b], non_blocking=True)

    e2e_ms = max_over_ranks(pipelined_e2e(e2e_steps, e2e_h2d, e2e_compute, e2e_d2h), world, "cuda")
    pos += e2e_steps
    qb, kb, vb = tok_sets[0]
    # untimed steps up to the timed region, which ends at the last position: it holds the step that
    # closes a chunk (position C-1 mod C) along with ordinary ones
    # the last (up to 64) of them also give the per-kernel breakdown, with events around each launch
    n_brk = min(64, cap - K - pos)
    still.still_timing_read()
    while pos < cap - K:
        if pos == cap - K - n_brk:
            still.still_timing_enable(True)
        still.still_decode_step(dims, state, cap, pos, wq, wk, qdd[pos - N], kdd[pos - N], vdd[pos - N], o_t)
        pos += 1
    torch.cuda.synchronize()
    still.still_timing_enable(False)
    brk = still.still_timing_read()
    kernel_ms = {k_: v_[0] / n_brk for k_, v_ in brk.items() if v_[1]} if n_brk > 0 else {}
    gpu_id = None
    try:
        gpu_id = f"GPU-{torch.cuda.get_device_properties(local).uuid}"
    except Exception:
        pass
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    sampler.start()
    n0 = still.still_launch_count()
    first = pos
    for s_, e_ in evs:
        s_.record(stream)
        still.still_decode_step(dims, state, cap, pos, wq, wk, qdd[pos - N], kdd[pos - N], vdd[pos - N], o_t)
        e_.record(stream)
        pos += 1
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    launches = still.still_launch_count() - n0
    times = [s_.elapsed_time(e_) for s_, e_ in evs]
    total_ms = max_over_ranks(sum(times), world, "cuda")
    ms_per_step = total_ms / K
    value = job_throughput(B, K, world, total_ms)
    nbytes = sum(decode_step_bytes(shape, p_) for p_ in range(first, first + K))
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    peak = peaks.get("hbm_gbs", 6650.0)
    achieved = nbytes / (sum(times) / 1e3) / 1e9
    close_steps = [j for j, p_ in enumerate(range(first, first + K)) if p_ % shape.C == shape.C - 1]
    status = still.still_get_device_status()
    line = {
        "metric": METRIC_DECODE,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": shape.dtype, "data": "synthetic",
        "config": dict(config_of(shape, args, name), decode_steps_timed=K, first_position=first,
                       chunk_close_steps_timed=len(close_steps),
                       l2="decode state (kept cache + window) larger than L2"),
        "roofline": {"kernel": "decode step (all kernels)", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": None,
                     "bytes_per_step": nbytes / K,
                     "peak_source": "measured hbm_gbs" if "hbm_gbs" in peaks else "fallback 6.65 TB/s"},
        "e2e": {"value": job_throughput(B, e2e_steps, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": (qb.numel() + kb.numel() + vb.numel()) * qb.element_size(),
                "d2h_bytes_per_step": o_host.numel() * o_host.element_size(),
                "pipelined": "token of step n+1 up and output of step n down on two copy streams, "
                             "overlapping the compute of step n+1"},
        "gpu_launches": launches, "clocks": clocks,
        "kernel_ms_per_step": kernel_ms, "kernel_ms_steps": n_brk,
        "step_ms": {"median": float(np.median(times)), "max": float(max(times)),
                    "chunk_close": [times[j] for j in close_steps],
                    # one chunk's worth of steps: C-1 ordinary steps and the one that closes the chunk
                    "chunk_cycle_mean": (float(np.median([t_ for j, t_ in enumerate(times) if j not in close_steps]))
                                         * (shape.C - 1) + max([times[j] for j in close_steps], default=0.0))
                    / shape.C if close_steps else None},
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_, t_, desc, nth = oracle_decode_sample(shape, cpu_seconds)
        line["cpu_baseline"] = {"value": v_, "unit": "tokens/s", "cores": nth, "kind": "oracle", "sample": desc}
    del state, qdd, kdd, vdd, o_t, qb, kb, vb, wq, wk
    return line


def backward_flops(shape):
    """Algorithmic FLOPs of the backward pass: per (query-head, softmax key) the forward recompute
    (QK^T, PV: 4d) and the backward (QK^T again, dO.V, dq, dk, dv: 10d); per query-head the NP-Map
    and linear-state products (about 12 d D); per unselected key of a decided chunk 8 d D."""
    rows = shape.B * shape.H
    return rows * (14 * shape.d * int(soft_sizes(shape).sum()) + shape.N * 12 * shape.d * shape.D) + \
        shape.B * shape.Hkv * shape.N * 8 * shape.d * shape.D


def bench_backward(args, name, rank, world, local, cpu_seconds):
    """The backward pass of one prefill workload on this rank; returns the JSON line as a dict."""
    import numpy as np
    import torch

    from linear_attention_still_b200 import still
    shape = workload_shape(args, name)
    tdt = torch.bfloat16 if shape.dtype == "bf16" else torch.float32
    inp = make_inputs(shape.replace(seed=rank))
    host = {n: torch.from_numpy(np.ascontiguousarray(getattr(inp, n))).to(tdt) for n in ("q", "k", "v", "wq", "wk")}
    host["do"] = torch.from_numpy(np.random.default_rng(rank).standard_normal(inp.q.shape).astype(np.float32)).to(tdt)
    del inp
    devt = {n: t.cuda() for n, t in host.items()}
    dims = still.dims_of(shape)
    # the selection the forward makes, held fixed by the backward
    ws_f = torch.empty(still.still_prefill_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(devt["q"])
    still.still_hybrid_prefill(dims, devt["q"], devt["k"], devt["v"], devt["wq"], devt["wk"], o, workspace=ws_f)
    idx = None
    lay = still.still_prefill_workspace_layout(dims)
    if shape.k > 0 and shape.T > 0:
        off = lay["idx"]
        n_idx = shape.B * shape.Hkv * shape.T * shape.k
        idx = ws_f[off:off + 4 * n_idx].view(torch.int32).clone()
    saved = args.bwd_stats == "saved"
    if saved:
        # what a training step's forward leaves for the backward: its output and every row's normaliser
        n_rows = shape.B * shape.H * shape.N
        host["o"] = o.cpu()
        host["lse"] = ws_f[lay["lse"]:lay["lse"] + 4 * n_rows].view(torch.float32).cpu().clone()
        devt["o"], devt["lse"] = o, host["lse"].cuda()
    del ws_f, o
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = [torch.empty(shape.B, shape.H, shape.N, shape.d, **f32),
             torch.empty(shape.B, shape.Hkv, shape.N, shape.d, **f32),
             torch.empty(shape.B, shape.Hkv, shape.N, shape.d, **f32),
             torch.empty(shape.H, shape.d, shape.D, **f32), torch.empty(shape.Hkv, shape.d, shape.D, **f32)]
    ws = torch.empty(still.still_backward_workspace_bytes(dims), dtype=torch.uint8, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(t):
        if saved:
            still.still_hybrid_backward_saved(dims, t["q"], t["k"], t["v"], t["wq"], t["wk"], idx, t["do"], t["o"],
                                              t["lse"], *grads, workspace=ws)
        else:
            still.still_hybrid_backward(dims, t["q"], t["k"], t["v"], t["wq"], t["wk"], idx, t["do"], *grads,
                                        workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step(devt)
    torch.cuda.synchronize()
    if still.still_get_device_status() != 0:
        raise RuntimeError("device-side check failed during warm-up")
    gpu_id = None
    try:
        gpu_id = f"GPU-{torch.cuda.get_device_properties(local).uuid}"
    except Exception:
        pass
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_id)
    sampler.start()
    n0 = still.still_launch_count()
    for s_, e_ in evs:
        flush.zero_()
        s_.record(stream)
        step(devt)
        e_.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    launches = still.still_launch_count() - n0
    total_ms = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in evs), world, "cuda")
    ms_per_step = total_ms / args.steps
    tokens = shape.B * shape.N
    # end to end: inputs and dO from pinned host memory, the five gradients back to the host
    pinned = {n: t.pin_memory() for n, t in host.items()}
    outs = [torch.empty(g_.shape, dtype=g_.dtype).pin_memory() for g_ in grads]
    e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.e2e_steps)]
    for s_, e_ in e_evs:
        flush.zero_()
        s_.record(stream)
        for n in devt:
            devt[n].copy_(pinned[n], non_blocking=True)
        step(devt)
        for h_, g_ in zip(outs, grads):
            h_.copy_(g_, non_blocking=True)
        e_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in e_evs), world, "cuda")
    # per-kernel breakdown: two more steps with events around the launches (outside the timed region)
    still.still_timing_read()
    still.still_timing_enable(True)
    for _ in range(2):
        flush.zero_()
        step(devt)
    torch.cuda.synchronize()
    still.still_timing_enable(False)
    kernel_ms = {k_: v_[0] / 2 for k_, v_ in still.still_timing_read().items() if v_[1]}
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except OSError:
        pass
    pairs = int(soft_sizes(shape).sum()) * shape.B * shape.H
    if "bwd_dq" in kernel_ms:
        # tensor-core path: the dominant kernel is the dq kernel; its algorithmic work is S = Q K^T,
        # dP = dO V^T and dQ += dS K (6 d FLOP per query-head and softmax key; with --bwd-stats recompute
        # the statistics sweep that forms S and dP a first time is not counted)
        peak = peaks.get("bf16_tflops", 1590.0)
        dq_flops = 6 * shape.d * pairs
        roof = {"kernel": "bwd_dq_tc_kernel (dq of the softmax branch)", "bound": "tensor",
                "achieved": dq_flops / (kernel_ms["bwd_dq"] / 1e3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                "traffic": profiled_traffic(name, prefix="bwd_"),
                "flops_per_launch": dq_flops,
                "peak_source": "measured bf16_tflops (burst)" if "bf16_tflops" in peaks else "fallback 1.59 PFLOP/s",
                "key_kernel": {"kernel": "bwd_dkv_tc_kernel (window and kept keys)", "ms": kernel_ms.get("bwd_dkv"),
                               "flops": 8 * shape.d * pairs,
                               "achieved": 8 * shape.d * pairs / (kernel_ms["bwd_dkv"] / 1e3) / 1e12
                               if kernel_ms.get("bwd_dkv") else None},
                "whole_pass": {"flops_per_step": backward_flops(shape),
                               "achieved": backward_flops(shape) / (ms_per_step / 1e3) / 1e12}}
        roof["frac"] = roof["achieved"] / peak
    else:
        # SIMT fp32 kernels: the ALU roofline is the FFMA rate, 148 SMs x 128 lanes x 2 FLOP x 1965 MHz
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        achieved = backward_flops(shape) / (ms_per_step / 1e3) / 1e12
        roof = {"kernel": "backward pass (all kernels)", "bound": "alu", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x 1965 MHz (SIMT kernels)",
                "flops_per_step": backward_flops(shape)}
    line = {
        "metric": METRIC_BACKWARD,
        "value": job_throughput(tokens, args.steps, world, total_ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": shape.dtype, "data": "synthetic",
        "config": dict(config_of(shape, args, name), **{"pass": "backward", "stats": args.bwd_stats}),
        "roofline": roof,
        "kernel_ms_per_step": kernel_ms,
        "e2e": {"value": job_throughput(tokens, args.e2e_steps, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in pinned.values()),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in outs)},
        "gpu_launches": launches, "clocks": clocks, "device_status": still.still_get_device_status(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_, t_, desc, nth = oracle_backward_sample(shape, cpu_seconds)
        line["cpu_baseline"] = {"value": v_, "unit": "tokens/s", "cores": nth, "kind": "oracle", "sample": desc}
    return line


# the other layer configurations a default single-GPU run also reports (under `workloads`)
EXTRA_WORKLOADS = ("llama31_8b_layer_b4_n16k", "llama31_8b_layer_n64k", "llama31_8b_decode_b16_ctx64k")
EXTRA_CPU_SECONDS = 8.0


def to_host_tensor(a, tdt):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(tdt)


def bench_one(args, name, rank, world, local, cpu_seconds, extra=False):
    if WORKLOADS[name].decode_steps > 0:
        return bench_decode(args, name, rank, world, local, cpu_seconds, all_steps=extra)
    if args.pass_ == "backward":
        return bench_backward(args, name, rank, world, local, cpu_seconds)
    return bench_prefill(args, name, rank, world, local, cpu_seconds)


def run_ours(args):
    import torch

    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    line = bench_one(args, args.workload, rank, world, local, args.cpu_seconds)
    extras = args.workloads == "auto" and world == 1 and not args.workload_given and args.pass_ == "forward" \
        and args.router == "saliency" and args.keep == "config"
    if extras:
        line["workloads"] = {}
        for name in EXTRA_WORKLOADS:
            torch.cuda.empty_cache()
            line["workloads"][name] = bench_one(args, name, rank, world, local, EXTRA_CPU_SECONDS, extra=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
