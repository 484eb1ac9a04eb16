#!/usr/bin/env python
"""Benchmark of the tiled MonarchRT attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one forward pass (aggregated queries, R-step, L-step with the
output) of the 720p Wan-shaped clip: B=1, H=12, d=128, f=21, h=45, w=80
(N=75600 tokens), blocks (945, 80), 4 tiles, 1 iteration, bfloat16.  Inputs are
seeded synthetic video tokens (positional code plus planted semantic pairs).
With N > 1 (torchrun, one process per GPU) every rank runs its own clip (weak
scaling, no data-path collective); the device time is the max over ranks.

Prints ONE JSON line (rank 0).  `value` is dense-equivalent effective TFLOP/s
(4*B*H*N^2*d per step over the device time, summed over ranks); `roofline`
describes the dominant kernel, `path_roofline` the whole step against
max(Monarch FLOPs / bf16 peak, Q/K/V/O bytes / HBM bandwidth).
`also_480p` adds the device time of the 480p full clip (B=1 H=12 N=32760, blocks
(630,52), 1 tile) at N=1, beside the line (not a bench line of its own).
`--impl reference` times the float64 CPU oracle instead, on bounded samples.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from structured_attention_video_b200 import synth  # noqa: E402

METRIC = "Monarch-attn fwd ms & effective TFLOP/s at 720p Wan shape; % of roofline"
UNIT = "TFLOP/s (dense-equivalent effective)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(wl: synth.Workload, world: int, shard: bool = False) -> dict:
    par = ("units x%d (one clip's (head, tile) units split across GPUs, disjoint output rows)"
           % world if shard else "replicas x%d (independent clips per GPU)" % world)
    return {"workload": "%s Wan clip: B=%d H=%d d=%d f=%d h=%d w=%d (N=%d), blocks (%d,%d), "
                        "tiles=%d, iters=%d" % (wl.name, wl.B, wl.H, wl.d, wl.f, wl.h, wl.w,
                                                wl.N, wl.b1, wl.b2, wl.tiles, wl.iters),
            "B": wl.B, "H": wl.H, "d": wl.d, "f": wl.f, "h": wl.h, "w": wl.w, "N": wl.N,
            "b1": wl.b1, "b2": wl.b2, "tiles": wl.tiles, "iters": wl.iters,
            "parallelism": par,
            "l2": "inputs (%.2f GB) larger than L2, and a %d MB buffer written between "
                  "timed steps" % (3 * wl.B * wl.H * wl.N * wl.d * 2 / 1e9, L2_FLUSH_BYTES >> 20)}


# ---------------------------------------------------------------------------
# CPU oracle samples (baseline and reference arm)
# ---------------------------------------------------------------------------
def sample_dense_flops(wl: synth.Workload, probs) -> float:
    """Share of the dense-equivalent work that the sampled problems' output rows carry."""
    rows = sum(((g + 1) * wl.b1) // wl.tiles - (g * wl.b1) // wl.tiles for _, g, _ in probs)
    return 4.0 * rows * wl.N * wl.d


class OracleSampler:
    """Runs the float64 oracle on (head, tile, column) problems of one workload."""

    def __init__(self, wl: synth.Workload, heads: int = 2):
        from oracle import oracle
        self.oracle = oracle
        self.wl = wl
        pos = synth.positional_code(wl.f, wl.h, wl.w, wl.d)
        self.heads = list(range(min(heads, wl.B * wl.H)))
        xs = [synth.make_head(wl, bh // wl.H, bh % wl.H, 0, pos) for bh in self.heads]
        self.q = np.stack([x["q"] for x in xs])
        self.k = np.stack([x["k"] for x in xs])
        self.v = np.stack([x["v"] for x in xs])
        self.cores = len(os.sched_getaffinity(0))

    def problems(self, count: int, seed: int):
        rng = np.random.default_rng(seed)
        return [(int(rng.integers(len(self.heads))), int(rng.integers(self.wl.tiles)),
                 int(rng.integers(self.wl.b2))) for _ in range(count)]

    def run(self, probs):
        """Seconds taken, and the oracle's output [heads, N, d] (only the problems' rows)."""
        wl = self.wl
        t0 = time.perf_counter()
        y = self.oracle.monarch_problems(self.q, self.k, self.v, wl.b1, wl.b2, wl.tiles,
                                         wl.iters, probs, nthreads=self.cores)
        return time.perf_counter() - t0, y


def problem_rows(wl: synth.Workload, g: int, c: int) -> np.ndarray:
    """Token rows (u, c), u in tile g, that one (tile, column) problem writes."""
    return np.arange((g * wl.b1) // wl.tiles, ((g + 1) * wl.b1) // wl.tiles) * wl.b2 + c


def sampled_rel_err(wl: synth.Workload, probs, y_ref, rows_of_head) -> dict:
    """Relative Frobenius error of the device output on the sampled problems' rows.

    rows_of_head(bh, rows) returns the device output rows of head bh as float64."""
    got, ref = [], []
    for bh, g, c in probs:
        rows = problem_rows(wl, g, c)
        got.append(rows_of_head(bh, rows))
        ref.append(y_ref[bh][rows])
    got, ref = np.concatenate(got), np.concatenate(ref)
    return {"value": float(np.linalg.norm(got - ref) / np.linalg.norm(ref)),
            "rows": int(got.shape[0]), "vs": "float64 oracle, same seeded inputs",
            "tolerance": 1e-2 if wl.dtype == "bf16" else 1e-5}


def cpu_baseline(wl: synth.Workload, target_s: float, rows_of_head=None) -> dict:
    """Times the oracle on a bounded sample; with rows_of_head (the device output of
    the same inputs) it also reports the device's error on that sample."""
    smp = OracleSampler(wl)
    probe = smp.problems(smp.cores, seed=1)
    t, _ = smp.run(probe)
    count = max(smp.cores, int(smp.cores * max(1.0, target_s / max(t, 1e-3))))
    count = min(count, 4096)
    probs = smp.problems(count, seed=2)
    t, y = smp.run(probs)
    value = sample_dense_flops(wl, probs) / t / 1e12
    rec = {"value": value, "unit": UNIT, "cores": smp.cores, "kind": "oracle",
           "seconds": t,
           "sample": "%d (head, tile, column) problems of the %s workload (%.2f%% of one "
                     "step's output rows), float64 C oracle with OpenMP" %
                     (count, wl.name, 100.0 * sample_dense_flops(wl, probs) / wl.dense_flops())}
    if rows_of_head is not None:
        rec["rel_err"] = sampled_rel_err(wl, probs, y, rows_of_head)
    return rec


def run_reference(args, wl: synth.Workload, world: int, rank: int):
    if rank != 0:
        return
    smp = OracleSampler(wl)
    per_step = smp.cores
    times, flops = [], []
    for step in range(args.warmup + args.steps):
        probs = smp.problems(per_step, seed=100 + step)
        t, _ = smp.run(probs)
        if step >= args.warmup:
            times.append(t)
            flops.append(sample_dense_flops(wl, probs))
    value = sum(flops) / sum(times) / 1e12
    sample = ("each step: %d (head, tile, column) problems of the %s workload (%.3f%% of its "
              "output rows), float64 C oracle with OpenMP on %d cores" %
              (per_step, wl.name, 100.0 * flops[0] / wl.dense_flops(), smp.cores))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": smp.cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.file.seek(0)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        self.file.close()
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# kernel roofline bookkeeping
# ---------------------------------------------------------------------------
def kernel_roofline(name: str, ms_per_launch: float, wl: synth.Workload, peaks, peak_kind):
    """Algorithmic work of one launch of kernel family `name` and its roofline fraction."""
    BH, N, d, t = wl.B * wl.H, wl.N, wl.d, wl.tiles
    es = 2 if wl.dtype == "bf16" else 4
    if name.endswith("rstep_kernel"):
        flops = 6.0 * t * N * wl.b2 * d * BH
    elif name.endswith("lstep_kernel"):
        flops = 4.0 * N * wl.b1 * d * BH
    elif name == "tc_lstat_kernel":       # logits only (no products with Z)
        flops = 2.0 * N * wl.b1 * d * BH
    elif name in ("qbar_weighted_kernel", "tc_qagg_kernel"):
        flops = 4.0 * N * wl.b1 * d * BH
    else:
        flops = None
    tensor = name.startswith("tc_")
    if flops is None:   # query aggregation: reads Q once
        nbytes = BH * N * d * es
        achieved = nbytes / (ms_per_launch * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": peak_kind + " hbm_gbs"}
    achieved = flops / (ms_per_launch * 1e-3) / 1e12
    if tensor:
        # the timed region is tens of milliseconds, short enough to run at boost
        # clocks: the burst GEMM figure is the peak.  The sustained figure (a
        # seconds-long GEMM under the power cap) is reported beside it, and
        # clock_scaled() adds the fraction at the clock the run actually saw.
        peak = peaks["bf16_tflops"]
        out = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
               "frac": achieved / peak, "peak_source": peak_kind + " bf16_tflops (burst)"}
        if "bf16_tflops_sustained" in peaks:
            out["frac_of_sustained"] = achieved / peaks["bf16_tflops_sustained"]
        return out
    # SIMT float32 FMA: 148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock
    peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "peak_source": "derived: 148 SMs x 128 FP32 FMA lanes x 2 x %s sm_max_mhz" % peak_kind}


def clock_scaled(roof: dict, clocks: dict, peaks) -> dict:
    """Adds the fraction of the peak scaled to the run's median SM clock.

    The burst peak was measured at the maximum SM clock; a run whose median
    clock sat lower (power cap) could at most reach peak * median / max."""
    mhz, mhz_max = clocks.get("sm_mhz"), peaks.get("sm_max_mhz")
    if roof.get("bound") == "tensor" and mhz and mhz_max:
        scale = min(1.0, mhz / mhz_max)
        roof["frac_at_run_clock"] = roof["achieved"] / (roof["peak"] * scale)
        roof["run_clock_mhz"] = mhz
        roof["peak_clock_mhz"] = mhz_max
    return roof


def step_stats(times_ms) -> dict:
    """Median and 10th/90th percentiles of the per-step device times."""
    xs = sorted(times_ms)
    if not xs:
        return {}

    def pct(p):
        return float(np.percentile(np.asarray(xs), p))
    return {"median": pct(50), "p10": pct(10), "p90": pct(90), "min": xs[0], "max": xs[-1]}


def kernel_traffic(name: str):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh).get(name)
    if not rec:
        return None
    # the kernel's sources (its .cu and the headers it inlines), hashed in order
    h = hashlib.sha256()
    for name_ in rec["sources"]:
        src = os.path.join(ROOT, "structured_attention_video_b200", "csrc", name_)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    return rec["dram_bytes_per_launch"] if h.hexdigest() == rec["sources_sha256"] else None


# ---------------------------------------------------------------------------
# ranks (one process per GPU; every rank runs its own clip, no data-path collective)
# ---------------------------------------------------------------------------
def rank_barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: every rank must call this, in the same order."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def unit_partition(total_units: int, world: int, rank: int):
    """Rank's contiguous, balanced share [begin, end) of one clip's (head, tile) units."""
    return (total_units * rank) // world, (total_units * (rank + 1)) // world


def unit_rows(wl: synth.Workload, unit: int):
    """(head, token rows) that one (head, tile) unit writes: rows (u, v), u in tile g."""
    bh, g = divmod(unit, wl.tiles)
    u = np.arange((g * wl.b1) // wl.tiles, ((g + 1) * wl.b1) // wl.tiles)
    return bh, (u[:, None] * wl.b2 + np.arange(wl.b2)[None, :]).ravel()


def job_throughput(world: int, dense_flops_per_clip: float, ms_step: float) -> float:
    """Whole-job dense-equivalent TFLOP/s: every rank processed one clip per step."""
    return world * dense_flops_per_clip / (ms_step * 1e-3) / 1e12


def secondary_workload(wl: synth.Workload, steps: int, warmup: int, flush, stream) -> dict:
    """Device time of one more Wan-shaped clip (480p), reported beside the bench line.

    Same timing rules as the main measurement (CUDA events on the launch stream,
    L2 flushed between steps); runs on one GPU only and never fails the bench."""
    import torch
    from structured_attention_video_b200 import _lib
    try:
        dev = flush.device
        shape = (wl.B, wl.H, wl.N, wl.d)
        hq, hk, hv = (torch.empty(shape, dtype=torch.int16) for _ in range(3))
        synth.fill_device_bits(wl, hq.numpy().view(np.uint16), hk.numpy().view(np.uint16),
                               hv.numpy().view(np.uint16), 0)
        q, k, v = (x.to(dev).view(torch.bfloat16) for x in (hq, hk, hv))
        out = torch.empty_like(q)
        sargs = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
        ws_bytes = _lib.monarch_attn_workspace_bytes(*sargs, _lib.BF16)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        sh = stream.cuda_stream

        def step():
            _lib.check(_lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                out.data_ptr(), *sargs, _lib.BF16, ws.data_ptr(),
                                                ws_bytes, sh), "monarch_attn_fwd_ws")

        for _ in range(warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            torch.cuda.synchronize()
            total += a.elapsed_time(b)
        _lib.check(_lib.monarch_last_device_status(sh), "device status (secondary workload)")
        ms = total / steps
        return {"workload": workload_config(wl, 1)["workload"], "ms_per_step": ms,
                "value": job_throughput(1, wl.dense_flops(), ms), "unit": UNIT,
                "monarch_tflops": wl.monarch_flops() / (ms * 1e-3) / 1e12,
                "kernel_path": "sm100 tensor-core" if _lib.monarch_attn_path(*sargs, _lib.BF16) == 1
                else "generic SIMT", "steps": steps, "warmup": warmup}
    except Exception as exc:   # reported, never fatal to the bench line
        return {"workload": wl.name, "error": str(exc)}


# ---------------------------------------------------------------------------
# error-vs-cost sweeps (tiles on the 480p clip, iterations on the Wan-14B shape)
# ---------------------------------------------------------------------------
def dense_rows_error(wl: synth.Workload, q, k, v, out, heads, rows_per_head: int, seed: int):
    """Relative Frobenius error of the device output against exact softmax attention,
    softmax(Q K^T / sqrt(d)) V in float64 on the host from the same (rounded) inputs,
    on `rows_per_head` seeded query rows of each listed head (rows are independent,
    so exact attention on a row subset is exact for those rows)."""
    import torch
    rng = np.random.default_rng(seed)
    num = den = 0.0

    def f64(t):
        return synth.from_device_bits(t.contiguous().view(torch.int16).cpu().numpy()
                                      .view(np.uint16), "bf16")
    for bh in heads:
        b, h = divmod(bh, wl.H)
        rows = np.sort(rng.choice(wl.N, rows_per_head, replace=False))
        idx = torch.as_tensor(rows, device=q.device)
        qr, kk, vv, o = f64(q[b, h, idx]), f64(k[b, h]), f64(v[b, h]), f64(out[b, h, idx])
        s = qr @ kk.T / np.sqrt(wl.d)
        s -= s.max(axis=1, keepdims=True)
        pr = np.exp(s)
        y = (pr / pr.sum(axis=1, keepdims=True)) @ vv
        num += float(((o - y) ** 2).sum())
        den += float((y ** 2).sum())
    return float(np.sqrt(num / den))


def time_forward(wl: synth.Workload, q, k, v, out, steps: int, warmup: int, flush, stream,
                 axis: int = 0):
    """Per-step device times (ms) of monarch_attn_fwd_tiled_ws on resident inputs, with
    the tiles on the query rows (axis 0, monarch_attn_fwd_ws's reading) or the key
    columns (axis 1)."""
    import torch
    from structured_attention_video_b200 import _lib
    sargs = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
    ws_bytes = _lib.monarch_attn_tiled_workspace_bytes(*sargs, _lib.BF16, axis)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    sh = stream.cuda_stream

    def step():
        _lib.check(_lib.monarch_attn_fwd_tiled_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  out.data_ptr(), *sargs, _lib.BF16, axis,
                                                  _lib.BHND, ws.data_ptr(), ws_bytes, sh),
                   "monarch_attn_fwd_tiled_ws")
    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    _lib.check(_lib.monarch_last_device_status(sh), "device status (sweep)")
    return times, _lib.monarch_attn_tiled_path(*sargs, _lib.BF16, axis)


def run_backward(args, wl: synth.Workload) -> None:
    """One JSON line: device ms of the backward pass of one iteration
    (monarch_attn_bwd_ws on resident bfloat16 inputs and upstream gradient), its
    algorithmic FLOPs against the roofline of the kernels that ran (the measured
    bfloat16 tensor peak for the tensor-core backward, the float32 SIMT peak for
    the generic kernels), and the per-family split.  Parity is checked by the GPU
    tests, not here."""
    import torch
    from structured_attention_video_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks, peak_kind = load_peaks()
    shape = (wl.B, wl.H, wl.N, wl.d)
    hq, hk, hv = (torch.empty(shape, dtype=torch.int16) for _ in range(3))
    synth.fill_device_bits(wl, hq.numpy().view(np.uint16), hk.numpy().view(np.uint16),
                           hv.numpy().view(np.uint16), 0)
    q, k, v = (x.to(dev).view(torch.bfloat16) for x in (hq, hk, hv))
    dy = torch.randn(shape, generator=torch.Generator().manual_seed(3)).to(dev, torch.bfloat16)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    sargs = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, 1)
    nb = _lib.monarch_attn_bwd_workspace_bytes(*sargs, _lib.BF16)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)

    def step():
        _lib.check(_lib.monarch_attn_bwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            dy.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                            dv.data_ptr(), *sargs, _lib.BF16, ws.data_ptr(), nb,
                                            sh), "monarch_attn_bwd_ws")
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    _lib.monarch_profile_enable(1)
    _lib.monarch_profile_collect()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    _lib.monarch_profile_enable(0)
    prof = _lib.monarch_profile_collect()
    _lib.check(_lib.monarch_last_device_status(sh), "device status (backward)")
    kernels = {name: ms_tot / max(1, args.steps) for name, (ms_tot, cnt) in prof.items() if cnt > 0}
    ms = float(np.median(times))
    flops = wl.backward_flops()
    achieved = flops / (ms * 1e-3) / 1e12
    simt_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    tensor = _lib.monarch_attn_path(*sargs, _lib.BF16) == 1
    if tensor:
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "peak_source": "%s bf16_tflops (burst)" % peak_kind}
    else:
        roof = {"bound": "alu", "achieved": achieved, "peak": simt_peak, "unit": "TFLOP/s",
                "frac": achieved / simt_peak,
                "peak_source": "derived: 148 SMs x 128 FP32 FMA lanes x 2 x %s sm_max_mhz"
                               % peak_kind}
    print(json.dumps({
        "metric": "Monarch-attn backward ms (one iteration)", "value": ms, "unit": "ms",
        "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
        "ms_stats": step_stats(times), "dtype": "bf16", "data": "synthetic",
        "config": workload_config(wl, 1),
        "backward_gflop": flops / 1e9,
        "roofline": roof,
        "kernel_path": "sm100 tensor-core" if tensor else "generic SIMT",
        "kernels_ms_per_step": kernels, "workspace_bytes": nb,
        "gpu": torch.cuda.get_device_name(0)}), flush=True)


def keytile_cpu_baseline(wl: synth.Workload, got_bits: np.ndarray, samples: int) -> dict:
    """The float64 oracle of key-column tiles on `samples` seeded (head, column)
    problems, all query rows of each, on the host's cores: its time scaled to a
    whole step (B*H*b2 problems), and the rel-Frobenius error of the device output
    (`got_bits`, bfloat16 storage [B][H][N][d]) on those rows."""
    from oracle import oracle
    rng = np.random.default_rng(5)
    probs = sorted({(int(rng.integers(wl.B * wl.H)), int(rng.integers(wl.b2)))
                    for _ in range(samples)})
    pos = synth.positional_code(wl.f, wl.h, wl.w, wl.d)
    num = den = 0.0
    secs = 0.0
    for bh in sorted({pr[0] for pr in probs}):
        b, h = divmod(bh, wl.H)
        x = synth.make_head(wl, b, h, 0, pos)
        cols = [c for (hh, c) in probs if hh == bh]
        t0 = time.perf_counter()
        y = oracle.monarch_attn_keytiles(x["q"][None], x["k"][None], x["v"][None], wl.b1, wl.b2,
                                         wl.tiles, wl.iters, probs=[(0, c) for c in cols])[0]
        secs += time.perf_counter() - t0
        for c in cols:
            rows = np.arange(wl.b1) * wl.b2 + c
            o = synth.from_device_bits(got_bits[b, h, rows], "bf16")
            num += float(((o - y[rows]) ** 2).sum())
            den += float((y[rows] ** 2).sum())
    total = wl.B * wl.H * wl.b2
    return {"value": secs * 1e3 * total / len(probs), "unit": "ms", "cores": oracle.max_threads(),
            "kind": "oracle", "seconds": secs,
            "sample": "%d (head, column) problems of the workload (%.2f%% of one step's output "
                      "rows), float64 C oracle with OpenMP, scaled to a whole step"
                      % (len(probs), 100.0 * len(probs) / total),
            "rel_err": {"value": float(np.sqrt(num / den)), "rows": len(probs) * wl.b1,
                        "vs": "float64 oracle, same seeded inputs", "tolerance": 0.01}}


def run_keytiles(args, wl: synth.Workload) -> None:
    """One JSON line: device ms of the forward pass with key-column tiles (the
    key columns of every block split into wl.tiles tiles; each query row's L over
    the b1*t super-keys) on resident bfloat16 inputs, its algorithmic FLOPs against
    the path roofline, the per-kernel split, and the rel-Frobenius error of sampled
    (head, column) problems against the float64 oracle."""
    import torch
    from structured_attention_video_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks, peak_kind = load_peaks()
    shape = (wl.B, wl.H, wl.N, wl.d)
    hq, hk, hv = (torch.empty(shape, dtype=torch.int16) for _ in range(3))
    synth.fill_device_bits(wl, hq.numpy().view(np.uint16), hk.numpy().view(np.uint16),
                           hv.numpy().view(np.uint16), 0)
    q, k, v = (x.to(dev).view(torch.bfloat16) for x in (hq, hk, hv))
    out = torch.empty_like(q)
    sargs = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
    axis = _lib.TILE_KEY_COLUMNS
    nb = _lib.monarch_attn_tiled_workspace_bytes(*sargs, _lib.BF16, axis)
    path = _lib.monarch_attn_tiled_path(*sargs, _lib.BF16, axis)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)

    def step():
        _lib.check(_lib.monarch_attn_fwd_tiled_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  out.data_ptr(), *sargs, _lib.BF16, axis,
                                                  _lib.BHND, ws.data_ptr(), nb, sh),
                   "monarch_attn_fwd_tiled_ws")
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    _lib.monarch_profile_enable(1)
    _lib.monarch_profile_collect()
    times = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    _lib.monarch_profile_enable(0)
    prof = _lib.monarch_profile_collect()
    _lib.check(_lib.monarch_last_device_status(sh), "device status (key tiles)")
    kernels = {name: ms_tot / max(1, args.steps) for name, (ms_tot, cnt) in prof.items() if cnt > 0}
    ms = float(np.median(times))
    flops = wl.monarch_flops_keytiles()
    io = wl.io_bytes()
    roof_ms = max(flops / (peaks["bf16_tflops"] * 1e12), io / (peaks["hbm_gbs"] * 1e9)) * 1e3
    # the CPU-baseline leg: the oracle on sampled (head, column) problems (every
    # query row of each), timed and scaled to a whole step; the same rows give the
    # rel-Frobenius error of the device output
    base = None
    if not args.no_cpu_baseline and args.keytile_samples > 0:
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
        base = keytile_cpu_baseline(wl, got, args.keytile_samples)
    cfg = workload_config(wl, 1)
    cfg["tile_axis"] = "key columns"
    print(json.dumps({
        "metric": "Monarch-attn forward ms, key-column tiles", "value": ms, "unit": "ms",
        "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
        "ms_stats": step_stats(times), "dtype": "bf16", "data": "synthetic", "config": cfg,
        "monarch_gflop": flops / 1e9, "monarch_tflops": flops / (ms * 1e-3) / 1e12,
        "path_roofline": {"roofline_ms": roof_ms, "frac": roof_ms / ms,
                          "peak_source": "%s bf16_tflops (burst) and hbm_gbs" % peak_kind},
        "kernels_ms_per_step": kernels,
        "kernel_path": "sm100 tensor-core" if path == 1 else "generic SIMT",
        "rel_err": None if base is None else base.pop("rel_err"), "cpu_baseline": base,
        "workspace_bytes": nb,
        "gpu": torch.cuda.get_device_name(0)}), flush=True)


# (workload, swept key, values, heads of the dense check): "key_tiles" sweeps the tile
# count with the tiles on the key columns (t = b2 = 52 is exact attention)
SWEEPS = (("480p_full", "tiles", (1, 2, 4, 8), None),
          ("14b", "iters", (1, 2, 5, 10), (0, 13, 27, 40, 53, 79)),
          ("480p_full", "key_tiles", (1, 2, 4, 8, 52), None))


def run_sweeps(args) -> None:
    """One JSON line: for each sweep point, device ms (median of the timed steps),
    Monarch TFLOP/s, the path roofline fraction and the error against exact
    attention; the pages claim the error is monotonically tunable by the tile
    count and falls with more iterations in the training-free regime."""
    import torch
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    peaks, peak_kind = load_peaks()
    records = []
    for base, key, values, heads in SWEEPS:
        wl0 = synth.WORKLOADS[base]
        shape = (wl0.B, wl0.H, wl0.N, wl0.d)
        hq, hk, hv = (torch.empty(shape, dtype=torch.int16) for _ in range(3))
        synth.fill_device_bits(wl0, hq.numpy().view(np.uint16), hk.numpy().view(np.uint16),
                               hv.numpy().view(np.uint16), 0)
        q, k, v = (x.to(dev).view(torch.bfloat16) for x in (hq, hk, hv))
        del hq, hk, hv
        out = torch.empty_like(q)
        bhs = list(heads) if heads else list(range(wl0.B * wl0.H))
        for val in values:
            keys = key == "key_tiles"
            wl = wl0.replace(**{"tiles" if keys else key: val})
            steps = max(3, args.sweep_steps // max(1, wl.iters))
            times, path = time_forward(wl, q, k, v, out, steps, 3, flush, stream,
                                       axis=1 if keys else 0)
            ms = float(np.median(times))
            flops = wl.monarch_flops_keytiles() if keys else wl.monarch_flops()
            io = wl.io_bytes()
            roof_ms = max(flops / (peaks["bf16_tflops"] * 1e12),
                          io / (peaks["hbm_gbs"] * 1e9)) * 1e3
            err = dense_rows_error(wl, q, k, v, out, bhs, args.sweep_rows, seed=val)
            records.append({
                "workload": workload_config(wl, 1)["workload"]
                            + (" (tiles on the key columns)" if keys else ""),
                key: val, "ms_median": ms,
                "steps": steps, "monarch_gflop": flops / 1e9,
                "monarch_tflops": flops / (ms * 1e-3) / 1e12,
                "path_roofline_frac": roof_ms / ms,
                "kernel_path": "sm100 tensor-core" if path == 1 else "generic SIMT",
                "rel_err_vs_dense": err,
                "dense_rows": "%d seeded query rows in each of %d heads" % (args.sweep_rows,
                                                                             len(bhs))})
        del q, k, v, out
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "error against exact attention vs cost (sweeps)",
                      "records": records, "peaks": peak_kind, "gpu": torch.cuda.get_device_name(0)}),
          flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, wl: synth.Workload, world: int, rank: int, local: int):
    import torch
    from structured_attention_video_b200 import _lib

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shape = (wl.B, wl.H, wl.N, wl.d)
    hq, hk, hv = (torch.empty(shape, dtype=torch.int16).pin_memory() for _ in range(3))
    # replicas: every rank its own clip; shard: every rank the same clip, its own units
    shard = args.shard
    synth.fill_device_bits(wl, hq.numpy().view(np.uint16), hk.numpy().view(np.uint16),
                           hv.numpy().view(np.uint16), 0 if shard else rank)
    units = unit_partition(wl.B * wl.H * wl.tiles, world, rank) if shard else None
    q, k, v = (x.to(dev).view(torch.bfloat16) for x in (hq, hk, hv))
    out = torch.empty_like(q)
    hout = torch.empty(shape, dtype=torch.int16).pin_memory()
    sargs = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
    ws_bytes = _lib.monarch_attn_workspace_bytes(*sargs, _lib.BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    path = _lib.monarch_attn_path(*sargs, _lib.BF16)

    def step():
        if shard:
            _lib.check(_lib.monarch_attn_fwd_units_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                      out.data_ptr(), *sargs, _lib.BF16, *units,
                                                      ws.data_ptr(), ws_bytes, sh),
                       "monarch_attn_fwd_units_ws")
        else:
            _lib.check(_lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                out.data_ptr(), *sargs, _lib.BF16, ws.data_ptr(),
                                                ws_bytes, sh), "monarch_attn_fwd_ws")

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    _lib.check(_lib.monarch_last_device_status(sh), "device status after warm-up")
    _lib.monarch_profile_collect()

    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler("GPU-" + str(props.uuid))
    clocks.start()
    time.sleep(0.3)
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    rank_barrier(world)
    torch.cuda.synchronize()
    _lib.monarch_profile_enable(1)
    for a, b in events:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    rank_barrier(world)
    _lib.monarch_profile_enable(0)
    clock_rec = clocks.stop()
    prof = _lib.monarch_profile_collect()
    _lib.check(_lib.monarch_last_device_status(sh), "device status after timed steps")
    step_ms = [a.elapsed_time(b) for a, b in events]
    ms_step = max_over_ranks(sum(step_ms) / args.steps, world, dev)
    # percentiles of the per-step times, each the max over ranks (same order on every rank)
    stats = {k: max_over_ranks(v, world, dev) for k, v in step_stats(step_ms).items()}

    # end to end through the C ABI with host buffers: H2D inputs, forward, D2H output.
    # Replicas: monarch_attn_fwd_host.  Shard: pinned copies of the clip in, the
    # rank's units through monarch_attn_fwd_units_ws, the rank's heads out.
    e2e_times = []
    es = 2
    head_bytes = wl.N * wl.d * es
    if shard:
        hb, he = units[0] // wl.tiles, (units[1] + wl.tiles - 1) // wl.tiles
        h2d_bytes, d2h_bytes = 3 * wl.B * wl.H * head_bytes, (he - hb) * head_bytes
    else:
        h2d_bytes, d2h_bytes = 3 * wl.B * wl.H * head_bytes, wl.B * wl.H * head_bytes
    for i in range(args.e2e_warmup + args.e2e_steps if args.e2e_steps > 0 else 0):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if shard:
            for dst, src in ((q, hq), (k, hk), (v, hv)):
                dst.view(torch.int16).copy_(src, non_blocking=True)
            step()
            hout.view(wl.B * wl.H, -1)[hb:he].copy_(
                out.view(torch.int16).view(wl.B * wl.H, -1)[hb:he], non_blocking=True)
        else:
            _lib.check(_lib.monarch_attn_fwd_host(hq.data_ptr(), hk.data_ptr(), hv.data_ptr(),
                                                  hout.data_ptr(), *sargs, _lib.BF16, sh),
                       "monarch_attn_fwd_host")
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.e2e_warmup:
            e2e_times.append(a.elapsed_time(b))
    e2e_ms = max_over_ranks(statistics.mean(e2e_times), world, dev) if e2e_times else None

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    dense = wl.dense_flops()
    clips = 1 if shard else world   # clips the whole job processes per step
    value = job_throughput(clips, dense, ms_step)
    kernels = {name: {"ms_per_launch": ms / n, "launches": n, "share": ms / max(1e-9, sum(
        m for m, _ in prof.values()))} for name, (ms, n) in prof.items() if n > 0}
    dominant = max(kernels, key=lambda kk: kernels[kk]["ms_per_launch"] * kernels[kk]["launches"])
    roof = kernel_roofline(dominant, kernels[dominant]["ms_per_launch"], wl, peaks, peak_kind)
    roof["kernel"] = dominant
    clock_scaled(roof, clock_rec, peaks)
    traffic = kernel_traffic(dominant)
    roof["traffic"] = traffic
    roof["traffic_unit"] = "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"
    flops = wl.monarch_flops()
    io = wl.io_bytes()
    roof_ms = max(flops / (peaks["bf16_tflops"] * 1e12), io / (peaks["hbm_gbs"] * 1e9)) * 1e3
    launches = sum(kk["launches"] for kk in kernels.values())
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(wl, world, shard),
        "ms_stats": stats,
        "monarch_tflops": clips * flops / (ms_step * 1e-3) / 1e12,
        "path_roofline": {"roofline_ms": roof_ms, "frac": roof_ms / ms_step,
                          "flops_per_step": flops, "io_bytes_per_step": io,
                          "peak_source": "%s bf16_tflops (burst) and hbm_gbs" % peak_kind,
                          "note": "the whole step against max(Monarch FLOPs / bf16 peak, "
                                  "Q/K/V/O bytes / HBM bandwidth): the figure the 50%% "
                                  "target reads; roofline.frac covers one kernel only"},
        "roofline": roof,
        "kernels": kernels,
        "kernel_path": "sm100 tensor-core" if path == 1 else "generic SIMT",
        "gpu_launches": launches,
        "e2e": None if e2e_ms is None else {
            "value": job_throughput(clips, dense, e2e_ms), "unit": UNIT,
            "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": h2d_bytes,
            "d2h_bytes_per_step": d2h_bytes,
            "api": ("monarch_attn_fwd_units_ws with pinned host copies (rank's heads out)"
                    if shard else "monarch_attn_fwd_host (C ABI, pinned host buffers)")},
        "clocks": clock_rec,
        "gpu": props.name,
    }
    if shard:
        line["units"] = {"rank0": list(units), "total": wl.B * wl.H * wl.tiles}
    if world == 1 and args.secondary_steps > 0 and args.workload == "720p" and args.heads == 0:
        line["also_480p"] = secondary_workload(synth.WORKLOADS["480p_full"], args.secondary_steps,
                                               3, flush, stream)
    if world == 1 and not args.no_cpu_baseline:
        def rows_of_head(bh, rows):
            b, h = divmod(bh, wl.H)
            bits = out[b, h, torch.as_tensor(rows, device=dev)].view(torch.int16).cpu().numpy()
            return synth.from_device_bits(bits.view(np.uint16), "bf16")
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, rows_of_head)
        line["rel_err"] = line["cpu_baseline"].pop("rel_err")
    else:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="720p", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-warmup", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--secondary-steps", type=int, default=50,
                    help="timed steps of the 480p full clip reported beside the line (0: skip)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (smaller cases for ncu captures; not a bench line)")
    ap.add_argument("--iters", type=int, default=0,
                    help="override the alternating rounds (captures of the iteration kernels; "
                         "not a bench line)")
    ap.add_argument("--shard", action="store_true",
                    help="N > 1: split ONE clip's (head, tile) units across the ranks "
                         "(strong scaling) instead of one clip per rank")
    ap.add_argument("--sweep", action="store_true",
                    help="error-vs-cost sweeps (tiles on 480p, iterations on Wan-14B) instead "
                         "of the bench line; one GPU")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass of one iteration on --workload instead of "
                         "the forward bench line; one GPU")
    ap.add_argument("--key-tiles", action="store_true",
                    help="time the forward pass with key-column tiles (the other reading of "
                         "the tiles) on --workload instead of the bench line; one GPU")
    ap.add_argument("--keytile-samples", type=int, default=8,
                    help="(head, column) problems checked against the oracle by --key-tiles")
    ap.add_argument("--sweep-steps", type=int, default=20)
    ap.add_argument("--sweep-rows", type=int, default=1024)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and "OMP_NUM_THREADS" not in os.environ:
        # each rank generates its own clip on the host with OpenMP: share the cores
        # (set before torch loads the OpenMP runtime, which reads it once)
        per_node = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
        os.environ["OMP_NUM_THREADS"] = str(max(1, len(os.sched_getaffinity(0)) // per_node))
    if args.gpus != world:
        ap.error("--gpus %d but WORLD_SIZE=%d: launch N > 1 with torchrun" % (args.gpus, world))
    wl = synth.WORKLOADS[args.workload]
    if args.heads > 0:
        wl = wl.replace(H=args.heads)
    if args.iters > 0:
        wl = wl.replace(iters=args.iters)

    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    if args.sweep:
        if world != 1:
            ap.error("--sweep runs on one GPU")
        run_sweeps(args)
        return
    if args.backward:
        if world != 1:
            ap.error("--backward runs on one GPU")
        run_backward(args, wl)
        return
    if args.key_tiles:
        if world != 1:
            ap.error("--key-tiles runs on one GPU")
        run_keytiles(args, wl)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    try:
        run_ours(args, wl, world, rank, local)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
