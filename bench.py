"""Benchmark of one TriAttention prune step on B200 (libtri, sm_100a).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c4]
                    [--impl reference] [--n-seq S] [--n-layers L]
                    [--no-cpu-baseline] [--no-sub]

A step is one pass of the whole prune path (fold, score, z-normalise / max,
top-B select, order-preserving gather of K, V and positions) over every unit
of the workload.  Units are independent, so at N GPUs every rank prunes its
own copy of the workload (weak scaling, no collective on the data path) and
``value`` counts the keys of all ranks over the slowest rank's time.

Default workload: the long-prefill compaction (32 layers x 8 KV heads x 4
sequences, GQA 32/8, 131072 bf16 keys per head, budget 4096), the largest
configuration that fits one GPU.  The same line carries driver-timed
sub-records of the other 32K-token configurations (one layer of 4 KV heads
at 32768 keys; the windowed decode step; the streaming step), each with its
time per step, keys/s and fraction of the HBM roofline.  Metric: keys
scored and pruned per second, plus the achieved HBM bandwidth of the step's
compulsory bytes (read every key, read the kept values, write the kept keys
and values, indices and positions) against the measured copy peak (and,
as ``hbm_frac_of_nominal``, against the nominal 8 TB/s).

Timing: W warm-up steps, then K steps captured as one CUDA graph and replayed
between CUDA events on the launching stream, with a barrier and a device
synchronise on both sides; the inputs rotate over enough copies that their
total exceeds the 126 MB L2 (no step reads a cache another step left in L2).
Per-kernel durations come from events the library records after each of its
launches inside the same graph.  ``e2e`` repeats the step through the public
Python API with host (pinned) buffers: the copy of the inputs in and of the
compacted cache out is inside its timed region.

``--impl reference`` times the float64 CPU oracle (the baseline) on the host
cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "keys scored+pruned/sec and achieved HBM GB/s (% of ~8 TB/s) per prune step"
# The nominal HBM3e figure the metric's percentage names; the roofline
# fractions use the measured copy peak instead (MEASURED_PEAKS.json, else the
# 6650 GB/s fallback), which a plain copy can reach.
NOMINAL_HBM_GBS = 8000.0

WORKLOAD_TEXT = {
    "c1": "single head fp32, 4096 keys -> 512, G=1",
    "c2": "1 layer, GQA 28/4, 32768 bf16 keys per KV head -> 2048",
    "c3": "windowed decode step, 28 layers x 4 KV heads x 16 seqs, 3200 -> 3072 keys, G=7",
    "c4": "long prefill compaction, 32 layers x 8 KV heads x 4 seqs, 131072 -> 4096 keys, G=4",
    "c5": "streaming step, 28 layers x 4 KV heads x 64 seqs, 2176 -> 2048 keys, G=7",
}


def compulsory_bytes(spec) -> int:
    """Per step: read every valid key, read the kept values, write the kept
    keys and values, plus 4-byte index and position of every kept row read and
    written (12 bytes per kept key)."""
    e = spec.esize
    m = min(spec.n_valid, spec.B)
    per_unit = spec.n_valid * spec.d * e + m * spec.d * e + 2 * m * spec.d * e + 12 * m
    return per_unit * spec.n_units


def score_bytes(spec) -> int:
    """Algorithmic bytes of the score kernel per launch: every valid key read once."""
    return spec.n_units * spec.n_valid * spec.d * spec.esize


def fused_bytes(spec) -> int:
    return compulsory_bytes(spec)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel per launch, from one ncu capture each (summaries under profiles/),
# keyed by workload and kernel, with the hash of the kernel sources it was
# taken on: once the sources change, ``traffic`` is reported as null until the
# kernel is captured again.  "scale" multiplies a capture of a smaller case of
# the workload up to one full launch (traffic grows with the units processed).
TRAFFIC = {
    # profiles/prune_coop_kernel_c2_full.txt
    ("c2", "prune_coop_kernel"): {"bytes_per_launch": 36205824, "src": "c77c64c097379d81"},
    # profiles/prune_pipe_kernel_c3-2seq_full.txt: 224 of 1792 units captured, x 8
    ("c3", "prune_pipe_kernel"): {"bytes_per_launch": 7422631936, "src": "91d6d2f340ec24f9"},
    # profiles/score_kernel_c4-1seq-2layers_full.txt: 16 of 1024 units captured, x 64
    ("c4", "score_kernel"): {"bytes_per_launch": 36379787264, "src": "e5c635935b897aaa"},
}


def _code_only(text: str) -> str:
    """C++ source without comments and with whitespace collapsed, so that a
    change to comments alone does not count as a change of the kernels
    (string literals in these sources hold no comment markers)."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


# Translation unit of each kernel whose traffic is recorded.
KERNEL_SOURCE = {
    "prune_coop_kernel": "coop.cu",
    "prune_fused_kernel": "fused.cu",
    "prune_pipe_kernel": "pipe.cu",
    "score_kernel": "score.cu",
}


def kernel_sources_hash(kernel: str = "") -> str:
    """Hash of the code (comments stripped) a kernel is compiled from: its
    translation unit and every local header it includes, transitively; with
    no kernel named, of every source file."""
    import hashlib
    import re

    d = os.path.join(ROOT, "rope_aware_kv_b200", "csrc")
    if kernel in KERNEL_SOURCE:
        files, todo = set(), [KERNEL_SOURCE[kernel]]
        while todo:
            name = todo.pop()
            if name in files or not os.path.exists(os.path.join(d, name)):
                continue
            files.add(name)
            with open(os.path.join(d, name), encoding="utf-8") as fh:
                todo += re.findall(r'#include\s+"([^"/]+)"', fh.read())
        names = sorted(files)
    else:
        names = sorted(n for n in os.listdir(d) if n.endswith((".cu", ".cuh", ".h")))
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(d, name), encoding="utf-8") as fh:
            h.update(name.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, kernel: str, cut: bool):
    rec = TRAFFIC.get((workload, kernel))
    if rec is None or cut or rec["src"] != kernel_sources_hash(kernel):
        return None
    return rec["bytes_per_launch"]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# clocks (NVML polled in a thread during the timed region)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        reasons = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# the oracle (CPU baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(spec, seconds_hint: float = 8.0, units=None):
    """Bounded sample of the workload for the CPU oracle: ``units`` units (one
    per oracle thread by default) drawn from the generator on the host, cut
    to a key count that keeps each unit to roughly ``seconds_hint`` seconds of
    one core.  Returns (inputs, keys, description, units)."""
    import oracle

    threads = oracle.threads()
    n_units = max(1, min(spec.n_units, units if units is not None else threads))
    # ~ 17 offsets x 64 bands x G cosines per key, about 25 ns each
    per_key = 17 * 64 * spec.G * 25e-9
    n_keys = int(min(spec.n_valid, max(256, seconds_hint / per_key)))
    sub = synth.Spec(spec.name + "-sample", 1, 1, n_units, spec.G, n_keys, n_keys,
                     min(spec.B, max(1, n_keys * spec.B // max(spec.n_valid, 1))), spec.dtype,
                     min(spec.n_cal, 2048), spec.p_cur, positions="dense", R_range=spec.R_range,
                     outlier_frac=spec.outlier_frac, stream=spec.stream)
    wl = synth.make_workload(sub, "cpu")
    q = synth.calib_queries(sub, wl.hp, 0, "cpu")
    st = oracle.calibrate(synth.host_elems(q))[None]
    inputs = dict(k=synth.host_elems(wl.k), v=synth.host_elems(wl.v), pos=wl.pos.numpy(),
                  p_cur=wl.p_cur.numpy(), stats=st, sub=sub)
    desc = (f"sampled: {n_units} unit(s) x {n_keys} keys (G={spec.G}, B={sub.B}) of "
            f"{spec.name}")
    return inputs, n_units * n_keys, desc, n_units


def oracle_step(inp):
    import oracle

    sub = inp["sub"]
    oracle.prune(inp["k"], inp["v"], inp["pos"], 1, 1, sub.n_kvheads, sub.G, inp["stats"],
                 inp["p_cur"], sub.B, want_raw=False, want_gather=True)


def cpu_baseline(spec):
    """The float64 oracle on the host cores, on a sample of the workload: one
    unit per thread with every thread, then one unit on one thread."""
    import oracle

    threads = oracle.threads()
    inp, keys, desc, n_units = oracle_sample(spec)
    t0 = time.perf_counter()
    oracle_step(inp)
    dt_all = time.perf_counter() - t0
    inp1, keys1, desc1, _ = oracle_sample(spec, units=1)
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle_step(inp1)
        dt_one = time.perf_counter() - t0
    finally:
        oracle.set_threads(threads)
    return {"value": keys / dt_all, "unit": "keys/s", "cores": os.cpu_count(),
            "threads": min(n_units, threads), "kind": "oracle",
            "sample": desc + f", oracle on {min(n_units, threads)} thread(s)",
            "seconds": round(dt_all, 3),
            "single_thread": {"value": keys1 / dt_one, "unit": "keys/s", "threads": 1,
                              "sample": desc1 + ", oracle on 1 thread",
                              "seconds": round(dt_one, 3)}}


def run_reference_decode(args):
    """The oracle's decode attention on a sample of the compacted streaming
    cache (a few units), scaled to a whole decode step of the workload."""
    import oracle

    spec = synth.SPECS["c5"]
    rng = np.random.default_rng(5)
    units = min(spec.n_units, max(1, oracle.threads()))
    q = rng.normal(size=(units, spec.G, spec.d)).astype(np.float32) * 0.1
    k = rng.normal(size=(units, spec.B, spec.d)).astype(np.float32)
    v = rng.normal(size=(units, spec.B, spec.d)).astype(np.float32)
    to_bf16 = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)
    q, k, v = to_bf16(q), to_bf16(k), to_bf16(v)
    for _ in range(args.warmup):
        oracle.decode_attention(q, k, v)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.decode_attention(q, k, v)
    dt = (time.perf_counter() - t0) / args.steps
    step_s = dt * spec.n_units / units
    value = spec.n_seq / step_s
    desc = (f"sampled: {units} unit(s) x {spec.B} kept rows (G={spec.G}), oracle on "
            f"{min(units, oracle.threads())} thread(s), scaled to {spec.n_units} units")
    line = {
        "impl": "reference",
        "metric": "decode-attention tokens/s over the compacted cache (all layers and KV heads)",
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode", "sample": desc},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": os.cpu_count(),
                         "threads": min(units, oracle.threads()), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference(args, ws, rank):
    if rank != 0:
        return
    import oracle

    if args.workload == "decode":
        run_reference_decode(args)
        return
    stream_run = args.workload == STREAM
    spec = synth.SPECS["c5" if stream_run else args.workload]
    inp, keys, desc, n_units = oracle_sample(spec, seconds_hint=0.5)
    for _ in range(args.warmup):
        oracle_step(inp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp)
    dt = (time.perf_counter() - t0) / args.steps
    value = keys / dt
    threads = min(n_units, oracle.threads())
    desc = desc + f", oracle on {threads} thread(s)"
    if stream_run:
        # Seconds per key of the sample, scaled to the 240 prunes of the
        # stream at full width, per generated token.
        prunes = (synth.STREAM_TOKENS - spec.cap) // synth.STREAM_WINDOW + 1
        us_tok = dt / keys * spec.n_units * spec.cap * prunes / synth.STREAM_TOKENS * 1e6
        line = {
            "impl": "reference",
            "metric": "prune-path time per generated token (appends included), streaming run",
            "value": us_tok, "unit": "us/token", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": STREAM, "sample": desc + "; scaled by keys to the 240 "
                       "prunes of the full-width stream (appends not counted)"},
            "cpu_baseline": {"value": us_tok, "unit": "us/token", "cores": os.cpu_count(),
                             "threads": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": us_tok, "unit": "us/token", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]}",
                   "sample": desc},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": os.cpu_count(),
                         "threads": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
class StepRunner:
    """Inputs, destinations and workspace of one prune step, rotated over
    enough input copies that every step reads from HBM."""

    def __init__(self, spec, device, n_copies=None):
        import rope_aware_kv_b200 as tri

        self.tri = tri
        self.spec = spec
        wl = synth.make_workload(spec, device)
        self.wl = wl
        stats = torch.empty((spec.n_layers, spec.n_qheads, 64, 4), dtype=torch.float32,
                            device=device)
        for layer in range(spec.n_layers):
            q = synth.calib_queries(spec, wl.hp, layer, device)
            tri.tri_calibrate(q, stats=stats[layer])
            del q
        self.stats = stats
        copy_bytes = 2 * wl.k.numel() * wl.k.element_size() + wl.pos.numel() * 4
        if n_copies is None:
            n_copies = max(1, math.ceil(4 * L2_BYTES / copy_bytes))
            free = torch.cuda.mem_get_info()[0]
            n_copies = max(1, min(n_copies, int(0.5 * free // max(copy_bytes, 1))))
        self.inputs = [(wl.k, wl.v, wl.pos)]
        for _ in range(n_copies - 1):
            self.inputs.append((wl.k.clone(), wl.v.clone(), wl.pos.clone()))
        U, B = spec.n_units, spec.B
        m = min(B, spec.cap)
        self.dst = []
        for _ in range(n_copies):
            kd = torch.empty((U, m, spec.d), dtype=wl.k.dtype, device=device)
            self.dst.append((kd, torch.empty_like(kd),
                             torch.empty((U, m), dtype=torch.int32, device=device)))
        self.n_kept = torch.empty((U,), dtype=torch.int32, device=device)
        self.kept = torch.empty((U, B), dtype=torch.int32, device=device)
        self.ws = tri.workspace(tri.tri_prune_workspace_bytes(
            spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.cap, B))
        self.cfg = tri.config()
        self.n_copies = n_copies

    def step(self, i):
        k, v, pos = self.inputs[i % self.n_copies]
        kd, vd, pd = self.dst[i % self.n_copies]
        s = self.spec
        self.tri.tri_prune(self.cfg, k, v, pos, s.n_seq, s.n_layers, s.n_kvheads, s.G,
                           self.wl.p_cur, self.stats, s.B, kd, vd, pd, self.n_kept,
                           n_valid=self.wl.n_valid, kept=self.kept, ws=self.ws)


KERNEL_NAMES = {
    "pipe_small": ["prune_pipe_kernel"],
    "pipe_big": ["fold_kernel", "prune_pipe_kernel"],
    "fused": ["prune_fused_kernel"],
    "coop": ["prune_coop_kernel"],
    "split": ["fold_kernel", "score_kernel", "moment_merge_kernel", "zmax_kernel",
              "zsel_bin_kernel", "zsel_collect_kernel", "zsel_rank_kernel", "zsel_compact_kernel",
              "gather_kernel"],
}


def path_name(tri, spec):
    path = tri.tri_prune_path(spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.cap,
                              spec.B, spec.torch_dtype)
    if path == tri.PATH_PIPE:
        return "pipe_small" if tri.tri_last_launch_count() == 1 else "pipe_big"
    return {tri.PATH_FUSED: "fused", tri.PATH_COOP: "coop"}.get(path, "split")


def time_workload(args, spec, dev, stream, ws, steps):
    """Time `steps` prune steps of spec as one CUDA graph (max over ranks) and
    break the step down per launch.  Returns (runner, record)."""
    import rope_aware_kv_b200 as tri

    runner = StepRunner(spec, dev)
    with torch.cuda.stream(stream):
        # Eager warm-up (also initialises the library's static state).
        for i in range(max(args.warmup, 3)):
            runner.step(i)
        torch.cuda.synchronize()
        tri.tri_set_timing_events(None)
        runner.step(0)
        launches = tri.tri_last_launch_count()
        pname = path_name(tri, spec)

        # Per-launch events inside the timed graph.
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(launches)]
               for _ in range(steps)]
        starts = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(steps)]
        for e in starts + [x for row in evs for x in row]:
            e.record(stream)
        torch.cuda.synchronize()

        # Timed graph: K steps, nothing but the library's own launches.
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            for i in range(steps):
                runner.step(args.warmup + i)
        # Breakdown graph: the same K steps with an event after every launch.
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=stream, capture_error_mode="relaxed"):
            for i in range(steps):
                starts[i].record(stream)
                tri.tri_set_timing_events(evs[i])
                runner.step(args.warmup + i)
            tri.tri_set_timing_events(None)
        gw = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gw, stream=stream, capture_error_mode="relaxed"):
            for i in range(args.warmup):
                runner.step(i)

    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    gw.replay()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    clocks.start()
    with torch.cuda.stream(stream):
        t0.record(stream)
        g.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(ws)
    ms_total = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms_total, ws)
    ms_step = ms_max / steps

    # Per-kernel durations from the breakdown graph (an interval runs from the
    # previous launch's event to this launch's event; the first launch's
    # interval includes the workspace memsets).
    with torch.cuda.stream(stream):
        gw.replay()
        ge.replay()
    torch.cuda.synchronize()
    per_launch = np.zeros(launches)
    ev_total = 0.0
    for i in range(steps):
        prev = starts[i]
        for j in range(launches):
            per_launch[j] += prev.elapsed_time(evs[i][j])
            prev = evs[i][j]
        ev_total += starts[i].elapsed_time(evs[i][-1])
    per_launch /= steps
    ev_step = ev_total / steps
    flags = tri.tri_check_device_error(runner.ws)
    del g, ge, gw
    peak_gbs, peak_kind = measured_peaks()
    comp = compulsory_bytes(spec)
    keys_rank = spec.n_units * spec.n_valid
    rec = {
        "workload": f"{spec.name}: {WORKLOAD_TEXT.get(spec.name, spec.name)}",
        "path": pname, "ms_per_step": ms_step, "value": keys_rank * ws / (ms_step * 1e-3),
        "unit": "keys/s", "hbm_gbs": comp / (ms_step * 1e-3) / 1e9,
        "frac": comp / (ms_step * 1e-3) / 1e9 / peak_gbs, "peak_gbs": peak_gbs,
        "peak_kind": peak_kind, "compulsory_bytes_per_step": comp, "steps": steps,
        "launches_per_step": launches, "device_flags": flags,
        "per_launch_ms": [round(float(x), 5) for x in per_launch],
        "evented_ms_per_step": ev_step, "clocks": clk,
        "l2": f"inputs rotated over {runner.n_copies} copies "
              f"({runner.n_copies * comp / 2**20:.0f} MiB compulsory > 126 MB L2)",
    }
    return runner, rec


def dominant(spec, rec, ms_step):
    """The dominant kernel of a step, its algorithmic bytes and its time."""
    names = KERNEL_NAMES[rec["path"]]
    per_launch = rec["per_launch_ms"]
    dom = int(np.argmax(per_launch))
    dom_name = names[dom] if dom < len(names) else f"launch{dom}"
    if dom_name in ("prune_pipe_kernel", "prune_fused_kernel", "prune_coop_kernel"):
        # One kernel runs the whole path: the step's compulsory bytes.
        dom_bytes = compulsory_bytes(spec)
    else:
        gather_bytes = spec.n_units * min(spec.B, spec.n_valid) * (3 * spec.d * spec.esize + 12)
        dom_bytes = {"score_kernel": score_bytes(spec), "gather_kernel": gather_bytes}.get(dom_name, 0)
    # The breakdown graph's events stretch each step a little; scale the
    # dominant kernel's interval by the plain graph's step time.
    ev = rec["evented_ms_per_step"]
    dom_ms = float(per_launch[dom]) * (ms_step / ev if ev > 0 else 1.0)
    return dom_name, dom_bytes, dom_ms


SUB_WORKLOADS = ("c2", "c3", "c5")
STREAM = "c5-stream"


def time_stream(args, dev, stream, ws, inplace_too=True):
    """The streaming workload end to end (64 sequences x 28 layers x 4 KV
    heads, G 7, B 2048): from an empty cache, the 256 windows of 128 generated
    tokens (32768 tokens) are appended with tri_append and the cache is
    pruned back to B whenever it holds B + 128 rows (240 prunes), through the
    window driver, on two cache buffers (tri_prune) and, on the same windows,
    on one buffer compacted in place (tri_prune_inplace).  Each window's keys
    are drawn at their own positions before its segment; the library's
    launches of a segment (append, then prune) are timed between CUDA events
    on the launching stream and summed, max over ranks."""
    import rope_aware_kv_b200 as tri
    from rope_aware_kv_b200.window import WindowDriver

    spec = synth.SPECS["c5"]
    hp = synth.head_params(spec)
    stats = torch.empty((spec.n_layers, spec.n_qheads, 64, 4), dtype=torch.float32, device=dev)
    for layer in range(spec.n_layers):
        q = synth.calib_queries(spec, hp, layer, dev)
        tri.tri_calibrate(q, stats=stats[layer])
        del q
    window = synth.STREAM_WINDOW
    n_windows = synth.STREAM_TOKENS // window
    modes = [False, True] if inplace_too else [False]
    drivers = {m: WindowDriver(spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.B, stats,
                               window=window, device=dev, inplace=m) for m in modes}

    launches = {m: 0 for m in modes}

    def run(n, timed):
        ev = {m: [] for m in modes}
        with torch.cuda.stream(stream):
            for d in drivers.values():
                d.reset()
            for w in range(n):
                k_new, v_new, pos_new = synth.stream_window(spec, hp, w, dev)
                for m, d in drivers.items():
                    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                    e[0].record(stream)
                    d.append(k_new, v_new, pos_new, auto_prune=False, stream=stream)
                    if timed:
                        launches[m] += tri.tri_last_launch_count()
                    e[1].record(stream)
                    if d.full:
                        d.prune(stream=stream)
                        if timed:
                            launches[m] += tri.tri_last_launch_count()
                    e[2].record(stream)
                    ev[m].append(e)
                del k_new, v_new, pos_new
        torch.cuda.synchronize()
        return ev

    run(spec.cap // window + 3, False)  # warm-up: three prunes per driver
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    barrier(ws)
    clocks.start()
    ev = run(n_windows, True)
    clk = clocks.stop()
    barrier(ws)
    peak_gbs, peak_kind = measured_peaks()
    comp = compulsory_bytes(spec)
    out = {}
    for m, d in drivers.items():
        app = sum(e[0].elapsed_time(e[1]) for e in ev[m])
        pru = sum(e[1].elapsed_time(e[2]) for e in ev[m])
        flags = tri.tri_check_device_error(d.ws)
        total = max_over_ranks(app + pru, ws)
        roof_ms = d.prunes * comp / (peak_gbs * 1e9) * 1e3
        out["inplace" if m else "pingpong"] = {
            "tokens": d.tokens, "windows": n_windows, "prunes": d.prunes,
            "total_ms": total, "append_ms": app, "prune_ms": pru,
            "prune_ms_mean": pru / max(d.prunes, 1),
            "us_per_token": total * 1e3 / d.tokens,
            "keys_per_s": d.prunes * spec.n_units * spec.cap * ws / (total * 1e-3),
            "path": {tri.PATH_PIPE: "pipe", tri.PATH_SPLIT: "split", tri.PATH_COOP: "coop",
                     tri.PATH_FUSED: "fused"}.get(
                tri.tri_prune_path(spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G, spec.cap,
                                   spec.B, inplace=m), "none"),
            "roofline_us_per_token": roof_ms * 1e3 / d.tokens,
            "frac": roof_ms / total if total > 0 else 0.0,
            "device_flags": flags, "gpu_launches": launches[m],
        }
    del drivers
    torch.cuda.empty_cache()
    return {
        "workload": f"{STREAM}: {synth.STREAM_TOKENS} generated tokens, 64 seqs x 28 layers x "
                    f"4 KV heads, G 7, B {spec.B}, prune every {window} tokens "
                    f"(cache B + {window} rows)",
        "compulsory_bytes_per_prune": comp, "peak_gbs": peak_gbs, "peak_kind": peak_kind,
        "timing": "per window: CUDA events around the append and the prune on the launching "
                  "stream, summed over the stream; key generation outside the timed segments",
        "clocks": clk, **out,
    }


def run_tri(args, ws, rank, local):
    import rope_aware_kv_b200 as tri
    from rope_aware_kv_b200 import build as tri_build

    if rank == 0:
        tri_build.build()
    barrier(ws)
    tri.load()
    if args.workload == STREAM:
        run_stream_line(args, ws, rank, local)
        return
    if args.workload == "decode":
        run_decode_line(args, ws, rank, local)
        return
    spec = synth.SPECS[args.workload]
    if args.n_seq:
        spec = spec.scaled(n_seq=args.n_seq)
    if args.n_layers:
        spec = spec.scaled(n_layers=args.n_layers)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    peak_gbs, peak_kind = measured_peaks()

    runner, rec = time_workload(args, spec, dev, stream, ws, args.steps)
    ms_step = rec["ms_per_step"]
    dom_name, dom_bytes, dom_ms = dominant(spec, rec, ms_step)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9 if dom_ms > 0 else 0.0
    e2e = None if args.no_e2e else run_e2e(args, runner, stream, spec, ws)
    launches = rec["launches_per_step"]
    del runner
    torch.cuda.empty_cache()

    # Timed sub-records of the other 32K-token configurations.
    subs = {}
    if not (args.no_sub or args.n_seq or args.n_layers):
        for name in SUB_WORKLOADS:
            if name == args.workload:
                continue
            r2, srec = time_workload(args, synth.SPECS[name], dev, stream, ws,
                                     min(args.steps, 50))
            dn, db, dms = dominant(synth.SPECS[name], srec, srec["ms_per_step"])
            srec["roofline"] = {"kernel": dn, "achieved": db / (dms * 1e-3) / 1e9 if dms > 0 else 0,
                                "algorithmic_bytes": db, "ms_per_launch": dms,
                                "traffic": measured_traffic(name, dn, False)}
            subs[name] = srec
            del r2
            torch.cuda.empty_cache()
        subs[STREAM] = time_stream(args, dev, stream, ws)
        subs["decode"] = time_decode(args, dev, stream, ws, min(args.steps, 50))

    cpu = cpu_baseline(spec) if (rank == 0 and ws == 1 and not args.no_cpu_baseline) else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": rec["value"], "unit": "keys/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if spec.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {
                "workload": rec["workload"] + (
                    f" (cut to {spec.n_seq} sequence(s) x {spec.n_layers} layer(s))"
                    if (args.n_seq or args.n_layers) else ""),
                "units": spec.n_units, "keys_per_unit": spec.n_valid, "budget": spec.B,
                "group": spec.G, "head_dim": spec.d, "parallelism": f"dp{ws} (independent units)",
                "l2": rec["l2"],
                "timing": "one CUDA graph of K steps between CUDA events, max over ranks",
            },
            "hbm_gbs": rec["hbm_gbs"], "hbm_frac_of_peak": rec["frac"],
            "hbm_frac_of_nominal": rec["hbm_gbs"] / NOMINAL_HBM_GBS,
            "compulsory_bytes_per_step": rec["compulsory_bytes_per_step"],
            "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": achieved,
                         "peak": peak_gbs, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak_gbs,
                         "traffic": measured_traffic(args.workload, dom_name,
                                                     bool(args.n_seq or args.n_layers)),
                         "algorithmic_bytes": dom_bytes, "ms_per_launch": dom_ms},
            "per_launch_ms": rec["per_launch_ms"],
            "path": rec["path"],
            "evented_ms_per_step": rec["evented_ms_per_step"],
            "gpu_launches": int(launches * args.steps),
            "device_flags": rec["device_flags"],
            "clocks": rec["clocks"],
            "e2e": e2e,
            "cpu_baseline": cpu,
            "sub_workloads": subs,
        }
        print(json.dumps(line), flush=True)


def time_decode(args, dev, stream, ws, steps, n_seq=0):
    """Decode attention of the next token over the streaming workload's
    compacted cache (64 seqs x 28 layers x 4 KV heads, G 7, B 2048 kept rows
    per unit): K and V rows read once per step, 7.5 GB > L2.  One CUDA graph
    of ``steps`` calls between CUDA events, max over ranks.  ``n_seq``: a
    cut to fewer sequences (profiler captures)."""
    import rope_aware_kv_b200 as tri

    spec = synth.SPECS["c5"]
    if n_seq:
        spec = spec.scaled(n_seq=n_seq)
    U, B, G = spec.n_units, spec.B, spec.G
    g = torch.Generator(device=dev).manual_seed(5)
    k = torch.empty((U, B, spec.d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    for u0 in range(0, U, 512):
        k[u0:u0 + 512] = torch.randn((min(512, U - u0), B, spec.d), generator=g, device=dev)
        v[u0:u0 + 512] = torch.randn((min(512, U - u0), B, spec.d), generator=g, device=dev)
    q = (torch.randn((U, G, spec.d), generator=g, device=dev) * 0.1).to(torch.bfloat16)
    nv = torch.full((U,), B, dtype=torch.int32, device=dev)
    out = torch.empty((U, G, spec.d), dtype=torch.float32, device=dev)
    wsb = tri.workspace(tri.load().tri_decode_workspace_bytes(U, G, B), dev)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            tri.tri_decode_attention(q, k, v, n_valid=nv, out=out, ws=wsb, stream=stream)
        torch.cuda.synchronize()
        launches = tri.tri_last_launch_count()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream, capture_error_mode="relaxed"):
            for _ in range(steps):
                tri.tri_decode_attention(q, k, v, n_valid=nv, out=out, ws=wsb, stream=stream)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        t0.record(stream)
        gr.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), ws) / steps
    flags = tri.tri_check_device_error(wsb)
    del gr, k, v
    torch.cuda.empty_cache()
    peak_gbs, peak_kind = measured_peaks()
    nbytes = U * B * spec.d * 2 * 2 + U * G * spec.d * (2 + 4)
    return {"workload": f"decode attention over the compacted streaming cache: {U} units x {B} "
                        "kept bf16 rows, G 7, one query token per head",
            "ms_per_step": ms, "tokens_per_s": spec.n_seq * ws / (ms * 1e-3),
            "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "frac": nbytes / (ms * 1e-3) / 1e9 / peak_gbs,
            "bytes_per_step": nbytes, "peak_gbs": peak_gbs, "peak_kind": peak_kind,
            "launches_per_step": launches, "device_flags": flags, "steps": steps}


def run_decode_line(args, ws, rank, local):
    """``--workload decode``: decode attention over the compacted streaming
    cache as the bench line (``--n-seq`` cuts it for profiler captures)."""
    import rope_aware_kv_b200 as tri
    from rope_aware_kv_b200 import build as tri_build

    if rank == 0:
        tri_build.build()
    barrier(ws)
    tri.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    rec = time_decode(args, dev, stream, ws, args.steps, n_seq=args.n_seq)
    if rank == 0:
        line = {
            "metric": "decode-attention tokens/s over the compacted cache (all layers and KV heads)",
            "value": rec["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": rec["workload"], "parallelism": f"dp{ws} (independent units)",
                       "l2": f"{rec['bytes_per_step'] / 2**20:.0f} MiB read per step",
                       "timing": "one CUDA graph of K steps between CUDA events"},
            "roofline": {"bound": "hbm", "kernel": "decode_attn_kernel", "achieved": rec["hbm_gbs"],
                         "peak": rec["peak_gbs"], "peak_kind": rec["peak_kind"], "unit": "GB/s",
                         "frac": rec["frac"], "traffic": None},
            "gpu_launches": rec["launches_per_step"] * args.steps,
            "device_flags": rec["device_flags"],
        }
        print(json.dumps(line), flush=True)


def run_stream_line(args, ws, rank, local):
    """``--workload c5-stream``: the streaming run as the bench line (metric:
    prune-path time per generated token, appends included)."""
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    rec = time_stream(args, dev, stream, ws)
    pp = rec["pingpong"]
    if rank == 0:
        line = {
            "metric": "prune-path time per generated token (appends included), streaming run",
            "value": pp["us_per_token"], "unit": "us/token", "n_gpus": ws,
            "steps": pp["prunes"], "warmup": 3, "ms_per_step": pp["total_ms"] / pp["prunes"],
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": rec["workload"], "parallelism": f"dp{ws} (independent units)",
                       "l2": "each prune reads 4.0 GB of keys (> 126 MB L2)",
                       "timing": rec["timing"]},
            "roofline": {"bound": "hbm", "kernel": "whole prune step",
                         "achieved": pp["prunes"] * rec["compulsory_bytes_per_prune"]
                         / (pp["prune_ms"] * 1e-3) / 1e9,
                         "peak": rec["peak_gbs"], "peak_kind": rec["peak_kind"], "unit": "GB/s",
                         "frac": pp["prunes"] * rec["compulsory_bytes_per_prune"]
                         / (pp["prune_ms"] * 1e-3) / 1e9 / rec["peak_gbs"], "traffic": None},
            "gpu_launches": pp["gpu_launches"], "clocks": rec["clocks"], "stream": rec,
        }
        print(json.dumps(line), flush=True)


def run_e2e(args, runner, stream, spec, ws):
    """The same step through the Python API with host buffers: pinned host
    inputs copied in, the prune, and the compacted cache copied out."""
    tri = runner.tri
    wl = runner.wl
    hk = torch.empty(wl.k.shape, dtype=wl.k.dtype, pin_memory=True)
    hv = torch.empty(wl.v.shape, dtype=wl.v.dtype, pin_memory=True)
    hp = torch.empty(wl.pos.shape, dtype=wl.pos.dtype, pin_memory=True)
    hk.copy_(wl.k)
    hv.copy_(wl.v)
    hp.copy_(wl.pos)
    k, v, pos = runner.inputs[0]
    kd, vd, pd = runner.dst[0]
    ok = torch.empty(kd.shape, dtype=kd.dtype).pin_memory()
    ov = torch.empty(vd.shape, dtype=vd.dtype).pin_memory()
    op = torch.empty(pd.shape, dtype=pd.dtype).pin_memory()
    big = hk.numel() * hk.element_size() > (8 << 30)
    steps = 3 if big else max(3, min(args.steps, 20))

    def one():
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        pos.copy_(hp, non_blocking=True)
        tri.tri_prune(runner.cfg, k, v, pos, spec.n_seq, spec.n_layers, spec.n_kvheads, spec.G,
                      wl.p_cur, runner.stats, spec.B, kd, vd, pd, runner.n_kept,
                      n_valid=wl.n_valid, kept=runner.kept, ws=runner.ws)
        ok.copy_(kd, non_blocking=True)
        ov.copy_(vd, non_blocking=True)
        op.copy_(pd, non_blocking=True)

    with torch.cuda.stream(stream):
        one()
        torch.cuda.synchronize()
        barrier(ws)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            one()
        b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), ws) / steps
    h2d = hk.numel() * hk.element_size() + hv.numel() * hv.element_size() + hp.numel() * 4
    d2h = ok.numel() * ok.element_size() + ov.numel() * ov.element_size() + op.numel() * 4
    return {"value": spec.n_units * spec.n_valid * ws / (ms * 1e-3), "unit": "keys/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tri", choices=["tri", "reference"])
    ap.add_argument("--workload", default="c4", choices=sorted(synth.SPECS) + [STREAM, "decode"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-sub", action="store_true",
                    help="time the chosen workload only (no sub-records of the others)")
    ap.add_argument("--n-seq", type=int, default=0,
                    help="run the workload with this many sequences instead (a smaller case "
                         "of the same kernel for profiler captures; not a bench line)")
    ap.add_argument("--n-layers", type=int, default=0,
                    help="run the workload with this many layers instead (as --n-seq)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    ws, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
        else:
            run_tri(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
