#!/usr/bin/env python
"""Benchmark of the speculative flash-decode step on synthetic caches.

One step = one decode token through the 32 layers of a Llama-3.1-8B-shaped
model at 131072 context (batch 1, 32 query / 8 KV heads, d 128, bf16 KV
cache, sink 4, window 1024, lambda 0.10): per layer the sink-set kernel (at
high launch priority), the split exact-attention kernel beside it and the
merge + relative-L2 + flag kernel, all captured in one CUDA graph.  Layers are
independent caches generated from the seed; inputs are resident in HBM.

The other four workloads (a tiny fp32 layer, a 32K layer, a ragged batch of
eight 16K-64K sequences, a Llama-70B-shaped batch of four 128K sequences) are
timed the same way, a few steps each, and reported in the line's per_config
object.

Output: one JSON line on rank 0 (see the keys at the end of run_alspec()).
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl alspec|reference]
With --impl reference the fp64 CPU oracle is timed on the host cores on a
bounded sample of the same workload instead.
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
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV GB/s (fraction of HBM peak) and µs/decode-step to commit flag at 128K"
FALLBACK_HBM_GBS = 6650.0
# The sources a stored ncu traffic figure depends on: the kernels and the
# host planner (which sets the items and partials each launch writes).
KERNEL_SRCS = [os.path.join(ROOT, "speculative_flash_decoding_b200", "csrc", f)
               for f in ("attn_kernels.cuh", "alspec.cu")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_mid_llama8b_128k_traffic.md")
FUSED_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fused_llama8b_128k_ncu.md")


NOMINAL_HBM_GBS = 8000.0  # the HBM3e figure the target is stated against


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["alspec", "reference"], default="alspec")
    ap.add_argument("--config", type=int, default=2, help="workload index (2 = 32 layers @128K)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (0 = workload's)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU-baseline budget (oracle time) on rank 0")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--split-tokens", type=int, default=0,
                    help="exact-path item size for the longest sequence (0 = library's choice)")
    ap.add_argument("--engine", default="auto", choices=["auto", "cuda_cores", "tensor_cores"])
    ap.add_argument("--schedule", default="auto",
                    choices=["auto", "streams", "fused", "sink_first"],
                    help="launch schedule: streams (sink-set, exact-path and merge kernels "
                         "chained on one stream, the exact path beside the sink set), fused "
                         "(one persistent launch) or sink_first (the exact path after the sink "
                         "set); auto = streams")
    ap.add_argument("--oproj", action="store_true",
                    help="speculative output projection against the serial one (32 x 128K)")
    ap.add_argument("--lambda-sweep", action="store_true",
                    help="hit rate against the threshold on the commit-mixing workload family")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' entries (per_config) of the line")
    ap.add_argument("--per-config-steps", type=int, default=10,
                    help="timed steps of each other workload in per_config")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


# ------------------------------------------------------------------ helpers

class Ranks:
    """One process per GPU (launched by torchrun): rank and world size from
    the environment, a process group (NCCL on the GPUs, gloo in the CPU
    tests) for the barrier and the max-over-ranks reduction of times.  The
    ranks are independent replicas: no collective touches the data path."""

    def __init__(self, backend, device):
        import torch
        self.torch = torch
        self.rank, self.world, self.local = dist_env()
        self.device = device
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.pg = dist

    def barrier(self):
        if self.device.type == "cuda":
            self.torch.cuda.synchronize(self.device)
        if self.pg:
            self.pg.barrier()

    def max(self, x):
        """The largest x over all ranks (every rank gets it)."""
        if not self.pg:
            return float(x)
        t = self.torch.tensor([float(x)], dtype=self.torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()
            self.pg = None


def job_throughput(bytes_per_rank, world, ms_per_step):
    """Whole-job GB/s: every rank's bytes over the slowest rank's step time."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            val = float(json.load(f)["hbm_gbs"])
        return val, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def stored_traffic(path, workload):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary of `workload`, or None when the summary covers another workload
    or the kernel or planner source changed since it was captured
    (`source_sha256` is over the files in KERNEL_SRCS, in order)."""
    try:
        text = open(path).read()
    except OSError:
        return None
    m_hash = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    m_work = re.search(r"traffic_workload:\s*(\S+)", text)
    if not (m_hash and m_bytes and m_work) or m_work.group(1) != workload:
        return None
    h = hashlib.sha256()
    for f in KERNEL_SRCS:
        h.update(open(f, "rb").read())
    src = h.hexdigest()
    return int(m_bytes.group(1)) if src == m_hash.group(1) else None


class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
               "-lms", "20"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # nvidia-smi takes a while to start; a timed region shorter than
            # that would get no sample, so wait for the first one (3 s at most).
            t0 = time.time()
            while not self.lines and self.proc.poll() is None and time.time() - t0 < 3.0:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        return self

    def mark(self):
        """Start of the region of interest: samples from here on count."""
        self.start = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=5)

    def summary(self):
        mhz, mx, reasons = [], None, set()
        for line in self.lines[getattr(self, "start", 0):]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                mhz.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


# ------------------------------------------------------------ CPU oracle leg

def oracle_layer_sample(wl, layer, heads_kv=None):
    """Generate one layer on the CPU and return oracle inputs (optionally only
    the first heads_kv KV heads and their query heads) and its KV bytes."""
    import numpy as np
    import workloads
    data = workloads.make_layer(wl, layer=layer, device="cpu")
    q, k, v = data["q"], data["k"], data["v"]
    if heads_kv is not None:
        q = q[:, : heads_kv * wl.g].contiguous()
        k = k[:, :heads_kv].contiguous()
        v = v[:, :heads_kv].contiguous()
    nkv = k.shape[1]
    lens = np.array(data["lens"], np.int32)
    bytes_ = int(sum(data["lens"]) * nkv * wl.d * 2 * wl.elem_bytes)
    return (workloads.to_numpy_bits(q), workloads.to_numpy_bits(k), workloads.to_numpy_bits(v),
            lens), bytes_


def cpu_baseline(wl, budget_s):
    """Time the oracle as it stands on whole layers until ~budget_s of oracle time."""
    import oracle
    total_bytes, total_t, layers, threads = 0, 0.0, 0, 0
    for layer in range(wl.n_layers):
        (q, k, v, lens), nbytes = oracle_layer_sample(wl, layer)
        t0 = time.perf_counter()
        res = oracle.decode(q, k, v, lens, wl.S, wl.W, wl.lam)
        total_t += time.perf_counter() - t0
        total_bytes += nbytes
        threads = res["threads"]
        layers += 1
        if total_t >= budget_s:
            break
    return {"value": total_bytes / total_t / 1e9, "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{layers} of {wl.n_layers} layers of the {wl.name} step (full cache, all "
                      f"heads), fp64 C oracle with OpenMP; {total_t:.1f} s oracle time",
            "us_per_step": total_t / layers * wl.n_layers * 1e6}


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    # Each step: one 128K layer of the workload, its first 2 of 8 KV heads
    # (8 of 32 query heads), generated once outside the timed region.
    (q, k, v, lens), nbytes = oracle_layer_sample(wl, 0, heads_kv=2)
    for _ in range(args.warmup):
        oracle.decode(q, k, v, lens, wl.S, wl.W, wl.lam)
    times, threads = [], 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        res = oracle.decode(q, k, v, lens, wl.S, wl.W, wl.lam)
        times.append(time.perf_counter() - t0)
        threads = res["threads"]
    t = sum(times) / len(times)
    value = nbytes / t / 1e9
    sample = (f"per step: layer 0 of {wl.name}, KV heads 0-1 with their 8 query heads "
              f"({nbytes / 1e6:.0f} MB of KV), fp64 C oracle with OpenMP")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.layers or wl.n_layers, world),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU leg

PROBE_LIB = os.path.join(ROOT, "speculative_flash_decoding_b200", "libalspec_read_probe.so")


def read_probe_fn():
    """alspec_read_probe from libalspec_read_probe.so (include/alspec_read_probe.h):
    (buf, bytes, err, stream) -> status; a measurement aid outside the
    decode library."""
    import ctypes
    lib = ctypes.CDLL(PROBE_LIB)
    fn = lib.alspec_read_probe
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
    return lambda buf, nbytes, stream, err=0: int(fn(buf, nbytes, err or None, stream))


def gpu_uuid(device):
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        return None


def workload_config(wl, n_layers, world):
    """The `config` object of both arms' lines: the workload, nothing about
    how either arm runs it."""
    return {"workload": wl.name, "layers": n_layers, "batch": wl.B, "q_heads": wl.Hq,
            "kv_heads": wl.Hkv, "head_dim": wl.d, "context": wl.L,
            "ragged": list(wl.ragged) if wl.ragged else None, "sink": wl.S, "window": wl.W,
            "lambda": wl.lam, "cache_dtype": wl.dtype,
            "parallelism": "replicas" if world > 1 else "single"}


def middle_bytes(wl, lens, fused):
    """Algorithmic bytes of one launch of the dominant kernel: the middle
    rows [S, L - W) of every sequence (two-stream schedules), or every row
    (one-launch schedule, whose kernel reads the sink set too)."""
    import workloads
    if fused:
        return workloads.kv_bytes(wl, lens)
    return sum(max(0, L - wl.W - min(wl.S, L)) * wl.Hkv * wl.d * 2 * wl.elem_bytes for L in lens)


def quantiles_us(ms):
    if len(ms) < 2:
        return None
    q = statistics.quantiles(ms, n=10)
    return [float(q[0] * 1e3), float(statistics.median(ms) * 1e3), float(q[-1] * 1e3)]


def measure(wl, n_layers, steps, warmup, device, ranks, args, want_e2e=True, lat_layers=4):
    """Time one workload on this rank's GPU (every rank runs the same steps).

    A step is one decode token through the workload's n_layers layers (each
    its own seeded cache, all resident in HBM): per layer the sink-set
    kernel (high launch priority), the exact-path (middle) kernel beside it
    and the merge, captured as one CUDA graph per step.  Passes:
      timed     `steps` graph replays, CUDA events on the launch stream;
                a step whose caches fit a few times in L2 is preceded by an
                untimed L2 flush and timed on its own;
      profiled  the same step with per-layer event nodes: the middle
                kernel's duration (the roofline's denominator).  Events
                between the kernels take away their overlap, so there the
                middle kernel runs once the sink-set kernel has completed:
                its duration alone;
      latency   graphs through the traced entry point (kernel-written time
                stamps of O_spec's and O_exact's publication), over the
                step's layers, or over `lat_layers` distinct layers when the
                step has one, each replay timed too (per-layer time);
      e2e       the step through the public API with host buffers.
    Returns a dict of raw measurements (times in ms)."""
    import torch
    import workloads
    import speculative_flash_decoding_b200 as sfd

    n_lat = n_layers if n_layers >= 2 else lat_layers
    layers = [workloads.make_layer(wl, layer=i, device=device) for i in range(max(n_layers, n_lat))]
    # Each layer's query vectors and lengths side by side in one buffer
    # (q_i, then lens_i padded to 16 bytes), so that a step's inputs are one
    # contiguous host-to-device copy; likewise every layer's rel_l2, then
    # every layer's flag, for the copy back.
    q_bytes = wl.B * wl.Hq * wl.d * wl.elem_bytes
    l_bytes = wl.B * 4
    in_stride = q_bytes + (l_bytes + 15) // 16 * 16
    inputs = torch.empty(len(layers) * in_stride, dtype=torch.uint8, device=device)
    for i, d in enumerate(layers):
        base = i * in_stride
        q_view = inputs[base:base + q_bytes].view(d["q"].dtype).view(d["q"].shape)
        l_view = inputs[base + q_bytes:base + q_bytes + l_bytes].view(torch.int32)
        q_view.copy_(d["q"])
        l_view.copy_(d["seq_lens"])
        d["q"] = q_view
        d["seq_lens"] = l_view
    kv_bytes = sum(workloads.kv_bytes(wl, d["lens"]) for d in layers[:n_layers])
    lat_kv_bytes = sum(workloads.kv_bytes(wl, d["lens"]) for d in layers[:n_lat])
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=device,
                      split_tokens=args.split_tokens, engine=args.engine, schedule=args.schedule)
    plan = dec.plan()
    fused = plan["schedule"] == sfd.ALSPEC_SCHEDULE_FUSED
    n_all = len(layers)
    out_spec = torch.empty(n_all, wl.B, wl.Hq, wl.d, dtype=torch.float32, device=device)
    out_exact = torch.empty_like(out_spec)
    results = torch.empty(n_all * wl.B * 5, dtype=torch.uint8, device=device)
    rel_all = results[:n_all * wl.B * 4].view(torch.float32).view(n_all, wl.B)
    commit_all = results[n_all * wl.B * 4:].view(n_all, wl.B)
    outs = [dict(out_spec=out_spec[i], out_exact=out_exact[i], rel_l2=rel_all[i],
                 commit=commit_all[i]) for i in range(n_all)]
    stream = torch.cuda.Stream(device)
    step_layers = layers[:n_layers]

    def new_events():
        evs = [[torch.cuda.Event(enable_timing=True, external=True)
                for _ in range(sfd.ALSPEC_PROF_EVENTS)] for _ in range(n_layers)]
        for row in evs:      # torch creates the CUDA event at its first record
            for e in row:
                e.record(stream)
        return evs

    def capture(events=None, traces=None, which=None):
        which = step_layers if which is None else which
        with torch.cuda.stream(stream):
            st = sfd.alspec_graph_begin(stream.cuda_stream)
            assert st == 0, sfd.alspec_status_string(st)
            for i, d in enumerate(which):
                dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=outs[i],
                           stream=stream, prof_events=events[i] if events else None,
                           trace=traces[i] if traces is not None else None)
            st, g = sfd.alspec_graph_end(stream.cuda_stream)
            assert st == 0, sfd.alspec_status_string(st)
        return g

    # First call outside capture creates the library's stream and events.
    with torch.cuda.stream(stream):
        for i, d in enumerate(layers):
            dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=outs[i], stream=stream)
    stream.synchronize()

    # Timed graphs carry no profiling events (so nothing sits between the
    # kernels); separate graphs carry the events and the time stamps.
    warm_graph = capture()
    graphs = [capture() for _ in range(steps)]
    prof_steps = max(3, min(steps, 10))
    step_events = [new_events() for _ in range(prof_steps)]
    prof_graphs = [capture(events=ev) for ev in step_events]
    traces = torch.zeros(prof_steps, n_lat, 2, dtype=torch.int64, device=device)
    lat = [capture(traces=traces[j], which=layers[:n_lat]) for j in range(prof_steps)]

    for _ in range(warmup):
        sfd.alspec_graph_launch(warm_graph, stream.cuda_stream)
    ranks.barrier()

    uuid = gpu_uuid(device)
    # Steps whose cache fits a few times in L2 are preceded by an untimed
    # write of twice the L2 size, then a read of another such buffer (so the
    # step does not pay for writing the flush's dirty lines back); each step
    # is then timed on its own.
    l2_bytes = int(getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 0) or
                   (126 << 20))
    flush = kv_bytes < 4 * l2_bytes
    lat_flush = lat_kv_bytes < 4 * l2_bytes
    scrub = clean = sink = None
    if flush or lat_flush:
        scrub = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=device)
        clean = torch.ones(l2_bytes // 2, dtype=torch.int32, device=device)
        sink = torch.empty((), dtype=torch.int64, device=device)

    def flush_l2():
        with torch.cuda.stream(stream):
            scrub.zero_()
            torch.sum(clean, dim=0, out=sink)

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    step_begin = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    step_end = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    nvtx = torch.cuda.nvtx
    with ClockSampler(uuid) as clocks:
        ranks.barrier()
        clocks.mark()
        nvtx.range_push("timed steps " + wl.name)
        t_start.record(stream)
        for i in range(steps):
            if flush:
                flush_l2()
            step_begin[i].record(stream)
            st = sfd.alspec_graph_launch(graphs[i], stream.cuda_stream)
            assert st == 0
            step_end[i].record(stream)
        t_end.record(stream)
        ranks.barrier()
        nvtx.range_pop()
    per_step = [step_begin[i].elapsed_time(step_end[i]) for i in range(steps)]
    ms_total = sum(per_step) if flush else t_start.elapsed_time(t_end)
    ms_per_step = ranks.max(ms_total / steps)

    # Profiled pass: same step with per-layer events captured in the graphs.
    ranks.barrier()
    nvtx.range_push("profiled pass (per-layer events)")
    with torch.cuda.stream(stream):
        for g in prof_graphs:
            if flush:
                flush_l2()
            assert sfd.alspec_graph_launch(g, stream.cuda_stream) == 0
    ranks.barrier()
    nvtx.range_pop()

    # Latency pass (each replay also timed as a whole).
    ranks.barrier()
    nvtx.range_push("latency pass (kernel time stamps)")
    traces.zero_()
    lat_begin = [torch.cuda.Event(enable_timing=True) for _ in lat]
    lat_end = [torch.cuda.Event(enable_timing=True) for _ in lat]
    with torch.cuda.stream(stream):
        for j, g in enumerate(lat):
            if lat_flush:
                flush_l2()
            lat_begin[j].record(stream)
            assert sfd.alspec_graph_launch(g, stream.cuda_stream) == 0
            lat_end[j].record(stream)
    ranks.barrier()
    nvtx.range_pop()
    lat_ms = [lat_begin[j].elapsed_time(lat_end[j]) / n_lat for j in range(len(lat))]
    tr = traces.cpu().numpy().astype("int64")
    t_spec, t_exact = [], []
    for j in range(prof_steps):
        for i in range(1, n_lat):
            t_spec.append((tr[j, i, 0] - tr[j, i - 1, 1]) * 1e-6)   # ms
            t_exact.append((tr[j, i, 1] - tr[j, i - 1, 1]) * 1e-6)

    # Per-layer profiling events of every profiled step.
    mid_ms, spec_ms, layer_ms, pre_ms, post_ms, gap_ms = [], [], [], [], [], []
    for ev in step_events:
        for i, e in enumerate(ev):
            mid_ms.append(e[2].elapsed_time(e[3]))
            spec_ms.append(e[0].elapsed_time(e[1]))
            layer_ms.append(e[0].elapsed_time(e[4]))
            pre_ms.append(e[0].elapsed_time(e[2]))
            post_ms.append(e[3].elapsed_time(e[4]))
            if i + 1 < len(ev):
                gap_ms.append(e[4].elapsed_time(ev[i + 1][0]))
    hit_rate = float(commit_all[:n_layers].float().mean().item())
    st, err = dec.device_error(stream)
    assert st == 0 and err == 0, f"device error word {err:#x}"

    # End to end through the public API with host buffers: per step, copy the
    # step's query vectors (all layers) and lengths in from pinned memory,
    # replay the step, read every layer's rel_l2 and flag back.
    e2e = None
    if want_e2e:
        in_dev = inputs[:n_layers * in_stride]
        in_host = in_dev.cpu().pin_memory()
        out_host = torch.empty(results.numel(), dtype=torch.uint8).pin_memory()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        ranks.barrier()
        nvtx.range_push("end to end (host buffers)")
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                in_dev.copy_(in_host, non_blocking=True)
                sfd.alspec_graph_launch(graphs[i], stream.cuda_stream)
                out_host.copy_(results, non_blocking=True)
                stream.synchronize()
            e1.record(stream)
        ranks.barrier()
        nvtx.range_pop()
        e2e_ms = ranks.max(e0.elapsed_time(e1) / steps)
        h2d = in_host.numel()
        d2h = out_host.numel()
        e2e = {"value": job_throughput(kv_bytes, ranks.world, e2e_ms), "unit": "GB/s",
               "us_per_step": e2e_ms * 1e3, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "what": "per step: one pinned host-to-device copy of every layer's q and "
                       "seq_lens, the step's graph, one device-to-host read of every layer's "
                       "rel_l2 and commit flag, then a host synchronize; O_spec and O_exact "
                       "stay on the device, where the post-attention ops that consume them run"}

    for g in [warm_graph] + graphs + prof_graphs + lat:
        sfd.alspec_graph_destroy(g)
    lens0 = step_layers[0]["lens"]
    return {
        "plan": plan, "fused": fused, "kv_bytes": kv_bytes, "n_layers": n_layers,
        "ms_per_step": ms_per_step, "per_step": per_step, "flush": flush, "l2_bytes": l2_bytes,
        "mid_ms": mid_ms, "mid_bytes": middle_bytes(wl, lens0, fused), "spec_ms": spec_ms,
        "layer_ms": layer_ms, "pre_ms": pre_ms, "post_ms": post_ms, "gap_ms": gap_ms,
        "t_spec": t_spec, "t_exact": t_exact, "n_lat": n_lat, "lat_ms": lat_ms,
        "lat_flush": lat_flush, "hit_rate": hit_rate, "e2e": e2e, "clocks": clocks.summary(),
        "launches_per_layer": 1 if fused else (3 if plan["n2"] > 0 else 2),
    }


def spec_summary(m):
    ratio = [s / l for s, l in zip(m["t_spec"], m["t_exact"])]
    return {
        "us_median": statistics.median(m["t_spec"]) * 1e3 if m["t_spec"] else None,
        "ratio_to_layer_median": statistics.median(ratio) if ratio else None,
        "layer_us_median": statistics.median(m["t_exact"]) * 1e3 if m["t_exact"] else None,
        "us_p90": statistics.quantiles(m["t_spec"], n=10)[-1] * 1e3
        if len(m["t_spec"]) > 1 else None,
        "from": "kernel-written global-timer stamps: last write of layer l-1's outputs to the "
                "last write of layer l's O_spec (layer: to the last write of its O_exact and "
                "flags); graphs of %d distinct layers, layers 1..%d" % (m["n_lat"], m["n_lat"] - 1),
    }


def config_summary(wl, m, world, peak):
    """One workload's entry in the line's per_config object."""
    value = job_throughput(m["kv_bytes"], world, m["ms_per_step"])
    mid_avg = statistics.mean(m["mid_ms"]) if m["mid_ms"] else None
    mid_gbs = m["mid_bytes"] / (mid_avg * 1e-3) / 1e9 if mid_avg and m["mid_bytes"] else None
    lat_layer_ms = statistics.median(m["lat_ms"])
    return {
        "us_per_step": m["ms_per_step"] * 1e3,
        "us_per_step_p10_p50_p90": quantiles_us(m["per_step"]),
        "steps": len(m["per_step"]),
        "kv_bytes_per_step": m["kv_bytes"],
        "kv_gbs": value,
        "frac": value / world / peak,
        "frac_of_nominal_8000": value / world / NOMINAL_HBM_GBS,
        "us_per_layer_in_graph": lat_layer_ms * 1e3,
        "frac_per_layer_in_graph": (m["kv_bytes"] / m["n_layers"]) / (lat_layer_ms * 1e-3) / 1e9
        / peak,
        "layer_graph": "%d distinct layers per graph%s" % (
            m["n_lat"], ", L2 flushed before each" if m["lat_flush"] else ""),
        "middle_kernel": {"avg_launch_us": mid_avg * 1e3 if mid_avg else None,
                          "bytes_per_launch": m["mid_bytes"], "gbs": mid_gbs,
                          "frac": mid_gbs / peak if mid_gbs else None},
        "spec_latency": spec_summary(m),
        "hit_rate": m["hit_rate"],
        "e2e_us_per_step": m["e2e"]["us_per_step"] if m["e2e"] else None,
        "l2": "flushed before every timed step" if m["flush"] else "inputs larger than L2",
        "plan": m["plan"],
    }


def run_alspec(args, wl):
    import torch
    import workloads

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    ranks = Ranks("nccl", device)
    n_layers = args.layers or wl.n_layers
    m = measure(wl, n_layers, args.steps, args.warmup, device, ranks, args,
                want_e2e=not args.no_e2e)
    torch.cuda.empty_cache()

    # Every other workload, a few timed steps each (the same on every rank).
    peak, peak_kind = measured_peak()
    per_config = None
    if not args.no_per_config and args.layers == 0:
        per_config = {}
        # One clock record over all of them (each one's timed steps are far
        # shorter than the sampling period).
        with ClockSampler(gpu_uuid(device)) as clocks:
            for idx in sorted(workloads.CONFIGS):
                other = workloads.CONFIGS[idx]
                if other.name == wl.name:
                    continue
                mo = measure(other, other.n_layers, args.per_config_steps, max(3, args.warmup),
                             device, ranks, args, want_e2e=not args.no_e2e)
                per_config[other.name] = dict(workload_index=idx,
                                              **config_summary(other, mo, world, peak))
                del mo
                torch.cuda.empty_cache()
        per_config["clocks"] = clocks.summary()
    ranks.close()
    if rank != 0:
        return

    # Same-run read probe: a 4 GiB stream through bulk copies, nothing else.
    probe = read_probe_fn()
    nbytes = 4 << 30
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)
    evp = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        for r in range(7):
            if r == 2:
                evp[0].record(stream)
            assert probe(buf.data_ptr(), nbytes, stream.cuda_stream) == 0
        evp[1].record(stream)
    stream.synchronize()
    probe_gbs = nbytes * 5 / (evp[0].elapsed_time(evp[1]) * 1e-3) / 1e9
    read_probe = {"gbs": probe_gbs, "bytes_per_launch": nbytes, "launches": 5,
                  "library": "libalspec_read_probe.so"}
    del buf

    fused = m["fused"]
    mid_avg_ms = sum(m["mid_ms"]) / len(m["mid_ms"])
    achieved = m["mid_bytes"] / (mid_avg_ms * 1e-3) / 1e9
    traffic = stored_traffic(FUSED_TRAFFIC_FILE if fused else TRAFFIC_FILE, wl.name)
    value = job_throughput(m["kv_bytes"], world, m["ms_per_step"])

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl.replace(n_layers=n_layers), args.cpu_seconds)

    plan = m["plan"]
    l2_bytes = m["l2_bytes"]
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "us_per_step": m["ms_per_step"] * 1e3,
        "us_per_step_p10_p50_p90": quantiles_us(m["per_step"]),
        "frac_of_hbm_peak": value / world / peak,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic",
        "config": workload_config(wl, n_layers, world),
        "method": {
            "kv_bytes_per_step": m["kv_bytes"],
            "l2": ("L2 flushed before every timed step (untimed write of %d MB, then a read "
                   "of %d MB of other data); %.1f MB of KV per step"
                   % (2 * l2_bytes >> 20, 2 * l2_bytes >> 20, m["kv_bytes"] / 1e6))
            if m["flush"] else ("inputs larger than L2: %.1f MB of KV per step against %d MB "
                                "of L2; no flush" % (m["kv_bytes"] / 1e6, l2_bytes >> 20)),
            "timing": "CUDA graph per step, CUDA events on the launch stream; the middle "
                      "kernel's duration from a second pass of graphs with event nodes around "
                      "it (where it starts once the sink-set kernel has completed, so it runs "
                      "alone); O_spec latency from kernel-written time stamps in a third pass",
            "schedule": {1: "streams", 2: "fused", 3: "sink_first"}[plan["schedule"]],
            "plan": plan},
        "roofline": {"bound": "hbm",
                     "kernel": "attn_kernel<%s,%d,%d,%s,%s>" % (
                         wl.dtype, wl.d, wl.g, "fused" if fused else "middle",
                         {1: "cuda_cores", 2: "tensor_cores"}.get(plan["engine"], "?")),
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "bytes_per_launch": m["mid_bytes"], "avg_launch_us": mid_avg_ms * 1e3,
                     "launches_measured": len(m["mid_ms"]), "traffic": traffic,
                     "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                     "frac_of_same_run_read_probe": achieved / probe_gbs},
        "read_probe": read_probe,
        "frac_of_nominal_8000": value / world / NOMINAL_HBM_GBS,
        "spec_latency": dict(spec_summary(m),
                             profiled_graph_us_median=statistics.median(m["spec_ms"]) * 1e3,
                             profiled_graph_layer_us_median=statistics.median(m["layer_ms"]) * 1e3),
        "profiled_pass_us_median": {
            "what": "graphs with event nodes between the kernels (no overlap between them)",
            "start_to_middle_kernel": statistics.median(m["pre_ms"]) * 1e3,
            "middle_kernel": statistics.median(m["mid_ms"]) * 1e3,
            "middle_end_to_layer_end": statistics.median(m["post_ms"]) * 1e3,
            "between_layers": statistics.median(m["gap_ms"]) * 1e3 if m["gap_ms"] else None},
        "hit_rate": m["hit_rate"],
        "cpu_baseline": cpu,
        "e2e": m["e2e"],
        "gpu_launches": args.steps * n_layers * m["launches_per_layer"],
        "clocks": m["clocks"],
        "per_config": per_config,
    }
    print(json.dumps(line), flush=True)


LAMBDA_GRID = (0.0, 1e-4, 2e-4, 5e-4, 1e-3, 2e-3, 5e-3, 1e-2, 2e-2, 5e-2, 0.1, 0.2, 0.5, 1.0)


def run_lambda_sweep(args):
    """Hit rate (share of tokens whose speculative attention output would be
    committed) against the threshold lambda, on the commit-mixing family:
    per layer one decode of a batch of 8 sequences of 24K-32K tokens with
    strong sinks and occasional needles.  The flag is rel_l2 <= lambda, so
    one decode per layer gives the whole curve; the decode at the middle
    threshold checks the device's flags against that rule."""
    import numpy as np
    import torch
    import workloads
    import speculative_flash_decoding_b200 as sfd
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = workloads.COMMIT_VARIANT
    n_layers = args.layers or 8
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=device)
    rel = []
    for layer in range(n_layers):
        data = workloads.make_layer(wl, layer=layer, device=device)
        out = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
        r = out["rel_l2"].cpu().numpy().astype(np.float64)
        flags = out["commit"].cpu().numpy()
        assert (flags == (r <= wl.lam)).all()
        rel.append(r)
        del data
    r = np.concatenate(rel)
    hit = [float((r <= lam).mean()) for lam in LAMBDA_GRID]
    if rank != 0:
        return
    line = {"metric": "hit rate vs lambda (commit-mixing family)", "unit": "fraction of tokens",
            "lambdas": list(LAMBDA_GRID), "hit_rate": hit, "tokens": int(r.size),
            "rel_l2_quantiles": {q: float(np.quantile(r, q)) for q in (0.1, 0.25, 0.5, 0.75, 0.9)},
            "data": "synthetic",
            "config": {"workload": wl.name, "layers": n_layers, "batch": wl.B, "q_heads": wl.Hq,
                       "kv_heads": wl.Hkv, "head_dim": wl.d, "lengths": list(wl.ragged),
                       "sink": wl.S, "window": wl.W, "sink_bump": wl.sink_bump,
                       "needle_bump": wl.needle_bump, "needles": list(wl.needles)}}
    print(json.dumps(line), flush=True)


def run_oproj_bench(args):
    """Latency the speculative output projection hides.  Per layer of the
    32 x 128K step, the projection after attention (Llama-3.1-8B o_proj:
    4096 x 4096 bf16 weights, synthetic) is either run after the merge on
    O_exact (serial) or run on O_spec beside the exact path and redone on
    O_exact only for discarded tokens (speculative: gated by a kernel that
    reads the flags, or by a conditional graph node).  The steps are CUDA
    graphs of 32 layers, each layer after the previous one's projection;
    timed with events, warm-up first.  Two data
    sets: the workload as specified (every token discarded) and the same
    shape with strong sinks and no needles (tokens commit)."""
    import torch
    import workloads
    import speculative_flash_decoding_b200 as sfd
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    base = workloads.CONFIGS[2]
    n_layers = args.layers or base.n_layers
    hidden = 4096
    g = torch.Generator(device="cpu").manual_seed(4242)
    weights = [(torch.randn(hidden, base.Hq * base.d, generator=g) / 64.0).to(torch.bfloat16)
               .to(device) for _ in range(n_layers)]
    results = {}
    # The projection alone: a CUDA graph of back-to-back calls (one per
    # layer's weights, 32 MB each, larger than L2 together); each call's
    # weights start streaming while the call before it finishes.  Beside
    # it, one call on its own after an L2 scrub: launch, ramp and tail
    # included.
    x = torch.randn(base.B, base.Hq * base.d, device=device)
    y = torch.empty(base.B, hidden, device=device)
    st = torch.cuda.Stream(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def call(w):
        assert sfd.alspec_oproj(x.data_ptr(), w.data_ptr(), y.data_ptr(), 0, base.B,
                                base.Hq * base.d, hidden, st.cuda_stream) == 0

    with torch.cuda.stream(st):
        for w in weights:
            call(w)
        assert sfd.alspec_graph_begin(st.cuda_stream) == 0
        for w in weights:
            call(w)
        s_, gr = sfd.alspec_graph_end(st.cuda_stream)
        assert s_ == 0
        for _ in range(3):
            assert sfd.alspec_graph_launch(gr, st.cuda_stream) == 0
        ev[0].record(st)
        for _ in range(4):
            assert sfd.alspec_graph_launch(gr, st.cuda_stream) == 0
        ev[1].record(st)
    st.synchronize()
    us = ev[0].elapsed_time(ev[1]) * 1e3 / (4 * n_layers)
    assert sfd.alspec_graph_destroy(gr) == 0
    # The L2 scrub: a write of twice its size, then a read of another such
    # buffer, so the call does not pay for writing dirty lines back.
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.ones(32 << 20, dtype=torch.int32, device=device)
    sink = torch.empty((), dtype=torch.int64, device=device)
    # Everything is queued before the first scrub ends, so no call waits
    # for the host.
    iso_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(13)]
    with torch.cuda.stream(st):
        for i, (e0, e1) in enumerate(iso_ev):
            scrub.zero_()
            torch.sum(clean, dim=0, out=sink)
            e0.record(st)
            call(weights[i % n_layers])
            e1.record(st)
    st.synchronize()
    iso = [e0.elapsed_time(e1) * 1e3 for e0, e1 in iso_ev[3:]]
    del scrub, clean, sink
    us_iso = statistics.median(iso)
    w_bytes = hidden * base.Hq * base.d * 2
    peak, peak_kind = measured_peak()
    results["oproj_alone"] = {"us_per_call": us, "weight_bytes": w_bytes,
                              "gbs": w_bytes / (us * 1e-6) / 1e9,
                              "frac_of_hbm_peak": w_bytes / (us * 1e-6) / 1e9 / peak,
                              "peak_kind": peak_kind,
                              "timing": f"graph of {n_layers} back-to-back calls, 4 launches",
                              "one_call_us": us_iso,
                              "one_call_frac_of_hbm_peak": w_bytes / (us_iso * 1e-6) / 1e9 / peak}
    for tag, wl in (("as_specified", base),
                    ("strong_sinks_no_needles", base.replace(sink_bump=24.0, needles=("none",)))):
        layers = [workloads.make_layer(wl, layer=i, device=device) for i in range(n_layers)]
        dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=device)
        outs = []
        for _ in range(n_layers):
            o = dec.alloc_outputs()
            o["y"] = torch.empty(wl.B, hidden, device=device)
            outs.append(o)
        stream = torch.cuda.Stream(device)
        kdim = wl.Hq * wl.d
        with torch.cuda.stream(stream):
            for d, o in zip(layers, outs):   # creates the library's stream and events
                dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=o, stream=stream)
        stream.synchronize()

        def capture(speculative):
            with torch.cuda.stream(stream):
                assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
                for d, o, w in zip(layers, outs, weights):
                    if speculative:
                        dec.decode_oproj(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, w,
                                         out=o, stream=stream, gate=speculative)
                    else:
                        dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=o,
                                   stream=stream)
                        assert sfd.alspec_oproj(o["out_exact"].data_ptr(), w.data_ptr(),
                                                o["y"].data_ptr(), 0, wl.B, kdim, hidden,
                                                stream.cuda_stream) == 0
                st, gr = sfd.alspec_graph_end(stream.cuda_stream)
                assert st == 0
            return gr

        res = {}
        for name, spec in (("serial", False), ("speculative", "kernel"),
                           ("speculative_graph_conditional", "graph_conditional")):
            gr = capture(spec)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            with torch.cuda.stream(stream):
                for _ in range(max(3, args.warmup)):
                    assert sfd.alspec_graph_launch(gr, stream.cuda_stream) == 0
                ev[0].record(stream)
                for _ in range(args.steps):
                    assert sfd.alspec_graph_launch(gr, stream.cuda_stream) == 0
                ev[1].record(stream)
            stream.synchronize()
            ms = ev[0].elapsed_time(ev[1]) / args.steps
            res[name] = {"us_per_step": ms * 1e3, "us_per_layer": ms * 1e3 / n_layers}
            hit = float(torch.stack([o["commit"].float().mean() for o in outs]).mean().item())
            assert sfd.alspec_graph_destroy(gr) == 0
        res["hit_rate"] = hit
        res["hidden_us_per_layer"] = (res["serial"]["us_per_layer"] -
                                      res["speculative"]["us_per_layer"])
        results[tag] = res
        del layers, outs
        torch.cuda.empty_cache()
    if rank != 0:
        return
    line = {"metric": "per-layer latency to the output projection's result, serial vs "
                      "speculative", "unit": "us", "higher_is_better": False,
            "steps": args.steps, "data": "synthetic",
            "config": {"workload": base.name, "layers": n_layers, "hidden": hidden,
                       "weights": "bf16 [4096, 4096] per layer, N(0, 1/64^2)"},
            "results": results}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    import workloads
    wl = workloads.CONFIGS[args.config]
    if args.lambda_sweep:
        run_lambda_sweep(args)
    elif args.oproj:
        run_oproj_bench(args)
    elif args.impl == "reference":
        run_reference(args, wl)
    else:
        run_alspec(args, wl)


if __name__ == "__main__":
    main()
