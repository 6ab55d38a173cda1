#!/usr/bin/env python
"""Benchmark of the SSD forward pass on the Mamba-2 2.7B-shaped layer.

Workload: B=4, L=4096, H=80 heads, P=64, N=128, G=1, chunk 256, bf16 I/O,
seeded synthetic inputs (selective_state_space_17_b200.inputs). A step is one
ssd_forward call over the whole batch (all steps of the chunked algorithm).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0. ``value`` is Mtokens/s over all ranks (tokens
= B*L per rank per step; every rank runs its own copy of the layer: the work
shards by batch and head with no data-path collective, so scaling is weak).
Timing: CUDA events on the launching stream around each step, L2 flushed
between steps outside the events (a 256 MiB write, then a 256 MiB read so that
no dirty line is written back inside the next step), max over ranks.
``--impl reference`` times the fp64 CPU oracle on the host cores instead
(rank 0 only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
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

from selective_state_space_17_b200 import inputs as gen  # noqa: E402

METRIC = "SSD fwd Mtokens/s per layer on 1 B200; % of HBM/tensor-core roofline"
UNIT = "Mtokens/s"
WORKLOAD = gen.LAYER_2P7B
# other configurations of the same layer, selectable with --workload (the
# default is the one the metric is quoted on)
WORKLOADS = {"2.7b": gen.LAYER_2P7B, "370m": gen.LAYER_370M, "long": gen.LONG_CONTEXT}
WORKLOADS.update({f"sweep-n{w.N}-q{w.chunk}": w for w in gen.sweep_workloads()})
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Leaves the L2 cold and clean between timed steps: a write of a buffer
    larger than the L2 evicts everything, and a read of a second such buffer
    then evicts the written (dirty) lines, so their write-back happens here
    instead of inside the next timed step."""

    def __init__(self, dev, nbytes=L2_FLUSH_BYTES):
        import torch
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.r = torch.ones(nbytes, dtype=torch.uint8, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dtype=torch.int64)


def compulsory_bytes(w: gen.Workload) -> int:
    """x and y in the I/O dtype, dt, Bm and Cm once per group, final_state,
    A and D: every byte the layer must read or write at least once."""
    es = 2 if w.dtype == "bf16" else 4
    BL = w.B * w.L
    return (2 * BL * w.H * w.P * es + BL * w.H * 4 + 2 * BL * w.G * w.N * es
            + w.B * w.H * w.P * w.N * 4 + 2 * w.H * 4)


def algorithmic_flops(w: gen.Workload) -> int:
    """Per token and head: Q*P (causal half of the chunk's masked product with
    X) + 4*N*P (chunk states and the state read-out); per token and group:
    Q*N (causal half of C B^T)."""
    BL = w.B * w.L
    return BL * w.H * (w.chunk * w.P + 4 * w.N * w.P) + BL * w.G * w.chunk * w.N


def combine_ranks(local_ms: float, tokens_per_rank: int, world: int, dist=None, device=None):
    """Max of the per-rank step times (the slowest rank bounds the job) and the
    whole-job throughput in Mtokens/s. Only timings cross ranks; no data does."""
    import torch
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    return ms, tokens_per_rank * world / (ms / 1e3) / 1e6


def code_digest(paths) -> str:
    """sha256 over the given C/C++/CUDA sources with comments removed and
    whitespace collapsed: it changes with the code and not with its comments."""
    import hashlib
    h = hashlib.sha256()
    for path in paths:
        with open(os.path.join(ROOT, path), encoding="utf-8") as f:
            text = f.read()
        out, i, n = [], 0, len(text)
        while i < n:
            c = text[i]
            if text.startswith("//", i):
                j = text.find("\n", i)
                i = n if j < 0 else j
            elif text.startswith("/*", i):
                j = text.find("*/", i + 2)
                i = n if j < 0 else j + 2
                out.append(" ")
            elif c in "\"'":
                j = i + 1
                while j < n and text[j] != c:
                    j += 2 if text[j] == "\\" else 1
                out.append(text[i:j + 1])
                i = j + 1
            else:
                out.append(c)
                i += 1
        h.update(" ".join("".join(out).split()).encode())
        h.update(b"\0")
    return h.hexdigest()


# The forward kernel that one ssd_forward call runs, by ssd_forward_path.
KERNEL_OF_PATH = {1: "SIMT forward kernels", 2: "tc_forward_kernel",
                  3: "tc_forward_kernel (segment-parallel) + segment_scan_kernel",
                  4: "grouped_forward_kernel"}


def recorded_traffic(workload: str):
    """DRAM bytes (read + write) of one launch from the ncu capture recorded in
    profiles/traffic.json, or None when the kernel's code (its sources without
    comments) has changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(workload)
        if not rec:
            return None
        if code_digest(rec["sources"]) != rec["code_digest"]:
            return None
        return rec["traffic_bytes"]
    except (OSError, ValueError, KeyError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), max=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}
        reasons = set()
        for r in rows:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        loaded = [r["sm"] for r in rows if r["power"] > 200.0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle_sample(w: gen.Workload, inp, heads: int, min_seconds: float, threads=None):
    """Run the fp64 oracle on batch row 0, the first `heads` heads (their
    groups whole), full sequence; repeat until min_seconds. Returns
    (Mtokens/s-equivalent, threads, sample description, seconds)."""
    import oracle
    hpg = w.H // w.G
    if w.G > 1:  # keep whole groups so that B and C slices stay shared
        heads = max(hpg, (heads // hpg) * hpg)
    heads = min(heads, w.H)
    x, dt, A, Bm, Cm, D = inp.f64(0, 1, heads=(0, heads))
    threads = min(threads or oracle.default_threads(), heads)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(x, dt, A, Bm, Cm, D, nthreads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    tokens_equiv = reps * w.L * heads / w.H  # a full-layer token needs all H heads
    sample = (f"batch row 0 of {w.B}, heads 0..{heads - 1} of {w.H}, all {w.L} tokens, "
              f"{reps} run(s); tokens counted as L*heads/H")
    return tokens_equiv / el / 1e6, threads, sample, el


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = args.workload
    inp = w.make(0)
    per_step = []
    info = None
    for i in range(args.warmup + args.steps):
        v, threads, sample, el = time_oracle_sample(w, inp, heads=8, min_seconds=0.0)
        if i >= args.warmup:
            per_step.append(el)
            info = (threads, sample)
    tokens_equiv = w.L * 8 / w.H
    ms = statistics.mean(per_step) * 1e3
    value = tokens_equiv / (ms / 1e3) / 1e6
    threads, sample = info
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "global_batch": w.B, "seq_len": w.L,
                                        "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "per step: " + sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    from selective_state_space_17_b200 import ssd

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    w = args.workload
    inp = w.make(seed=rank)
    code = ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32

    def io(a):
        if w.dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(a)

    host = dict(x=io(inp.x), dt=torch.from_numpy(inp.dt), A=torch.from_numpy(inp.A),
                Bm=io(inp.Bm), Cm=io(inp.Cm), D=torch.from_numpy(inp.D))
    d = {k: v.to(dev) for k, v in host.items()}
    y = torch.empty_like(d["x"])
    fs = torch.empty((w.B, w.H, w.P, w.N), dtype=torch.float32, device=dev)
    ws = torch.zeros(ssd.workspace_size(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code),
                     dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        ssd.forward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], d["D"], chunk=w.chunk, y=y,
                    final_state=fs, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        flush()
        step()
    ssd.poll_status(stream)
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        barrier()
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        barrier()
    ssd.poll_status(stream)
    per_step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms, _ = combine_ranks(statistics.mean(per_step_ms), w.tokens, world, dist, dev)
    decode = time_decode(ssd, dev, flush, args.warmup, args.steps, world, dist)
    workloads = None
    if not args.no_workloads:
        workloads = [time_workload(ssd, v, dev, flush, 3, args.steps, world, dist)
                     for v in secondary_workloads() if v.name != w.name]
        torch.cuda.empty_cache()

    # end to end through the host-buffer entry point: H2D inputs, forward, D2H y + state
    if args.no_e2e:
        return _report(args, w, rank, world, ms, per_step_ms, clk, inp, None, host, ssd, code, dist,
                       decode, workloads)
    pin = {k: v.pin_memory() for k, v in host.items()}
    y_host = torch.empty_like(host["x"]).pin_memory()
    fs_host = torch.empty((w.B, w.H, w.P, w.N), dtype=torch.float32).pin_memory()
    dbuf = torch.zeros(ssd.forward_host_buffer_size(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code),
                       dtype=torch.uint8, device=dev)
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_step():
        ssd.forward_host(pin["x"], pin["dt"], pin["A"], pin["Bm"], pin["Cm"], pin["D"], y_host,
                         fs_host, chunk=w.chunk, device_buffer=dbuf, stream=stream)

    for _ in range(2):
        e2e_step()
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e_end.record(stream)
    barrier()
    e2e_ms, _ = combine_ranks(e_start.elapsed_time(e_end) / e2e_steps, w.tokens, world, dist, dev)
    return _report(args, w, rank, world, ms, per_step_ms, clk, inp, e2e_ms, host, ssd, code, dist,
                   decode, workloads)


def device_inputs(w: gen.Workload, seed: int, dev):
    """Inputs of the recipe in inputs.make_inputs (x ~ N(0,1); dt = exp(U[ln 1e-3,
    ln 1e-1]); A = -exp(U[0, ln 16]); Bm, Cm ~ N(0,1)/sqrt(N); D ~ N(0,1); the
    a = 1 and a = 0.99 kinds with dt = 1), drawn on the GPU with torch's seeded
    generator and rounded once to the I/O dtype. Used for the secondary
    workloads, whose timing needs their shapes and distributions; the headline
    workload uses the numpy sample the parity tests check."""
    import torch
    g = torch.Generator(device=dev).manual_seed(1000 + seed)
    io = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x = torch.randn(w.B, w.L, w.H, w.P, device=dev, generator=g).to(io)
    dt = torch.exp(torch.empty(w.B, w.L, w.H, device=dev).uniform_(
        float(np.log(1e-3)), float(np.log(1e-1)), generator=g))
    A = -torch.exp(torch.empty(w.H, device=dev).uniform_(0.0, float(np.log(16.0)), generator=g))
    Bm = (torch.randn(w.B, w.L, w.G, w.N, device=dev, generator=g) / w.N ** 0.5).to(io)
    Cm = (torch.randn(w.B, w.L, w.G, w.N, device=dev, generator=g) / w.N ** 0.5).to(io)
    D = torch.randn(w.H, device=dev, generator=g)
    if w.kind in ("linear_attention", "retnet"):
        dt.fill_(1.0)
        A.fill_(0.0 if w.kind == "linear_attention" else float(np.log(0.99)))
    return dict(x=x, dt=dt, A=A, Bm=Bm, Cm=Cm, D=D)


def secondary_workloads():
    """The other configurations of the layer: the 370M-shaped layer, the long
    context, the state-size / grouping sweep and its a = 1 and a = 0.99 runs."""
    ws = [gen.LAYER_370M, gen.LONG_CONTEXT] + gen.sweep_workloads()
    ws += [v for v in gen.sweep_workloads(("linear_attention", "retnet")) if " N128 Q256" in v.name]
    return ws


def time_workload(ssd, w: gen.Workload, dev, flush, warmup, steps, world, dist):
    """One secondary workload, timed like the headline: L2 flushed between steps
    outside the events, the mean of `steps` steps, max over ranks."""
    import torch
    d = device_inputs(w, 0, dev)
    code = ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32
    y = torch.empty_like(d["x"])
    fs = torch.empty((w.B, w.H, w.P, w.N), dtype=torch.float32, device=dev)
    ws = torch.zeros(ssd.workspace_size(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ssd.forward(d["x"], d["dt"], d["A"], d["Bm"], d["Cm"], d["D"], chunk=w.chunk, y=y,
                    final_state=fs, workspace=ws, stream=stream)

    for _ in range(warmup):
        flush()
        step()
    times = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        times.append((e0, e1))
    ssd.poll_status(stream)
    ms, value = combine_ranks(statistics.mean(a.elapsed_time(b) for a, b in times), w.tokens,
                              world, dist, dev)
    hbm_peak, tc_peak, _ = measured_peaks()
    t_roof = max(compulsory_bytes(w) / (hbm_peak * 1e9), algorithmic_flops(w) / (tc_peak * 1e12))
    return {"workload": w.name, "ms_per_step": ms, "value": value, "unit": UNIT,
            "roofline_frac": t_roof * 1e3 / ms,
            "path": ssd.forward_path(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code),
            "launches_per_step": ssd.kernel_count(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code)}


def time_decode(ssd, dev, flush, warmup, steps, world, dist, rotate=4):
    """ssd_step on the decode workload (one token for each of B sequences from a
    random fp32 state). The steps run back to back over `rotate` independent
    states (several layers' worth, 4 x 67 MB, twice the L2), all timed by one
    pair of events: each step's state write-back is evicted, and so paid for,
    inside the timed region (a flush between steps would pay it outside)."""
    import torch
    d = gen.DECODE
    s = gen.make_step_inputs(d["B"], d["H"], d["P"], d["G"], d["N"], d["dtype"], seed=5)
    io = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    x, Bm, Cm = io(s.x), io(s.Bm), io(s.Cm)
    dt, A, D = (torch.from_numpy(v).to(dev) for v in (s.dt, s.A, s.D))
    states = [torch.from_numpy(s.state).to(dev) for _ in range(rotate)]
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    n = max(steps, 4 * rotate)
    for i in range(max(warmup, rotate)):
        ssd.step(x, dt, A, Bm, Cm, D, states[i % rotate], y=y, stream=stream)
    flush()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        ssd.step(x, dt, A, Bm, Cm, D, states[i % rotate], y=y, stream=stream)
    e1.record(stream)
    ssd.poll_status(stream)
    ms, _ = combine_ranks(e0.elapsed_time(e1) / n, d["B"], world, dist, dev)
    nbytes = (2 * d["B"] * d["H"] * d["P"] * d["N"] * 4 + 2 * d["B"] * d["H"] * d["P"] * 2
              + d["B"] * d["H"] * 4 + 2 * d["B"] * d["G"] * d["N"] * 2 + 2 * d["H"] * 4)
    return {"workload": d["name"], "ms_per_step": ms,
            "value": d["B"] * world / (ms / 1e3) / 1e6, "unit": "Mtokens/s",
            "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / (ms / 1e3) / 1e9,
            "timing": f"{n} steps back to back over {rotate} independent states "
                      f"({rotate * d['B'] * d['H'] * d['P'] * d['N'] * 4 >> 20} MiB), one event pair"}


def _report(args, w, rank, world, ms, per_step_ms, clk, inp, e2e_ms, host, ssd, code, dist,
            decode=None, workloads=None):
    tokens_all = w.tokens * world
    value = tokens_all / (ms / 1e3) / 1e6
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host["x"].numel() * host["x"].element_size() + w.B * w.H * w.P * w.N * 4

    hbm_peak, tc_peak, peak_kind = measured_peaks()
    nbytes = compulsory_bytes(w)
    flops = algorithmic_flops(w)
    kernel_ms = ms  # one ssd_forward call: its kernels back to back
    achieved_gbs = nbytes / (kernel_ms / 1e3) / 1e9
    achieved_tflops = flops / (kernel_ms / 1e3) / 1e12
    t_hbm = nbytes / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    launches = ssd.kernel_count(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code)
    traffic = recorded_traffic(w.name)
    kernel = KERNEL_OF_PATH.get(ssd.forward_path(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, code), "?")

    result = None
    if rank == 0:
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; see inputs.py)",
            "config": {"workload": w.name, "global_batch": w.B * world, "seq_len": w.L,
                       "heads": w.H, "headdim": w.P, "d_state": w.N, "groups": w.G,
                       "chunk": w.chunk, "parallelism": f"replicas x{world} (batch/head shards)",
                       "l2": "flushed between steps (256 MiB write, then 256 MiB read, outside the events)"},
            "roofline": {"kernel": kernel, "bound": bound,
                         "achieved": achieved_gbs if bound == "hbm" else achieved_tflops,
                         "peak": hbm_peak if bound == "hbm" else tc_peak,
                         "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                         "frac": (achieved_gbs / hbm_peak) if bound == "hbm" else (achieved_tflops / tc_peak),
                         "traffic": traffic, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback",
                         "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                         "achieved_tflops": achieved_tflops,
                         "roofline_ms": max(t_hbm, t_tc) * 1e3,
                         "roofline_frac": max(t_hbm, t_tc) * 1e3 / kernel_ms},
            "clocks": clk.summary(),
            "e2e": None if e2e_ms is None else {
                "value": tokens_all / (e2e_ms / 1e3) / 1e6, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "api": "ssd_forward_host (pinned host buffers)"},
            "gpu_launches": launches * args.steps,
            "decode": None if decode is None else dict(
                decode, frac=decode["achieved_gbs"] / hbm_peak, bound="hbm",
                peak=hbm_peak, peak_unit="GB/s"),
            "per_step_ms": {"min": min(per_step_ms), "median": statistics.median(per_step_ms),
                            "max": max(per_step_ms)},
            "workloads": workloads,
        }
        if world == 1 and not args.no_cpu_baseline:
            v, threads, sample, el = time_oracle_sample(w, inp, heads=16, min_seconds=10.0)
            v1, _, sample1, el1 = time_oracle_sample(w, inp, heads=1, min_seconds=5.0, threads=1)
            result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads,
                                      "kind": "oracle", "sample": sample,
                                      "seconds": round(el, 2), "cpu_model": cpu_model(),
                                      "nproc": os.cpu_count(),
                                      "one_core": {"value": v1, "unit": UNIT, "cores": 1,
                                                   "sample": sample1, "seconds": round(el1, 2)}}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing on the host cores")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end timing (used for profiling runs)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the secondary workloads (370M, long context, sweep)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="2.7b",
                    help="layer configuration (default: the 2.7B-shaped layer)")
    args = ap.parse_args()
    args.workload = WORKLOADS[args.workload]
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps, reported as run
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
