"""Benchmark of the routed-expert MoE prefill layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline] [--no-graph]

A step is one pass of the whole layer (route, group, gate/up decode-GEMM +
SwiGLU, down decode-GEMM, combine) over one chunk of synthetic input, through
the library's C ABI (rl_moe_prefill_ws).  Default workload: the 2,048-token
chunk, H=2048, I=512, 512 experts, top-10, format Q2 (20,480 pairs).  The L2
is flushed (a 256 MB device write) before every timed step; each step is timed
with CUDA events on the launching stream.  The metric is routed pairs/s (the
layer's ms per step is in ms_per_step).  A second timed pass records the
library's CUDA events between its kernels for the stage times and the gate/up
kernel's duration (the roofline figure).  The line also carries the same call
replayed from a CUDA graph captured once (graph_replay), the end-to-end
figure with host copies every step (e2e), and (one GPU) the other four
workloads timed the same way (per_workload).

Multi-GPU: the layer does not shard (one GPU per layer call), so --gpus N runs
N independent replicas, one process per GPU under torchrun; value is the pairs
of all ranks divided by the slowest rank's time (scaling "weak").

--impl reference times the float64 C++ oracle, single-threaded on a host
core, each step a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_routed_expert_top_b200 import synth  # noqa: E402

METRIC = "ms/layer & routed pairs/s at 2048 tok, 512 experts top-10; % of roofline"
UNIT = "pairs/s"
FLUSH_BYTES = 256 << 20
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def layer_model(wl, touched_experts: int):
    """Algorithmic FLOPs and bytes of the layer and of its gate/up stage."""
    P = wl.T * wl.k
    flops = 6.0 * wl.H * wl.I * P
    flops_gu = 4.0 * wl.H * wl.I * P
    eb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
    bytes_w = touched_experts * eb
    act = 2.0 * wl.T * wl.H + 4.0 * wl.T * wl.E + 4.0 * wl.T * wl.H
    return dict(flops=flops, flops_gu=flops_gu, bytes=bytes_w + act,
                bytes_gu=touched_experts * eb * 2 / 3 + 2.0 * wl.T * wl.H)


def source_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def read_traffic(kernel_file):
    """dram bytes per launch of the gate/up kernel from the committed ncu
    summary, or None when the kernel source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "gateup_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha256_16") != source_hash(kernel_file):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = str(gpu_index)
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.gpu], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def max_over_ranks(x, world, device=None):
    """Max of a per-rank number over all ranks (every rank calls it at the
    same point, so it is also how an error on one rank reaches the others)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, steps, units_per_step, max_ms):
    """Whole-job units/s of `world` replicas, each doing `units_per_step`
    per step, timed by the slowest rank's total over `steps` steps."""
    return world * steps * units_per_step / (max_ms * 1e-3)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    return world, rank, local


def oracle_host():
    """The oracle's thread count (it is single-threaded) and this host."""
    from oracle import moe_oracle as O
    model = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return 1, f"{model}, {O.hardware_concurrency()} hardware threads"


def bench_reference(args, wl, world, rank):
    """The float64 C++ oracle as it stands, single-threaded on a host core
    (rank 0 only); each step's time is the oracle's own std::chrono figure."""
    if rank != 0:
        return
    from oracle import moe_oracle as O
    cores, host = oracle_host()
    inp = synth.make_inputs(wl)
    nb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    ntok = 2 if wl.T >= 2 else 1
    rng = np.random.default_rng(0)

    def step():
        toks = rng.integers(0, wl.T, ntok)
        return O.moe_prefill_tokens_timed(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, toks)[3]

    for _ in range(args.warmup):
        step()
    dt = sum(step() for _ in range(args.steps))
    value = args.steps * ntok * wl.k / dt
    sample = (f"{ntok} tokens x top-{wl.k} of the {wl.name} workload per step (routing, decode of "
              f"the selected experts, float64 FFN, ordered combine), {args.steps} steps; "
              f"single-threaded C++ oracle on {host}")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
                       "format": synth.FMT_NAMES[wl.fmt]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, budget_s=15.0):
    """The C++ oracle on a bounded sample of the workload, single-threaded;
    the time is the sum of the oracle's own std::chrono figures."""
    from oracle import moe_oracle as O
    cores, host = oracle_host()
    inp = synth.make_inputs(wl)
    nb = synth.expert_bytes(wl.fmt, wl.H, wl.I)
    blobs = [inp.blobs[e, :nb] for e in range(wl.E)]
    rng = np.random.default_rng(1)
    done = 0
    dt = 0.0
    while dt < budget_s:
        toks = rng.integers(0, wl.T, 2)
        dt += O.moe_prefill_tokens_timed(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, toks)[3]
        done += 2
    out = {"value": done * wl.k / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"{done} tokens ({done * wl.k} pairs) of {wl.name}, {dt:.1f} s, float64, "
                     f"single-threaded C++ oracle on {host}"}
    try:
        out["all_cores"] = oracle_all_cores(wl, inp, blobs, budget_s=budget_s / 2)
    except Exception as e:  # noqa: BLE001 - an optional figure; the single-thread one stands
        out["all_cores"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    return out


def oracle_all_cores(wl, inp, blobs, budget_s=7.5, threads=None):
    """The same oracle partitioned by token over every host thread: each
    thread runs 2-token calls (the C++ call releases the interpreter lock)
    until its own std::chrono time reaches the budget; the figure is all
    threads' pairs over the wall time.  Each token's result does not depend
    on which thread computes it."""
    import concurrent.futures as cf

    from oracle import moe_oracle as O
    # the CPUs this process may run on, at most 32 (each call holds ~25 MB
    # of decoded expert weights)
    n = threads or max(1, min(len(os.sched_getaffinity(0)), 32))

    def work(seed):
        rng = np.random.default_rng(seed)
        done, t = 0, 0.0
        while t < budget_s:
            toks = rng.integers(0, wl.T, 2)
            t += O.moe_prefill_tokens_timed(inp.x_bits, inp.logits, blobs, wl.fmt, wl.H, wl.I, wl.k, toks)[3]
            done += 2
        return done

    wall0 = time.perf_counter()
    with cf.ThreadPoolExecutor(n) as ex:
        done = sum(ex.map(work, range(100, 100 + n)))
    wall = time.perf_counter() - wall0
    return {"value": done * wl.k / wall, "unit": UNIT, "cores": n,
            "sample": f"{done} tokens on {n} threads, {wall:.1f} s wall"}


def touched_experts(api, torch, logits, wl, ws, dev):
    """Experts with at least one pair (the byte count of the roofline), from
    the library's own routing export."""
    P = wl.T * wl.k
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
    w_ = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
    off = torch.empty(wl.E + 1, dtype=torch.int32, device=dev)
    pl = torch.empty(P, dtype=torch.int32, device=dev)
    pp = torch.empty(P, dtype=torch.int32, device=dev)
    api.rl_moe_route(logits, wl.T, wl.E, wl.k, idx, w_, off, pl, pp, ws)
    return int((torch.diff(off) > 0).sum().item())


def per_workload_figures(args, dev, flush, headline):
    """The other workloads of the layer, each timed like the headline (L2
    flushed before every step, CUDA events around each call on the launching
    stream) and replayed from a CUDA graph: median ms per call, routed
    pairs/s, and the fraction of its own roofline."""
    import torch
    from bit_routed_expert_top_b200 import api

    peaks, _ = load_peaks()
    stream = torch.cuda.current_stream(dev)
    out = {}
    for wl in synth.WORKLOADS:
        if wl.name == headline:
            continue
        inp = synth.make_inputs(wl)
        x = torch.from_numpy(inp.x_bits.view(np.int16).copy()).to(dev)
        logits = torch.from_numpy(inp.logits).to(dev)
        blobs = torch.from_numpy(inp.blobs).to(dev)
        table = api.expert_table(blobs, wl.E)
        y = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
        ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, device=dev)

        def call(s=stream):
            api.rl_moe_prefill_ws(x, logits, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws, s)

        def timed(fn):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for i in range(args.warmup):
                flush.fill_(float(i))
                fn()
            for i, (a, b) in enumerate(ev):
                flush.fill_(float(i))
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            return [a.elapsed_time(b) for a, b in ev]

        ms = timed(call)
        bits = api.rl_moe_check_status(ws, stream)
        if bits:
            raise SystemExit(f"device status 0x{bits:x} on {wl.name}: {api.rl_last_error()}")
        graph_ms = None
        if not args.no_graph:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
                    call(side)
            torch.cuda.synchronize()
            graph_ms = statistics.median(timed(g.replay))
            del g
        touched = touched_experts(api, torch, logits, wl, ws, dev)
        model = layer_model(wl, touched)
        t_roof = max(model["flops"] / (peaks["bf16_tflops"] * 1e12), model["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
        med = statistics.median(ms)
        out[wl.name] = {"T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "format": synth.FMT_NAMES[wl.fmt],
                        "ms_median": med, "ms_mean": statistics.mean(ms), "pairs_per_s": wl.T * wl.k / (med * 1e-3),
                        "touched_experts": touched, "t_roof_ms": t_roof, "layer_roofline_frac": t_roof / med,
                        "graph_replay_ms_median": graph_ms,
                        "graph_layer_roofline_frac": t_roof / graph_ms if graph_ms else None}
        del x, logits, blobs, y, ws
        torch.cuda.empty_cache()
    return out


def router_gemm_figure(args, dev, flush, wl):
    """The router projection (x [T, H] times W_r [E, H] transposed, bf16 in,
    fp32 out) at the workload's shape: median ms over the timed steps (L2
    flushed before each), TFLOP/s and the fraction of the bf16 peak."""
    import torch
    from bit_routed_expert_top_b200 import api

    peaks, src = load_peaks()
    rng = np.random.default_rng(5)
    x = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((wl.T, wl.H), dtype=np.float32))
                         .view(np.int16).copy()).to(dev)
    w = torch.from_numpy(synth.router_weights(wl.E, wl.H, seed=6).view(np.int16).copy()).to(dev)
    logits = torch.empty((wl.T, wl.E), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.warmup):
        flush.fill_(float(i))
        api.rl_moe_router_logits(x, w, wl.T, wl.H, wl.E, logits)
    for i, (a, b) in enumerate(ev):
        flush.fill_(float(i))
        a.record(stream)
        api.rl_moe_router_logits(x, w, wl.T, wl.H, wl.E, logits)
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    tf = 2.0 * wl.T * wl.H * wl.E / (ms * 1e-3) / 1e12
    # the whole layer from x and W_r (router launch, then the layer from its
    # logits)
    inp = synth.make_inputs(wl)
    blobs = torch.from_numpy(inp.blobs).to(dev)
    table = api.expert_table(blobs, wl.E)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
    ws = torch.empty(api.rl_moe_router_workspace_bytes(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k), dtype=torch.uint8,
                     device=dev)
    for i in range(args.warmup):
        flush.fill_(float(i))
        api.rl_moe_prefill_router_ws(x, w, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    for i, (a, b) in enumerate(ev):
        flush.fill_(float(i))
        a.record(stream)
        api.rl_moe_prefill_router_ws(x, w, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
        b.record(stream)
    torch.cuda.synchronize()
    layer_ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    if api.rl_moe_check_status(ws) != 0:
        raise RuntimeError("router layer: device status " + api.rl_last_error())
    return {"T": wl.T, "H": wl.H, "E": wl.E, "ms_median": ms, "tflops": tf, "peak": peaks["bf16_tflops"],
            "frac": tf / peaks["bf16_tflops"], "peak_source": f"{src} bf16 dense, burst",
            "layer_from_x_ms_median": layer_ms,
            "layer_from_x_method": "rl_moe_prefill_router_ws: router GEMM, then the layer from its logits (routing, "
                                   "grouping, decode-GEMMs, combine); median of the timed steps"}


def shared_expert_figure(args, dev, flush, wl):
    """The layer with a shared expert (rl_moe_prefill_shared_ws: every token
    picks the shared expert last, weight 1) at the workload's shape, the
    shared blob at the routed experts' stride: median ms over the timed
    steps (L2 flushed before each), pairs/s over T*(k+1) pairs and the
    fraction of its roofline (FLOPs and bytes of k+1 picks per token)."""
    import torch
    from bit_routed_expert_top_b200 import api

    peaks, _ = load_peaks()
    wl1 = synth.Workload(wl.name, wl.T, wl.H, wl.I, wl.E + 1, wl.k, wl.fmt, wl.skew)
    inp = synth.make_inputs(wl1)
    x = torch.from_numpy(inp.x_bits.view(np.int16).copy()).to(dev)
    logits = torch.from_numpy(np.ascontiguousarray(inp.logits[:, :wl.E])).to(dev)
    blobs = torch.from_numpy(inp.blobs).to(dev)
    table = api.expert_table(blobs, wl.E)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
    ws = api.alloc_shared_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.warmup):
        flush.fill_(float(i))
        api.rl_moe_prefill_shared_ws(x, logits, table, blobs[wl.E], wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
    for i, (a, b) in enumerate(ev):
        flush.fill_(float(i))
        a.record(stream)
        api.rl_moe_prefill_shared_ws(x, logits, table, blobs[wl.E], wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws)
        b.record(stream)
    torch.cuda.synchronize()
    if api.rl_moe_check_status(ws) != 0:
        raise RuntimeError("shared-expert layer: device status " + api.rl_last_error())
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    top = np.argsort(-inp.logits[:, :wl.E], axis=1, kind="stable")[:, :wl.k]
    touched = int(np.unique(top).size) + 1
    wlk = synth.Workload(wl.name, wl.T, wl.H, wl.I, wl.E, wl.k + 1, wl.fmt, wl.skew)
    model = layer_model(wlk, touched)
    t_roof = max(model["flops"] / (peaks["bf16_tflops"] * 1e12), model["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    P = wl.T * (wl.k + 1)
    return {"T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k, "pairs": P, "ms_median": ms,
            "pairs_per_s": P / (ms * 1e-3), "t_roof_ms": t_roof, "layer_roofline_frac": t_roof / ms,
            "method": "rl_moe_prefill_shared_ws, the shared blob at the routed experts' stride; median of the "
                      "timed steps, L2 flushed before each"}


def expert_cache_figure(args, dev, flush):
    """Bounded verify steps (rl_moe_verify_bounded) at the 2-token verify
    shape on a cache of 64 of the 512 experts filled from pinned host memory:
    per step new router logits (new selections: misses are copied host ->
    device inside the step) and, separately, steps that repeat the previous
    step's selections (every expert resident).  Device time per step (CUDA
    events; the step reads its selections back to the host in between),
    misses and bytes copied per step, and a plain pinned host -> device copy
    of 64 MB as the copy bandwidth reference."""
    import torch
    from bit_routed_expert_top_b200 import api

    wl = [w for w in synth.WORKLOADS if w.name == "verify2"][0]
    base = synth.make_inputs(wl)
    host = torch.from_numpy(base.blobs).pin_memory()
    cache = api.ExpertCache(wl.fmt, wl.H, wl.I, wl.E, 64, host)
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, device=dev)
    rng = np.random.default_rng(13)
    stream = torch.cuda.current_stream(dev)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
    x = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((wl.T, wl.H), dtype=np.float32))
                         .view(np.int16).copy()).to(dev)

    def steps(n, fresh):
        times, misses, copied = [], [], []
        logits = torch.from_numpy(rng.standard_normal((wl.T, wl.E), dtype=np.float32)).to(dev)
        for i in range(n):
            if fresh:
                logits = torch.from_numpy(rng.standard_normal((wl.T, wl.E), dtype=np.float32)).to(dev)
            flush.fill_(float(i))
            st0 = cache.stats()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            api.rl_moe_verify_bounded(cache, x, logits, wl.T, wl.k, y, ws)
            b.record(stream)
            b.synchronize()
            st1 = cache.stats()
            times.append(a.elapsed_time(b))
            misses.append(st1["misses"] - st0["misses"])
            copied.append(st1["bytes_copied"] - st0["bytes_copied"])
        return times, misses, copied

    steps(args.warmup, True)
    t_miss, m_miss, b_miss = steps(args.steps, True)
    t_hit, m_hit, _ = steps(args.steps, False)
    if api.rl_moe_check_status(ws) != 0:
        raise RuntimeError("bounded verify: device status " + api.rl_last_error())
    # pinned host -> device copy bandwidth on the same stream
    src = torch.empty(64 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(4):
        dst.copy_(src, non_blocking=True)
    b.record(stream)
    b.synchronize()
    h2d_gbs = 4 * (64 << 20) / (a.elapsed_time(b) * 1e-3) / 1e9
    cache.close()
    med_miss = statistics.median(t_miss)
    bytes_med = statistics.median(b_miss)
    return {"shape": "verify2 (T=2, H=2048, I=512, E=512, k=10, Q2)", "slots": 64,
            "ms_median_new_selections": med_miss, "misses_median": statistics.median(m_miss),
            "bytes_copied_median": bytes_med,
            "copy_gbs_effective": bytes_med / (med_miss * 1e-3) / 1e9 if med_miss else None,
            "ms_median_resident": statistics.median(t_hit), "misses_resident": int(sum(m_hit)),
            "h2d_pinned_gbs": h2d_gbs,
            "method": "rl_moe_verify_bounded per step (selections read back to the host inside the step), "
                      "CUDA events on the stream, L2 flushed before each; steps with new router logits "
                      "(misses copied inside the step) and steps repeating the previous logits"}


def bench_ours(args, wl, world, rank, local):
    import torch
    import torch.distributed as dist
    from bit_routed_expert_top_b200 import api

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    inp = synth.make_inputs(wl)
    x = torch.from_numpy(inp.x_bits.view(np.int16).copy()).to(dev)
    logits = torch.from_numpy(inp.logits).to(dev)
    blobs = torch.from_numpy(inp.blobs).to(dev)
    table = api.expert_table(blobs, wl.E)
    y = torch.empty((wl.T, wl.H), dtype=torch.float32, device=dev)
    ws = api.alloc_workspace(wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    P = wl.T * wl.k

    def layer():
        api.rl_moe_prefill_ws(x, logits, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws, stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        layer()
    torch.cuda.synchronize()
    bits = api.rl_moe_check_status(ws, stream)
    if max_over_ranks(bits, world, dev):
        raise SystemExit(f"device status 0x{bits:x} on rank {rank}: {api.rl_last_error()}")

    touched = touched_experts(api, torch, logits, wl, ws, dev)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record(stream)
        layer()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    # second timed pass with CUDA events between the kernels (stage times and
    # the gate/up kernel's duration; the library then launches the kernels
    # without overlapping their starts)
    api.rl_moe_profile_enable(True)
    stage_ms = []
    for i in range(args.steps):
        flush.fill_(float(i))
        layer()
        stage_ms.append(api.rl_moe_profile_read())
    torch.cuda.synchronize()
    clocks = sampler.stop()
    api.rl_moe_profile_enable(False)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    bits = api.rl_moe_check_status(ws, stream)
    if max_over_ranks(bits, world, dev):
        raise SystemExit(f"device status 0x{bits:x} on rank {rank}: {api.rl_last_error()}")

    # end to end through the public API: every step copies its own inputs
    # host -> device and its output device -> host (pinned host buffers).
    # The steps are pipelined the way a serving loop runs them: two device
    # buffer sets; the next step's input copies and the previous step's
    # output copy run on their own streams while the current step's layer
    # runs.  Timed on the device from before the first timed input copy to
    # after the last output copy.
    hx = torch.from_numpy(inp.x_bits.view(np.int16).copy()).pin_memory()
    hl = torch.from_numpy(inp.logits.copy()).pin_memory()
    hy = [torch.empty((wl.T, wl.H), dtype=torch.float32).pin_memory() for _ in range(2)]
    xd, ld, yd = [x, torch.empty_like(x)], [logits, torch.empty_like(logits)], [y, torch.empty_like(y)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_in_free = [torch.cuda.Event() for _ in range(2)]
    ev_out_free = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(args.warmup + args.steps):
        b = i % 2
        if i == args.warmup:
            t0.record(s_in)
        if i >= 2:
            s_in.wait_event(ev_in_free[b])
        with torch.cuda.stream(s_in):
            xd[b].copy_(hx, non_blocking=True)
            ld[b].copy_(hl, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out_free[b])
        flush.fill_(float(i))
        api.rl_moe_prefill_ws(xd[b], ld[b], table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, yd[b], ws, stream)
        ev_out[b].record(stream)
        ev_in_free[b].record(stream)
        s_out.wait_event(ev_out[b])
        with torch.cuda.stream(s_out):
            hy[b].copy_(yd[b], non_blocking=True)
        ev_out_free[b].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

    # the same call captured once into a CUDA graph and replayed (the six
    # launches then cost one graph launch); one GPU only (with a process group
    # up, other threads make CUDA calls), skipped with --no-graph
    graph_ms, graph_err = None, None
    graph = None
    if not args.no_graph and world == 1:
        try:
            graph = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(dev)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
                    api.rl_moe_prefill_ws(x, logits, table, wl.fmt, wl.T, wl.H, wl.I, wl.E, wl.k, y, ws, side)
            torch.cuda.synchronize()
        except Exception as e:  # noqa: BLE001 - reported in the line, every rank agrees below
            graph, graph_err = None, f"{type(e).__name__}: {e}"[:200]
        # every rank times the replays only if every rank captured
        if max_over_ranks(0 if graph is not None else 1, world, dev):
            graph = None
            graph_err = graph_err or "capture failed on another rank"
    if graph is not None:
        gs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.warmup):
            flush.fill_(float(i))
            graph.replay()
        for i in range(args.steps):
            flush.fill_(float(i))
            gs[i].record(stream)
            graph.replay()
            ge[i].record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(gs, ge)), world, dev)
        bits = api.rl_moe_check_status(ws, stream)
        if max_over_ranks(bits, world, dev):
            raise SystemExit(f"device status 0x{bits:x} on rank {rank}: {api.rl_last_error()}")
        del graph
    per_wl = None
    router = None
    shared = None
    cache_fig = None
    if world == 1 and not args.no_per_workload:
        per_wl = per_workload_figures(args, dev, flush, wl.name)
        router = router_gemm_figure(args, dev, flush, wl)
        shared = shared_expert_figure(args, dev, flush, wl)
        cache_fig = expert_cache_figure(args, dev, flush)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    model = layer_model(wl, touched)
    gu_ms = statistics.mean(s["gateup"] for s in stage_ms)
    ms_step = total_ms / args.steps
    achieved_tf = model["flops_gu"] / (gu_ms * 1e-3) / 1e12
    peak_tf = peaks["bf16_tflops"]
    t_roof_ms = max(model["flops"] / (peaks["bf16_tflops"] * 1e12),
                    model["bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    kernel_file = os.path.join(ROOT, "bit_routed_expert_top_b200", "csrc", "gemm_tc.cuh")
    traffic = read_traffic(kernel_file)
    value = replica_throughput(world, args.steps, P, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "ms_per_step_median": statistics.median(step_ms),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
                   "format": synth.FMT_NAMES[wl.fmt], "pairs": P, "touched_experts": touched,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "flushed by a 256 MB device write before every timed step",
                   "arithmetic": "fp16 decoded weights and activations, fp32 accumulate, fp32 y"},
        "roofline": {"bound": "tensor", "kernel": "gate/up decode-GEMM + SwiGLU",
                     "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved_tf / peak_tf, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 dense (fp16 same rate), burst"},
        "layer_roofline": {"t_roof_ms": t_roof_ms, "t_meas_ms": ms_step,
                           "frac": t_roof_ms / ms_step,
                           "tflops": model["flops"] / (ms_step * 1e-3) / 1e12,
                           "algorithmic_bytes": model["bytes"]},
        "stages_ms": {k: statistics.mean(s[k] for s in stage_ms) for k in stage_ms[0]},
        "routed_tokens_per_s": world * args.steps * wl.T / (total_ms * 1e-3),
        "e2e": {"value": replica_throughput(world, args.steps, P, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * 2 + logits.numel() * 4),
                "d2h_bytes_per_step": int(y.numel() * 4),
                "ms_per_step": e2e_ms / args.steps,
                "method": "rl_moe_prefill_ws with pinned host x/logits in and y out every step; "
                          "copies of the next/previous step overlap the current step on two "
                          "copy streams (double-buffered); device-timed over all steps"},
        "gpu_launches": args.steps * api.rl_moe_launches_per_call(),
        "clocks": clocks,
        "wall_s_timed_region": wall,
    }
    if graph_err is not None:
        line["graph_replay"] = {"error": graph_err}
    if graph_ms is not None:
        line["graph_replay"] = {"value": replica_throughput(world, args.steps, P, graph_ms), "unit": UNIT,
                                "ms_per_step": graph_ms / args.steps,
                                "method": "rl_moe_prefill_ws captured once into a CUDA graph, replayed every "
                                          "step (inputs resident, L2 flushed outside the graph)"}
    if per_wl is not None:
        line["per_workload"] = per_wl
    if router is not None:
        line["router_gemm"] = router
    if shared is not None:
        line["shared_expert"] = shared
    if cache_fig is not None:
        line["expert_cache"] = cache_fig
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=synth.WORKLOADS[synth.HEADLINE].name,
                    choices=[w.name for w in synth.WORKLOADS])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip timing the layer call captured once into a CUDA graph and replayed")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the figures of the other workloads (one GPU only)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    wl = next(w for w in synth.WORKLOADS if w.name == args.workload)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        bench_reference(args, wl, world, rank)
    else:
        bench_ours(args, wl, world, rank, local)


if __name__ == "__main__":
    main()
