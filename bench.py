"""Benchmark of the reduced-matrix-multiplication hot path on B200.

One step = one pass of the reduced linear map over the seven projections of a
Llama-3-70B-shaped layer (q, k, v, o: 8192 -> 8192/1024/1024/8192; gate, up:
8192 -> 28672; down: 28672 -> 8192) on a prefill batch of T = 4096 tokens at
retention r = 0.5, with random-init bf16 weights ~N(0, 0.02) pre-transposed
once and synthetic activations N(0, 1) with 2 % of the channels x20.  As in
the layer, q/k/v read one activation matrix and gate/up another, so each of
those sets is one rmm_linear_group call (one score, one kept set, one grouped
tcgen05 GEMM launch); o and down are rmm_linear calls: four C-ABI calls, three
or four kernels each, per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl rmm|reference]

Prints one JSON line (rank 0).  value = effective TFLOP/s = sum 2*T*N*k over
all ranks' steps / max-over-ranks device time.  Extra keys: the dominant
kernel's roofline, the dense cuBLAS comparison (seven products, and the same
with q|k|v and gate|up concatenated into one product each), the end-to-end
number through the public call with host buffers, the oracle timed on the host
cores, the r sweep, the same step on Llama-3-8B shapes (T = 2048), and the
decode (T = 1) GEMV, attention, FFN-demo and decoder-layer rows, with SM clocks
sampled during timing.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import rmm_synth  # noqa: E402
from input_adaptive_reduced_rmm_b200 import metrics  # noqa: E402

R = 0.5
R_SWEEP = [0.125 * i for i in range(1, 9)]
CALLS = [(0, ["q", "k", "v"]), (1, ["o"]), (2, ["gate", "up"]), (3, ["down"])]  # (activation, members)
METRIC = "reduced-GEMM effective TFLOP/s (2*T*N*k / time)"


class Workload:
    """The seven projections of one decoder layer at a prefill batch of T tokens:
    (name, contraction size, output size, activation stream) per projection."""

    def __init__(self, label, cfg, T, H, Nq, Nkv, F):
        self.label, self.cfg, self.T = label, cfg, T
        self.proj = [("q", H, Nq, 0), ("k", H, Nkv, 0), ("v", H, Nkv, 0), ("o", Nq, H, 1),
                     ("gate", H, F, 2), ("up", H, F, 2), ("down", F, H, 3)]
        self.act_h = {0: H, 1: Nq, 2: H, 3: F}
        self.shape = {n: (h, N) for n, h, N, _ in self.proj}

    def name(self, r):
        return f"{self.label} 7 projections (q,k,v,o,gate,up,down), prefill T={self.T}, r={r}"

    def k(self, n, r):
        return metrics.k_for(self.shape[n][0], r)

    def flops(self, r):
        return sum(metrics.reduced_linear_flops(self.T, N, metrics.k_for(h, r)) for _, h, N, _ in self.proj)

    def dense_flops(self):
        return sum(metrics.gemm_flops(self.T, N, h) for _, h, N, _ in self.proj)

    def resident_gb(self):
        w = sum(h * N * 2 for _, h, N, _ in self.proj)
        a = sum(self.T * h * 2 for h in self.act_h.values()) + sum(self.T * N * 2 for _, _, N, _ in self.proj)
        return (w + a) / 1e9


LLAMA70 = Workload("llama3-70b", 4, 4096, 8192, 8192, 1024, 28672)
LLAMA8 = Workload("llama3-8b", 1, 2048, 4096, 4096, 1024, 14336)
HEADLINE = LLAMA70
# DRAM bytes (read + write) of one step's four GEMM launches at r = 0.5, from one
# ncu capture of the current GEMM kernel per workload; an entry is removed whenever
# the GEMM kernel changes, until it is captured again.
STEP_GEMM_DRAM_BYTES = {"llama3-8b": 361_726_464, "llama3-70b": 2_843_581_696}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while timing (the timed
    region of the default run is ~0.1 s, so a coarser interval would see one sample)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values (device time of a multi-GPU run is the slowest rank's)."""
    if world == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time (per second)."""
    return units_per_rank * world / (ms_max * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ oracle (CPU baseline)

_host = {}


def host_inputs(wl):
    """The workload's activations and weights drawn on the host (bf16), once: what the
    reference arm (no GPU) times the oracle on."""
    if wl.label not in _host:
        acts = {s: rmm_synth.activations(wl.T, h, rmm_synth.seed_for(wl.cfg, 70 + s, 0))
                for s, h in wl.act_h.items()}
        weights = {n: rmm_synth.weights(N, h, rmm_synth.seed_for(wl.cfg, 80 + i, 1), std=0.02)
                   for i, (n, h, N, _) in enumerate(wl.proj)}
        _host[wl.label] = (acts, weights)
    return _host[wl.label]


def oracle_sample(wl, inputs, rows_per_proj: int, seed: int, parallel: bool = False):
    """Time the CPU oracle on `rows_per_proj` token rows of every projection (its score and
    kept set over the full batch); parallel=True: its OpenMP build (output rows over the
    host's threads, same bits).  inputs = (activations, weights W [N, H]) on the host.

    Returns (flops, seconds, sample description)."""
    import oracle

    oracle.build(parallel=parallel)
    acts, weights = inputs
    g = torch.Generator().manual_seed(seed)
    flops, secs = 0, 0.0
    for name, h, N, s in wl.proj:
        rows = torch.randperm(wl.T, generator=g)[:rows_per_proj].tolist()
        t0 = time.perf_counter()
        oracle.linear(acts[s], weights[name], R, rows=rows, parallel=parallel)
        secs += time.perf_counter() - t0
        flops += metrics.reduced_linear_flops(rows_per_proj, N, metrics.k_for(h, R))
    kind = (f"fp64 C oracle, OpenMP build on {oracle.parallel_threads()} threads" if parallel
            else "single-threaded fp64 C oracle")
    desc = (f"{rows_per_proj} of {wl.T} token rows per projection, all 7 projections of {wl.label}, "
            f"score and kept set over the full batch; {kind}")
    return flops, secs, desc


def step_config(wl, world: int) -> dict:
    """The workload description both arms print."""
    return {"workload": wl.name(R), "T": wl.T, "r": R, "parallelism": f"replicas x{world}",
            "calls_per_step": "q+k+v grouped, o, gate+up grouped, down",
            "l2": f"inputs larger than L2 ({wl.resident_gb():.2f} GB of weights and activations per step)"}


def run_reference(args, world, rank):
    """The oracle timed on the host cores: each step is a bounded sample of the workload
    (inputs drawn on the host with the same recipe)."""
    if rank != 0:
        return
    wl = HEADLINE
    inputs = host_inputs(wl)
    rows = 1
    for _ in range(args.warmup):
        oracle_sample(wl, inputs, 1, seed=999)
    times, total_flops = [], 0
    sample = ""
    for s in range(args.steps):
        f, t, sample = oracle_sample(wl, inputs, rows, seed=s)
        times.append(t)
        total_flops += f
    value = total_flops / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": step_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def device_inputs(wl, dev):
    """Activations and pre-transposed weights W^T [H, N] drawn on the device (same recipe as
    the host draws, the device's generator)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    acts = {s: rmm_synth.activations(wl.T, h, rmm_synth.seed_for(wl.cfg, 70 + s, 0), device=dev)
            for s, h in wl.act_h.items()}
    Wts = {}
    for i, (n, h, N, _) in enumerate(wl.proj):
        W = rmm_synth.weights(N, h, rmm_synth.seed_for(wl.cfg, 80 + i, 1), std=0.02, device=dev)
        Wts[n] = rmm.rmm_transpose_weight(W)
        del W
    torch.cuda.synchronize()
    return acts, Wts


class PrefillStep:
    """The four calls of one step (q+k+v grouped, o, gate+up grouped, down) with their
    buffers and workspaces, allocated once."""

    def __init__(self, wl, acts, Wts, dev, opts=None):
        from input_adaptive_reduced_rmm_b200 import rmm

        self.rmm, self.wl, self.acts, self.Wts, self.opts = rmm, wl, acts, Wts, opts
        self.Ys = {n: torch.empty(wl.T, N, dtype=torch.bfloat16, device=dev) for n, _, N, _ in wl.proj}
        self.ws = {c: rmm.new_workspace(rmm.rmm_linear_group_workspace_bytes(
            wl.T, wl.act_h[s], [wl.shape[n][1] for n in names], opts), dev) for c, (s, names) in enumerate(CALLS)}

    def __call__(self, r=R, events=None):
        """One step; events = {call: (begin, end)} records the product kernel of each call."""
        rmm = self.rmm
        for c, (s, names) in enumerate(CALLS):
            o = self.opts
            if events is not None:
                base = self.opts
                o = rmm.options(product_events=events[c],
                                block_size=base.block_size if base is not None else 0)
            rmm.rmm_linear_group(self.acts[s], [self.Wts[n] for n in names], r, Ys=[self.Ys[n] for n in names],
                                 workspace=self.ws[c], opts=o)

    def check_status(self, what):
        for c in self.ws:
            if self.rmm.rmm_get_status(self.ws[c]) != self.rmm.RMM_OK:
                raise RuntimeError(f"device status not OK ({what})")


def time_steps(fn, steps, warmup):
    """Device time (ms) of `steps` back-to-back calls after `warmup` untimed ones."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        fn()
    t1.record()
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


def product_times(step, r, steps):
    """Per-call product-kernel time (ms, mean over `steps` steps), from the events the library
    records around each product launch; the step runs `steps` times for it."""
    evs = [{c: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for c in range(len(CALLS))} for _ in range(steps)]
    for i in range(steps):
        step(r, events=evs[i])
    torch.cuda.synchronize()
    return {c: sum(evs[i][c][0].elapsed_time(evs[i][c][1]) for i in range(steps)) / steps
            for c in range(len(CALLS))}


class DenseSteps:
    """cuBLAS (torch.matmul) on the same shapes, inputs and stream: the seven products one by
    one, and the like-for-like form with q|k|v and gate|up concatenated into one product each
    (as the reduced step groups them)."""

    def __init__(self, wl, acts, Wts, dev):
        self.wl, self.acts, self.Wts = wl, acts, Wts
        self.Ys = {n: torch.empty(wl.T, N, dtype=torch.bfloat16, device=dev) for n, _, N, _ in wl.proj}
        self.Wcat = {0: torch.cat([Wts["q"], Wts["k"], Wts["v"]], dim=1),
                     2: torch.cat([Wts["gate"], Wts["up"]], dim=1)}
        self.Ycat = {s: torch.empty(wl.T, W.shape[1], dtype=torch.bfloat16, device=dev) for s, W in self.Wcat.items()}

    def seven(self):
        for n, _, _, s in self.wl.proj:
            torch.matmul(self.acts[s], self.Wts[n], out=self.Ys[n])

    def grouped(self):
        torch.matmul(self.acts[0], self.Wcat[0], out=self.Ycat[0])
        torch.matmul(self.acts[1], self.Wts["o"], out=self.Ys["o"])
        torch.matmul(self.acts[2], self.Wcat[2], out=self.Ycat[2])
        torch.matmul(self.acts[3], self.Wts["down"], out=self.Ys["down"])

    def times(self, steps, warmup):
        t7 = time_steps(self.seven, steps, warmup)
        tg = time_steps(self.grouped, steps, warmup)
        return {"seven_products_ms": t7, "grouped_ms": tg, "best_ms": min(t7, tg),
                "tflops_best": self.wl.dense_flops() / (min(t7, tg) * 1e-3) / 1e12}

    def release(self):
        del self.Wcat, self.Ycat, self.Ys


def launches_per_step(wl, r, dev) -> int:
    """Our kernels launched by one step: per call the score pass, the select, the CTA-pair
    GEMM, and the fold of the split last wave when the call's tiles leave a partial wave
    that the GEMM splits (more than one K-range per tile)."""
    pairs = torch.cuda.get_device_properties(dev).multi_processor_count // 2
    n = 0
    for s, names in CALLS:
        nkb = -(-metrics.k_for(wl.act_h[s], r) // 64)
        tiles = sum(-(-wl.T // 256) * -(-wl.shape[m][1] // 512) for m in names)
        rem = tiles % pairs
        split = min(pairs // rem, 8, nkb) if rem else 1
        n += 3 + (1 if split > 1 else 0)
    return n


def prefill_row(wl, dev, peaks, steps, warmup):
    """Secondary row: the same step on another workload (value, GEMM fraction, speedup
    over the faster dense form)."""
    acts, Wts = device_inputs(wl, dev)
    step = PrefillStep(wl, acts, Wts, dev)
    ms = time_steps(step, steps, warmup)
    gms = product_times(step, R, steps)
    step.check_status(wl.label)
    dense = DenseSteps(wl, acts, Wts, dev)
    dt = dense.times(steps, warmup)
    dense.release()
    flops = wl.flops(R)
    gemm_ms = sum(gms.values())
    out = {"workload": wl.name(R), "ms_per_step": ms, "tflops": flops / (ms * 1e-3) / 1e12,
           "gemm_us": 1e3 * gemm_ms, "gemm_tflops": flops / (gemm_ms * 1e-3) / 1e12,
           "gemm_frac_of_peak": flops / (gemm_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "gemm_dram_bytes": STEP_GEMM_DRAM_BYTES.get(wl.label),
           "dense": dt, "speedup_vs_dense": dt["best_ms"] / ms}
    del step, acts, Wts
    torch.cuda.empty_cache()
    return out


def r_sweep(wl, step, dense_ms, peaks, steps, warmup):
    """The headline step at every retention ratio of the sweep: effective TFLOP/s of the
    step and of its GEMM launches, speedup over the faster dense form, and 1/r."""
    rows = []
    for r in R_SWEEP:
        ms = time_steps(lambda: step(r), steps, warmup)
        gms = sum(product_times(step, r, steps).values())
        f = wl.flops(r)
        rows.append({"r": r, "ms_per_step": ms, "tflops": f / (ms * 1e-3) / 1e12,
                     "gemm_tflops": f / (gms * 1e-3) / 1e12,
                     "gemm_frac_of_peak": f / (gms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "speedup_vs_dense": dense_ms / ms, "ideal_speedup": 1.0 / r})
    step.check_status("r sweep")
    return rows


def time_decode(wl, dev, peaks):
    """Secondary row: one decode step (T = 1) over the workload's seven projections, grouped
    like the prefill step, at r = 0.5; L2 flushed before every timed step."""
    from input_adaptive_reduced_rmm_b200 import rmm

    acts = {s: rmm_synth.activations(1, h, 500 + s, device=dev) for s, h in wl.act_h.items()}
    Wts = {n: rmm.rmm_transpose_weight(rmm_synth.weights(N, h, 600 + i, std=0.02, device=dev))
           for i, (n, h, N, _) in enumerate(wl.proj)}
    Ys = {n: torch.empty(1, N, dtype=torch.bfloat16, device=dev) for n, h, N, _ in wl.proj}
    ws = {c: rmm.new_workspace(rmm.rmm_linear_group_workspace_bytes(
        1, wl.act_h[s], [wl.shape[n][1] for n in names]), dev) for c, (s, names) in enumerate(CALLS)}
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        for c, (s, names) in enumerate(CALLS):
            rmm.rmm_linear_group(acts[s], [Wts[n] for n in names], R, Ys=[Ys[n] for n in names],
                                 workspace=ws[c])

    def dense_step():
        for n, h, N, s in wl.proj:
            torch.matmul(acts[s], Wts[n], out=Ys[n])

    def timed(fn, iters=20):
        # a decode loop replays a captured graph: capture the step once, then
        # time each replay with the weights evicted from L2 beforehand
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fn()
        for _ in range(3):
            graph.replay()
        total = 0.0
        for _ in range(iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        del graph
        return total / iters

    call_ms = timed(step)
    dense_ms = timed(dense_step)
    # the product kernels alone: the library records its product events as graph
    # nodes while the step is captured, so each replay times them in place
    ev_g = {c: (torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for c in range(len(CALLS))}
    opts_g = {c: rmm.options(product_events=ev_g[c]) for c in range(len(CALLS))}

    def step_events():
        for c, (s, names) in enumerate(CALLS):
            rmm.rmm_linear_group(acts[s], [Wts[n] for n in names], R, Ys=[Ys[n] for n in names],
                                 workspace=ws[c], opts=opts_g[c])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step_events()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step_events()
    iters = 20
    kern_ms = 0.0
    for i in range(iters + 3):
        flush.zero_()
        graph.replay()
        torch.cuda.synchronize()
        if i >= 3:
            kern_ms += sum(ev_g[c][0].elapsed_time(ev_g[c][1]) for c in ev_g)
    kern_ms /= iters
    del graph
    for c in ws:
        if rmm.rmm_get_status(ws[c]) != rmm.RMM_OK:
            raise RuntimeError("device status not OK (decode step)")
    kept_bytes = sum(metrics.gemv_bytes(1, h, N, metrics.k_for(h, R)) for _, h, N, _ in wl.proj)
    dense_bytes = sum(N * h * 2 + h * 2 + N * 2 for _, h, N, _ in wl.proj)
    out = {
        "workload": f"T=1, the 7 projections of {wl.label} (q+k+v, o, gate+up, down), r=0.5, CUDA-graph "
                    "replay, L2 flushed before each step",
        "step_us": 1e3 * call_ms,
        "kernel_us": 1e3 * kern_ms,
        "kernel_gbs": kept_bytes / (kern_ms * 1e-3) / 1e9,
        "kernel_frac_of_hbm": kept_bytes / (kern_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "step_gbs": kept_bytes / (call_ms * 1e-3) / 1e9,
        "step_frac_of_hbm": kept_bytes / (call_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "dense_us": 1e3 * dense_ms,
        "dense_gbs": dense_bytes / (dense_ms * 1e-3) / 1e9,
        "speedup_vs_dense": dense_ms / call_ms,
    }
    del Wts, ws, flush
    torch.cuda.empty_cache()
    return out


def time_blocks(wl, dev, acts, Wts, dense_ms, steps, warmup, block=64):
    """Secondary row: the same prefill step with block-granular kept sets (blocks of
    `block` consecutive slices scored by their largest slice score; with 64-slice runs
    the GEMM stages its operands by TMA tile copies)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    ks = {n: metrics.k_for(h // block, R) * block for n, h, _, _ in wl.proj}
    flops = sum(metrics.reduced_linear_flops(wl.T, N, ks[n]) for n, _, N, _ in wl.proj)
    step = PrefillStep(wl, acts, Wts, dev, opts=rmm.options(block_size=block))
    ms = time_steps(step, steps, warmup)
    gemm_ms = sum(product_times(step, R, steps).values())
    step.check_status("block-granular step")
    return {"blocks": {
        "workload": f"the prefill step ({wl.label}, T={wl.T}, r={R}) with {block}-slice block-granular kept sets",
        "ms_per_step": ms,
        "tflops": flops / (ms * 1e-3) / 1e12,
        "gemm_us": 1e3 * gemm_ms,
        "gemm_tflops": flops / (gemm_ms * 1e-3) / 1e12,
        "speedup_vs_dense": dense_ms / ms,
    }}


def time_attn_decode(dev, peaks, L=32768, block=64):
    """Secondary row: one long-context decode attention call (B = 1, 32 query / 8 KV heads,
    d = 128, T = 1, r = 0.5): the head-dim reduction, the same plus context blocks of 64 keys
    (r_ctx = 0.5, 0.25), and dense SDPA on the same cache.  The cache (134 MB of K and V)
    exceeds L2; L2 is flushed before each call anyway."""
    from input_adaptive_reduced_rmm_b200 import rmm

    B, Hq, Hkv, T, d, r = 1, 32, 8, 1, 128, 0.5
    Q = rmm_synth.normal((B, Hq, T, d), 701).to(dev)
    Kt = rmm_synth.normal((B, Hkv, d, L), 702).to(dev)
    V = rmm_synth.normal((B, Hkv, L, d), 703).to(dev)
    K = Kt.transpose(-1, -2).contiguous()
    O = torch.empty_like(Q)
    means = rmm.rmm_ctx_block_means(Kt, L, block)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def timed(fn, iters=30):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e3

    k = rmm.rmm_k_for(d, r)
    ws = rmm.new_workspace(rmm.rmm_attn_workspace_bytes(B, Hq, Hkv, T, L, d), dev)
    red_us = timed(lambda: rmm.rmm_attn_qk(Q, Kt, V, L, r, O=O, workspace=ws))
    red_bytes = Hkv * L * 2 * (k + d)
    out = {"workload": f"decode attention, B=1, Hq=32, Hkv=8, d=128, L={L}, T=1, r=0.5; context blocks of {block}",
           "reduced_us": red_us, "reduced_gbs": red_bytes / (red_us * 1e-6) / 1e9,
           "reduced_frac_of_hbm": red_bytes / (red_us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    nblk = rmm.ctx_num_blocks(L, block)
    for rc in (0.5, 0.25):
        kc = rmm.rmm_k_for(nblk, rc)
        wsc = rmm.new_workspace(rmm.rmm_attn_ctx_workspace_bytes(B, Hq, Hkv, T, L, block, rc), dev)
        us = timed(lambda: rmm.rmm_attn_ctx(Q, Kt, V, means, L, r, rc, block, O=O, workspace=wsc))
        if rmm.rmm_get_status(wsc) != rmm.RMM_OK:
            raise RuntimeError("device status not OK (context-block attention)")
        cbytes = Hkv * kc * block * 2 * (k + d) + Hkv * nblk * d * 4
        out[f"ctx_rc{rc}_us"] = us
        out[f"ctx_rc{rc}_gbs"] = cbytes / (us * 1e-6) / 1e9
    sdpa_us = timed(lambda: torch.nn.functional.scaled_dot_product_attention(Q, K, V, enable_gqa=True))
    out["dense_sdpa_us"] = sdpa_us
    out["dense_sdpa_gbs"] = Hkv * L * 2 * 2 * d / (sdpa_us * 1e-6) / 1e9
    out["speedup_reduced_vs_dense"] = sdpa_us / red_us
    out["speedup_ctx_rc0.25_vs_dense"] = sdpa_us / out["ctx_rc0.25_us"]
    if rmm.rmm_get_status(ws) != rmm.RMM_OK:
        raise RuntimeError("device status not OK (decode attention)")
    del Q, Kt, V, K, O, means, flush
    torch.cuda.empty_cache()
    return {"attn_decode": out}


def time_ffn_demo(dev):
    """Secondary row: the cf-1.com post's FFN demo (H = 1024, M = 4096, one token):
    gate/up in full, SwiGLU, the down projection reduced to the 64-neuron blocks of
    largest mean |h| at keep 0.5 -- against the dense FFN (cuBLAS products, the same
    SwiGLU kernel).  Both captured as CUDA graphs, L2 flushed before each replay; the
    output's mean |y_reduced - y_full| is the quantity the demo prints."""
    from input_adaptive_reduced_rmm_b200.ffn_demo import FfnBlockReduce

    H, M, T = 1024, 4096, 1
    W_gate = rmm_synth.weights(M, H, 801, std=0.02).to(dev)
    W_up = rmm_synth.weights(M, H, 802, std=0.02).to(dev)
    W_down = rmm_synth.weights(H, M, 803, std=0.02).to(dev)
    x = rmm_synth.normal((T, H), 804).to(dev)
    f = FfnBlockReduce(W_gate, W_up, W_down, block=64, keep=0.5)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def graph_time(fn, iters=30):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            out = fn()
        ts = []
        for _ in range(iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        del g
        return statistics.median(ts) * 1e3, out

    red_us, _ = graph_time(lambda: f.forward(x, want_blocks=False)[0])
    dense_us, _ = graph_time(lambda: f.forward_dense(x))
    y_red = f.forward(x)[0].float()
    y_full = f.forward_dense(x).float()
    torch.cuda.synchronize()
    out = {"ffn_demo": {
        "workload": "FFN of the post's demo: x [1, 1024], gate/up 4096x1024 full, SwiGLU, down 1024x4096 "
                    "reduced to mean-|h| blocks of 64 at keep 0.5",
        "reduced_us": red_us, "dense_us": dense_us, "speedup_vs_dense": dense_us / red_us,
        "down_proj_flops_fraction": f.kb * 64 / M,
        "mean_abs_diff_vs_full": float((y_red - y_full).abs().mean()),
        "mean_abs_full": float(y_full.abs().mean()),
    }}
    del f, W_gate, W_up, W_down, flush
    torch.cuda.empty_cache()
    return out


def time_layer(dev):
    """Secondary row: one Llama-3-8B decoder layer (hidden 4096, 32 query / 8 KV heads,
    MLP 14336, B = 1): prefill of T = 2048 tokens, then 128 decode steps against the
    growing KV cache, r = 0.5; against the same layer with dense products (cuBLAS) and
    dense attention (SDPA).  Prefill per op with CUDA events (L2 flushed before each
    run) from a captured graph with timing events as graph nodes; decode as CUDA-graph
    replays, one graph per cache position, timed end to end."""
    from input_adaptive_reduced_rmm_b200.layer import DecoderLayer, DenseLayer, LayerDims

    dims = LayerDims()
    wl = LLAMA8
    Tp, steps = wl.T, 128
    W = {n: rmm_synth.weights(N, h, rmm_synth.seed_for(3, 80 + i, 1), std=0.02, device=dev)
         for i, (n, h, N, _) in enumerate(wl.proj)}
    layers = {"rmm": DecoderLayer(dims, W, Tp + steps, R, dev), "dense": DenseLayer(dims, W, Tp + steps, dev)}
    xp = rmm_synth.activations(Tp, dims.H, 700, device=dev)
    xd = rmm_synth.activations(steps, dims.H, 701, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    out = {}
    for name, layer in layers.items():
        # prefill: captured once (timing events as graph nodes), replayed after an L2 flush
        layer.reset()
        layer.forward(xp)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        ev = []
        gp = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            layer.reset()
            with torch.cuda.graph(gp, stream=side):
                layer.forward(xp, events=ev)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        runs, totals = [], []
        for i in range(6):
            flush.zero_()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            gp.replay()
            t1.record()
            torch.cuda.synchronize()
            if i:
                runs.append({n: e0.elapsed_time(e1) for n, e0, e1 in ev})
                totals.append(t0.elapsed_time(t1))
        del gp
        per_op = {n: 1e3 * statistics.median(r[n] for r in runs) for n in runs[0]}
        prefill_us = 1e3 * statistics.median(totals)
        # decode: warm the T = 1 buffers eagerly, then capture one graph per position
        layer.reset()
        layer.forward(xp)
        layer.forward(xd[0:1])
        torch.cuda.synchronize()
        layer.pos = Tp
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        graphs = []
        with torch.cuda.stream(side):
            for t in range(steps):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=side):
                    layer.forward(xd[t:t + 1])
                graphs.append(g)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        times = []
        for _ in range(3):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for g in graphs:
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        del graphs
        out[name] = {"prefill_us": prefill_us, "prefill_per_op_us": per_op,
                     "decode_128_steps_us": 1e3 * statistics.median(times),
                     "decode_step_us": 1e3 * statistics.median(times) / steps}
    del layers, flush
    torch.cuda.empty_cache()
    r_, d_ = out["rmm"], out["dense"]
    return {"layer": {
        "workload": "Llama-3-8B decoder layer (RMSNorm, q/k/v, reduced attention over the head dim, o, "
                    "residual, RMSNorm, gate/up, SwiGLU, down, residual), B=1, prefill T=2048 then 128 "
                    "decode steps, r=0.5; dense = cuBLAS products (q|k|v and gate|up concatenated, one product each) "
                    "+ SDPA attention, the same norm kernels, torch's silu(g)*u",
        "rmm": r_, "dense": d_,
        "prefill_speedup_vs_dense": d_["prefill_us"] / r_["prefill_us"],
        "decode_speedup_vs_dense": d_["decode_128_steps_us"] / r_["decode_128_steps_us"],
        "total_us": r_["prefill_us"] + r_["decode_128_steps_us"],
        "dense_total_us": d_["prefill_us"] + d_["decode_128_steps_us"],
    }}


def run_rmm(args, world, rank, local):
    dev = torch.device("cuda", local if world > 1 else 0)
    peaks = load_peaks()
    wl = HEADLINE
    acts, Wts = device_inputs(wl, dev)
    step_flops = wl.flops(R)
    step = PrefillStep(wl, acts, Wts, dev)
    K, W = args.steps, args.warmup

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    step.check_status("warm-up")

    clocks = ClockSampler(local if world > 1 else 0)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(K):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    ms = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms, world)
    value = job_throughput(step_flops * K, world, ms_max) / 1e12

    # the same K steps again with events recorded around each product launch
    # (the events separate the product kernel from its predecessor, so this
    # pass is timed on its own and only its per-kernel split is used)
    barrier(world)
    torch.cuda.synchronize()
    gemm_ms = product_times(step, R, K)
    barrier(world)
    clk = clocks.stop()
    step.check_status("timed steps")

    # dominant kernel: the reduced GEMM launches, timed by events the library
    # records around each product launch inside the timed region
    gemm_total_ms = sum(gemm_ms.values())
    achieved = step_flops / (gemm_total_ms * 1e-3) / 1e12
    per_call = {}
    for c, (s, names) in enumerate(CALLS):
        f = sum(metrics.reduced_linear_flops(wl.T, wl.shape[n][1], wl.k(n, R)) for n in names)
        per_call["+".join(names)] = {"H": wl.act_h[s], "N": [wl.shape[n][1] for n in names], "k": wl.k(names[0], R),
                                     "gemm_us": 1e3 * gemm_ms[c], "gemm_tflops": f / (gemm_ms[c] * 1e-3) / 1e12}

    # dense cuBLAS products of the same shapes, same stream, same inputs
    dense = DenseSteps(wl, acts, Wts, dev)
    dense_t = dense.times(K, W)
    dense.release()
    dense_ms = dense_t["best_ms"]

    # end to end through the public calls with host buffers: H2D of the step's
    # activations, the four calls, D2H of the seven outputs, every step
    host_acts = {s: a.cpu().pin_memory() for s, a in acts.items()}
    host_Y = {n: torch.empty(wl.T, N, dtype=torch.bfloat16).pin_memory() for n, _, N, _ in wl.proj}
    h2d = sum(a.numel() * 2 for a in host_acts.values())
    d2h = sum(y.numel() * 2 for y in host_Y.values())

    def e2e_step():
        for s, a in host_acts.items():
            acts[s].copy_(a, non_blocking=True)
        step()
        for n in host_Y:
            host_Y[n].copy_(step.Ys[n], non_blocking=True)

    for _ in range(W):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_throughput(step_flops * K, world, e2e_ms) / 1e12
    del host_Y

    extra = {}
    if not args.skip_secondary:
        sweep_steps = max(5, K // 2)
        extra["r_sweep"] = r_sweep(wl, step, dense_ms, peaks, sweep_steps, 3)
        extra.update(time_blocks(wl, dev, acts, Wts, dense_ms, sweep_steps, 3))

    cpu = cpu_par = None
    if rank == 0 and not args.skip_cpu_baseline:
        # the oracle on the step's own inputs, copied to the host (W back to [N, H])
        inputs = ({s: a.cpu() for s, a in acts.items()}, {n: Wt.t().contiguous().cpu() for n, Wt in Wts.items()})
        f, t, desc = oracle_sample(wl, inputs, args.cpu_rows, seed=1)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": desc}
        # the same oracle's OpenMP build on all host threads (a reported baseline too)
        import oracle

        threads = oracle.parallel_threads()
        f, t, desc = oracle_sample(wl, inputs, args.cpu_rows * max(1, min(threads, 16)) // 2, seed=2,
                                   parallel=True)
        cpu_par = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle-openmp",
                   "sample": desc}
        del inputs

    launches = launches_per_step(wl, R, dev)
    del step, acts, Wts
    torch.cuda.empty_cache()
    if not args.skip_secondary:
        extra["prefill_llama3_8b"] = prefill_row(LLAMA8, dev, peaks, K, W)
        extra["decode_gemv"] = time_decode(LLAMA70, dev, peaks)
        extra["decode_gemv_llama3_8b"] = time_decode(LLAMA8, dev, peaks)
        extra.update(time_attn_decode(dev, peaks))
        extra.update(time_ffn_demo(dev))
        extra.update(time_layer(dev))

    if rank != 0:
        return
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": step_config(wl, world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": STEP_GEMM_DRAM_BYTES.get(wl.label),
                     "traffic_unit": "bytes (ncu dram read + write) over the step's 4 GEMM launches",
                     "kernel": "gemm_pair_kernel (tcgen05 cta_group::2 reduced GEMM), the 4 launches of a step",
                     "peak_source": f"{peaks['source']} bf16 burst"},
        "speedup_vs_dense": dense_ms / (ms_max / K),
        "dense": {**dense_t, "tflops": dense_t["tflops_best"],
                  "effective_tflops_at_reduced_flops": step_flops / (dense_ms * 1e-3) / 1e12},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "cpu_baseline": cpu,
        "cpu_baseline_parallel": cpu_par,
        "gpu_launches": launches * K,
        "clocks": clk,
        "per_call": per_call,
    }
    line.update(extra)
    print(json.dumps(line), flush=True)


def run_profile_step(args):
    """The headline step alone, --warmup then --steps times (profiling aid: nothing else
    runs, so an ncu capture holds only the step's own buffers)."""
    dev = torch.device("cuda", 0)
    wl = HEADLINE
    acts, Wts = device_inputs(wl, dev)
    step = PrefillStep(wl, acts, Wts, dev)
    ms = time_steps(step, args.steps, args.warmup)
    step.check_status("profile step")
    print(json.dumps({"profile_step": {"workload": wl.name(R), "ms_per_step": ms,
                                       "tflops": wl.flops(R) / (ms * 1e-3) / 1e12,
                                       "launches_per_step": launches_per_step(wl, R, dev)}}), flush=True)


def run_profile_decode(args):
    """The decode step (T = 1, the seven projections of --profile-decode's workload, grouped
    like the prefill step) eagerly, --warmup then --steps times (profiling aid)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    wl = {"llama3-8b": LLAMA8, "llama3-70b": LLAMA70}[args.profile_decode]
    dev = torch.device("cuda", 0)
    acts = {s: rmm_synth.activations(1, h, 500 + s, device=dev) for s, h in wl.act_h.items()}
    Wts = {n: rmm.rmm_transpose_weight(rmm_synth.weights(N, h, 600 + i, std=0.02, device=dev))
           for i, (n, h, N, _) in enumerate(wl.proj)}
    Ys = {n: torch.empty(1, N, dtype=torch.bfloat16, device=dev) for n, h, N, _ in wl.proj}
    ws = {c: rmm.new_workspace(rmm.rmm_linear_group_workspace_bytes(
        1, wl.act_h[s], [wl.shape[n][1] for n in names]), dev) for c, (s, names) in enumerate(CALLS)}

    def step():
        for c, (s, names) in enumerate(CALLS):
            rmm.rmm_linear_group(acts[s], [Wts[n] for n in names], R, Ys=[Ys[n] for n in names], workspace=ws[c])

    ms = time_steps(step, args.steps, args.warmup)
    for c in ws:
        if rmm.rmm_get_status(ws[c]) != rmm.RMM_OK:
            raise RuntimeError("device status not OK (decode profile)")
    print(json.dumps({"profile_decode": {"workload": wl.label, "ms_per_step_eager": ms}}), flush=True)


def run_single(args):
    """One rmm_linear shape timed alone (profiling aid): --single T,H,N,r."""
    from input_adaptive_reduced_rmm_b200 import rmm

    T, H, N, r = args.single.split(",")
    T, H, N, r = int(T), int(H), int(N), float(r)
    dev = torch.device("cuda", 0)
    X = rmm_synth.activations(T, H, 11).to(dev)
    Wt = rmm.rmm_transpose_weight(rmm_synth.weights(N, H, 12, std=0.02).to(dev))
    Y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    opts = rmm.options(gemm_producer=args.gemm_producer, block_size=args.block_size, product_events=ev)
    ws = rmm.new_workspace(rmm.rmm_linear_workspace_bytes(T, H, N, opts), dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        rmm.rmm_linear(X, Wt, r, Y=Y, workspace=ws, opts=opts)
    torch.cuda.synchronize()
    call, kern = [], []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        rmm.rmm_linear(X, Wt, r, Y=Y, workspace=ws, opts=opts)
        e1.record()
        torch.cuda.synchronize()
        call.append(e0.elapsed_time(e1))
        kern.append(ev[0].elapsed_time(ev[1]))
    if rmm.rmm_get_status(ws) != rmm.RMM_OK:
        raise RuntimeError("device status not OK")
    bs = args.block_size
    k = metrics.k_for(H // bs, r) * bs if bs else metrics.k_for(H, r)
    km = statistics.median(kern)
    out = {"single": {"T": T, "H": H, "N": N, "r": r, "k": k, "producer": args.gemm_producer, "block_size": bs,
                      "call_us": 1e3 * statistics.median(call), "product_us": 1e3 * km,
                      "product_tflops": metrics.reduced_linear_flops(T, N, k) / (km * 1e-3) / 1e12,
                      "product_gbs": metrics.gemv_bytes(T, H, N, k) / (km * 1e-3) / 1e9}}
    print(json.dumps(out), flush=True)


def run_single_attn(args):
    """One rmm_attn_qk call timed alone (profiling aid): --single-attn B,Hq,Hkv,T,L,r (causal,
    d = 128, queries at the last T positions of a cache of L keys)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    B, Hq, Hkv, T, L, r = args.single_attn.split(",")
    B, Hq, Hkv, T, L, r = int(B), int(Hq), int(Hkv), int(T), int(L), float(r)
    dev = torch.device("cuda", 0)
    D = 128
    Q = rmm_synth.normal((B, Hq, T, D), 21).to(dev)
    Kt = rmm_synth.normal((B, Hkv, D, L), 22).to(dev)
    V = rmm_synth.normal((B, Hkv, L, D), 23).to(dev)
    O = torch.empty_like(Q)
    ws = rmm.new_workspace(rmm.rmm_attn_workspace_bytes(B, Hq, Hkv, T, L, D), dev)
    for _ in range(args.warmup):
        rmm.rmm_attn_qk(Q, Kt, V, L, r, O=O, workspace=ws)
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        rmm.rmm_attn_qk(Q, Kt, V, L, r, O=O, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    if rmm.rmm_get_status(ws) != rmm.RMM_OK:
        raise RuntimeError("device status not OK")
    k = metrics.k_for(D, r)
    ms = statistics.median(ts)
    flops = metrics.attn_flops(B, Hq, T, L, D, k, causal=True)
    print(json.dumps({"single_attn": {"B": B, "Hq": Hq, "Hkv": Hkv, "T": T, "L": L, "r": r, "k": k,
                                      "call_us": 1e3 * ms, "tflops": flops / (ms * 1e-3) / 1e12}}), flush=True)


def run_single_ctx(args):
    """One rmm_attn_ctx call timed alone (profiling aid): --single-ctx B,Hq,Hkv,L,block,r,r_ctx
    (decode, T = 1, d = 128; the block means are made once, untimed)."""
    from input_adaptive_reduced_rmm_b200 import rmm

    B, Hq, Hkv, L, block, r, r_ctx = args.single_ctx.split(",")
    B, Hq, Hkv, L, block, r, r_ctx = int(B), int(Hq), int(Hkv), int(L), int(block), float(r), float(r_ctx)
    dev = torch.device("cuda", 0)
    D, T = 128, 1
    Q = rmm_synth.normal((B, Hq, T, D), 31).to(dev)
    Kt = rmm_synth.normal((B, Hkv, D, L), 32).to(dev)
    V = rmm_synth.normal((B, Hkv, L, D), 33).to(dev)
    O = torch.empty_like(Q)
    means = rmm.rmm_ctx_block_means(Kt, L, block)
    ws = rmm.new_workspace(rmm.rmm_attn_ctx_workspace_bytes(B, Hq, Hkv, T, L, block, r_ctx), dev)
    for _ in range(args.warmup):
        rmm.rmm_attn_ctx(Q, Kt, V, means, L, r, r_ctx, block, O=O, workspace=ws)
    torch.cuda.synchronize()
    ts = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        rmm.rmm_attn_ctx(Q, Kt, V, means, L, r, r_ctx, block, O=O, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    if rmm.rmm_get_status(ws) != rmm.RMM_OK:
        raise RuntimeError("device status not OK")
    print(json.dumps({"single_ctx": {"B": B, "Hq": Hq, "Hkv": Hkv, "L": L, "block": block, "r": r, "r_ctx": r_ctx,
                                     "call_us": 1e3 * statistics.median(ts)}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rmm", "reference"], default="rmm")
    ap.add_argument("--cpu-rows", type=int, default=8)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-secondary", action="store_true")
    ap.add_argument("--single", default=None, help="T,H,N,r: time one rmm_linear shape alone")
    ap.add_argument("--single-attn", default=None, help="B,Hq,Hkv,T,L,r: time one rmm_attn_qk call alone")
    ap.add_argument("--single-ctx", default=None,
                    help="B,Hq,Hkv,L,block,r,r_ctx: time one rmm_attn_ctx decode call alone")
    ap.add_argument("--profile-step", action="store_true", help="run only the headline step (profiling aid)")
    ap.add_argument("--profile-decode", default=None, choices=["llama3-8b", "llama3-70b"],
                    help="run only the decode (T = 1) step of that workload, eagerly (profiling aid)")
    ap.add_argument("--gemm-producer", type=int, default=0)
    ap.add_argument("--block-size", type=int, default=0, help="with --single: block-granular kept sets")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.single_attn:
        run_single_attn(args)
        return
    if args.single_ctx:
        run_single_ctx(args)
        return
    if args.single:
        run_single(args)
        return
    if args.profile_step:
        run_profile_step(args)
        return
    if args.profile_decode:
        run_profile_decode(args)
        return
    if args.impl == "reference":
        # the oracle on the host cores: rank 0 alone, no process group, no GPU
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()
    try:
        run_rmm(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
