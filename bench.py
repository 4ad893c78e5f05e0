#!/usr/bin/env python
"""Benchmark of the Sherry 3:4 ternary matmul on B200.

Headline workload (one "step"): the decode hot path at M = 1 token over the
three Llama-3-8B-shaped projections (K,N) = (4096,4096), (4096,14336),
(14336,4096), rotated across 32 independently seeded layer copies: for each
of the 96 layers, the per-token int8 activation quantiser and the tcgen05
GEMM with its fp32 epilogue.  The packed weights of one step are 671 MB, well
above the 126 MB L2, so every weight byte of a step comes from HBM.  The
step is captured once in a CUDA graph and replayed.

Metric: GB/s of algorithmic bytes (packed 5-bit codes + fp32 alpha + int8
activations + fp32 scales) per second of device time.  Extras in the same
JSON line: small-batch decode (M = 4..32) in GB/s and the prefill GEMM
(M = 2048) in int-TOPS against the INT8 tensor roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tc|simt|reference]

Under torchrun every rank runs the same workload on its own GPU with its own
layer copies (weak scaling, no data-path collective); the time is the max
over ranks.  ``--impl reference`` times the CPU oracle (the plain C statement
of the method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "3:4-ternary GEMV GB/s & GEMM int-TOPS on 1 B200; % of HBM/INT8 roofline"
PROJ_SHAPES = [(4096, 4096), (4096, 14336), (14336, 4096)]      # (K, N)
NOMINAL_INT8_OVER_BF16 = 2.0                                    # 4.5 / 2.25 PFLOP/s dense
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["auto", "decode", "tc", "gemv", "simt", "reference"], default="auto",
                    help="auto = sherry_linear (quantiser fused into the decode GEMM); others = "
                         "sherry_quant_act + that GEMM kernel")
    ap.add_argument("--copies", type=int, default=32)
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=["decode", "small", "prefill", "w4a8", "long"], default=None,
                    help="run a few launches of one layer shape (K=4096, N=14336; M=1, 16 or 2048; "
                         "w4a8: the SINT4 x int8 GEMM at M=2048; long: M=1, K=8192, N=28672) and exit: "
                         "the target of the committed ncu captures")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- helpers
def algorithmic_bytes(M: int, K: int, N: int) -> int:
    """Packed codes + alpha + int8 activations + activation scales."""
    return N * K * 5 // 32 + 4 * N + M * K + 4 * M


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms; only the
    samples whose timestamps fall inside the timed window are summarised."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.window = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t_end = time.time() + 5.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.02)

    def mark(self, begin: float, end: float):
        self.window = (begin, end)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        from datetime import datetime
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = rows
        if self.window is not None:
            b, e = self.window
            inside = [r for r in rows if b <= r[0] <= e] or \
                     [min(rows, key=lambda r: abs(r[0] - 0.5 * (b + e)))]
        reasons = set()
        for r in inside:
            for nm, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside),
                "window_s": round(self.window[1] - self.window[0], 3) if self.window else None}


# ------------------------------------------------------------- distributed
def dist_setup(gpus: int, need_cuda: bool):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if (need_cuda and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ CPU baseline
def oracle_codes(W):
    """The oracle's own ternarisation and packing (sec. 3.1, sec. 2.1): the
    oracle-side legs never load the CUDA library."""
    import oracle
    T, alpha = oracle.quantise(W)
    return oracle.pack(T), alpha


def cpu_baseline(seconds: float, copy: int = 0):
    """The oracle as it stands on a bounded sample: unpack + contract +
    epilogue (and the activation quantiser) over the three projections of
    one layer copy, repeated until ~`seconds` of CPU work."""
    import oracle
    import synth
    layers = []
    for K, N in PROJ_SHAPES:
        codes, alpha = oracle_codes(synth.config_weights(1, copy, K, N))
        x = synth.config_activations(1, copy, 1, K)
        layers.append((K, N, codes, alpha, x))
    done_bytes, t0, passes = 0, time.perf_counter(), 0
    while True:
        for K, N, codes, alpha, x in layers:
            q, s = oracle.quant_act(x)
            oracle.forward(q, s, codes, alpha, K)
            done_bytes += algorithmic_bytes(1, K, N)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": round(done_bytes / el / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{passes} pass(es) over the 3 projections of layer copy {copy} at M=1 "
                      f"(activation quantiser + unpack + int contraction + epilogue), {el:.1f} s"}


def cpu_lut_baseline(seconds: float, copy: int = 0):
    """The page's own CPU scheme (cpu_lut: 16-entry segment tables read with
    vpshufb, sign, integer sums, one float scaling) on the host cores, on
    the same bounded sample as cpu_baseline; int8 activations and the
    lookup layout are prepared before the timed passes."""
    try:
        import cpu_lut
        import oracle
        import synth
        layers = []
        for K, N in PROJ_SHAPES:
            codes, alpha = oracle_codes(synth.config_weights(1, copy, K, N))
            q, s = oracle.quant_act(synth.config_activations(1, copy, 1, K))
            layers.append((K, N, cpu_lut.prepare(codes, K), alpha, q, s))
        done_bytes, t0, passes = 0, time.perf_counter(), 0
        while True:
            for K, N, prep, alpha, q, s in layers:
                cpu_lut.gemm(q, s, prep, alpha, N, K, want_acc=False)
                done_bytes += algorithmic_bytes(1, K, N)
            passes += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
        working_set = sum(prep.nbytes + alpha.nbytes + q.nbytes for _, _, prep, alpha, q, _ in layers)
        return {"value": round(done_bytes / el / 1e9, 3), "unit": "GB/s", "cores": cpu_lut.num_threads(),
                "kind": "page_cpu_lut_" + ("avx2" if cpu_lut.has_avx2() else "scalar"),
                "working_set_bytes": int(working_set),
                "cache_resident": ("possibly: one layer copy (%.0f MB in the lookup layout) is rotated, which may "
                                   "fit the host's last-level cache; the GPU line streams 671 MB from HBM"
                                   % (working_set / 1e6)),
                "sample": f"{passes} pass(es) over the 3 projections of layer copy {copy} at M=1 "
                          f"(table build + lookups + int sums + epilogue; int8 activations prepared), {el:.1f} s"}
    except Exception as e:                      # a comparison line only: never fails the bench
        return {"unavailable": f"{type(e).__name__}: {e}"}


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle on a bounded sample, same metric."""
    if rank != 0:
        return
    import oracle
    import synth
    layers = []
    for K, N in PROJ_SHAPES:
        codes, alpha = oracle_codes(synth.config_weights(1, 0, K, N))
        layers.append((K, N, codes, alpha, synth.config_activations(1, 0, 1, K)))

    def step(i):
        K, N, codes, alpha, x = layers[i % 3]
        q, s = oracle.quant_act(x)
        oracle.forward(q, s, codes, alpha, K)
        return algorithmic_bytes(1, K, N)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    b = sum(step(i) for i in range(args.steps))
    el = time.perf_counter() - t0
    v = b / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": "decode GEMV M=1, Llama-3-8B projections (4096x4096, 4096->14336, "
                               "14336->4096); each reference step is one projection of layer copy 0",
                   "M": 1},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{args.steps} steps, one projection each, rotating the 3 shapes"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def build_layers(copies: int, copy_base: int, M: int, device):
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    layers = []
    for r in range(copies):
        copy = copy_base + r
        for K, N in PROJ_SHAPES:
            W = synth.config_weights(1, copy, K, N)
            codes, alpha = sbm.pack(W)
            del W
            codes_d = torch.from_numpy(codes).to(device)
            native = sbm.repack(codes_d, N, K)
            del codes_d
            x = synth.config_activations(1, copy, M, K)
            layers.append(dict(
                K=K, N=N, native=native, alpha=torch.from_numpy(alpha).to(device),
                x_host=torch.from_numpy(x).pin_memory(), x=torch.from_numpy(x).to(device),
                q=torch.empty((M, K), dtype=torch.int8, device=device),
                s=torch.empty(M, dtype=torch.float32, device=device),
                y=torch.empty((M, N), dtype=torch.float32, device=device),
                y_host=torch.empty((M, N), dtype=torch.float32).pin_memory()))
    torch.cuda.synchronize()
    return layers


def capture(fn, warm: int = 2):
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(g, steps: int, warmup: int, world: int, sampler=None):
    import torch
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    w1 = time.time()
    if sampler is not None:
        sampler.mark(w0, w1)
    barrier(world)
    return e0.elapsed_time(e1) / 1e3


def time_pipelined_e2e(g_comp, x_dev, x_host, y_dev, y_host, steps: int, warmup: int, world: int):
    """End-to-end steps with the copies overlapped, as a serving loop runs them:
    step k's inputs go host -> device on one copy stream while step k - 1
    computes, its outputs device -> host on another while step k + 1 computes.
    Two device buffers of inputs and of outputs (b = k mod 2); g_comp[b] is the
    captured compute of one step on buffer pair b.  Every step still copies
    its own inputs in and its own outputs out inside the timed region, which
    runs from before the first input copy to after the last output copy."""
    import torch
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_comp = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]

    def run(n):
        used = [False, False]
        for k in range(n):
            b = k & 1
            if used[b]:
                h2d.wait_event(ev_comp[b])            # step k - 2 has read x_dev[b]
            with torch.cuda.stream(h2d):
                x_dev[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(h2d)
            comp.wait_event(ev_in[b])
            if used[b]:
                comp.wait_event(ev_out[b])            # step k - 2's outputs have left y_dev[b]
            g_comp[b].replay()
            ev_comp[b].record(comp)
            d2h.wait_event(ev_comp[b])
            with torch.cuda.stream(d2h):
                y_host[b].copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(d2h)
            used[b] = True
        for b in range(min(n, 2)):
            comp.wait_event(ev_out[b])

    run(max(warmup, 2))
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    h2d.wait_event(e0)
    d2h.wait_event(e0)
    run(steps)
    e1.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1) / 1e3


def run_gpu(args, world, rank, local):
    import torch
    import sparse_bit_matmul_b200 as sbm

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    sbm.load()
    kernel = args.impl
    M = 1
    layers = build_layers(args.copies, rank * args.copies, M, device)
    step_bytes = sum(algorithmic_bytes(M, L["K"], L["N"]) for L in layers)
    code_bytes = sum(L["N"] * L["K"] * 5 // 32 for L in layers)

    # auto: sherry_linear, one fused launch per layer call (quantiser + GEMM);
    # otherwise sherry_quant_act + the named GEMM kernel, two launches
    fused = kernel == "auto"

    def layer(L, x=None, y=None):
        x = L["x"] if x is None else x
        y = L["y"] if y is None else y
        if fused:
            sbm.linear(x, L["native"], L["alpha"], L["N"], out=y)
        else:
            sbm.quant_act(x, L["q"], L["s"])
            sbm.gemm(L["q"], L["s"], L["native"], L["alpha"], L["N"], out=y, kernel=kernel)

    def step():
        for L in layers:
            layer(L)

    def gemm_only():
        for L in layers:
            sbm.gemm(L["q"], L["s"], L["native"], L["alpha"], L["N"], out=L["y"],
                     kernel="auto" if fused else kernel)

    def quant_only():
        for L in layers:
            sbm.quant_act(L["x"], L["q"], L["s"])

    def two_launch_step():
        for L in layers:
            sbm.quant_act(L["x"], L["q"], L["s"])
            sbm.gemm(L["q"], L["s"], L["native"], L["alpha"], L["N"], out=L["y"])

    # end to end, the step's inputs and outputs each in one pinned host
    # buffer: one H2D copy of all layer inputs, the layer calls on device
    # views of one input and one output buffer, one D2H copy of all outputs
    x_total = sum(L["x"].numel() for L in layers)
    y_total = sum(L["y"].numel() for L in layers)
    X_host = torch.empty(x_total, dtype=torch.float32).pin_memory()
    Y_host = torch.empty(y_total, dtype=torch.float32).pin_memory()
    X_dev = torch.empty(x_total, dtype=torch.float32, device=device)
    Y_dev = torch.empty(y_total, dtype=torch.float32, device=device)
    xo = yo = 0
    for L in layers:
        nx, ny = L["x"].numel(), L["y"].numel()
        X_host[xo:xo + nx].copy_(L["x_host"].reshape(-1))
        L["x_step"] = X_dev[xo:xo + nx].view(L["x"].shape)
        L["y_step"] = Y_dev[yo:yo + ny].view(L["y"].shape)
        xo += nx
        yo += ny

    def e2e_step():
        X_dev.copy_(X_host, non_blocking=True)
        for L in layers:
            layer(L, L["x_step"], L["y_step"])
        Y_host.copy_(Y_dev, non_blocking=True)

    # the pipelined end-to-end form: two device buffer pairs, the compute of
    # one step on each captured as its own graph
    X_dev2 = [X_dev, torch.empty_like(X_dev)]
    Y_dev2 = [Y_dev, torch.empty_like(Y_dev)]
    Y_host2 = [Y_host, torch.empty(y_total, dtype=torch.float32).pin_memory()]
    pipe_views = []
    for b in range(2):
        xo = yo = 0
        vb = []
        for L in layers:
            nx, ny = L["x"].numel(), L["y"].numel()
            vb.append((X_dev2[b][xo:xo + nx].view(L["x"].shape), Y_dev2[b][yo:yo + ny].view(L["y"].shape)))
            xo += nx
            yo += ny
        pipe_views.append(vb)

    def compute_on(b):
        for L, (xv, yv) in zip(layers, pipe_views[b]):
            layer(L, xv, yv)

    def e2e_per_layer_step():
        for L in layers:
            L["x"].copy_(L["x_host"], non_blocking=True)
            layer(L)
            L["y_host"].copy_(L["y"], non_blocking=True)

    for L in layers:                  # q, s for the GEMM-only graphs
        sbm.quant_act(L["x"], L["q"], L["s"])
    g_step = capture(step)
    g_gemm = capture(gemm_only)
    g_quant = capture(quant_only)
    g_two = capture(two_launch_step) if fused else None
    g_e2e = capture(e2e_step)
    g_e2e_layer = capture(e2e_per_layer_step)
    g_comp = [capture(lambda: compute_on(0)), capture(lambda: compute_on(1))]

    sampler = ClockSampler(local)
    sampler.start()
    t_step = time_graph(g_step, args.steps, args.warmup, world, sampler)
    clocks = sampler.stop()
    t_step = max_over_ranks(t_step, world)
    t_gemm = max_over_ranks(time_graph(g_gemm, args.steps, args.warmup, world), world)
    t_quant = max_over_ranks(time_graph(g_quant, args.steps, args.warmup, world), world)
    t_two = max_over_ranks(time_graph(g_two, args.steps, args.warmup, world), world) if fused else None
    t_e2e = max_over_ranks(time_graph(g_e2e, args.steps, args.warmup, world), world)
    t_e2e_layer = max_over_ranks(time_graph(g_e2e_layer, args.steps, args.warmup, world), world)
    t_e2e_pipe = max_over_ranks(time_pipelined_e2e(g_comp, X_dev2, X_host, Y_dev2, Y_host2, args.steps,
                                                   args.warmup, world), world)
    assert sbm.last_device_status() == 0, "a kernel reported a bounded wait running out"

    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    value = step_bytes * world * args.steps / t_step / 1e9
    n_launch = len(layers)
    # the dominant kernel: the fused kernel is the whole step; otherwise the GEMM
    t_dom = t_step if fused else t_gemm
    dom_launch_s = t_dom / (args.steps * n_launch)
    achieved = step_bytes / (t_dom / args.steps) / 1e9
    dom_name = "sherry_decode_kernel<1,true,RT>" if fused else f"sherry_gemm_{kernel}"
    traffic = load_traffic(dom_name, step_bytes / n_launch)
    h2d = sum(L["x"].numel() * 4 for L in layers)
    d2h = sum(L["y"].numel() * 4 for L in layers)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic: seeded splitmix64 + Box-Muller; W ~ N(0,0.02) fp32 packed to 5-bit codes, "
                "x ~ N(0,1) fp32",
        "config": {
            "workload": "decode GEMV M=1 over Llama-3-8B-shaped projections (K,N) = (4096,4096), "
                        "(4096,14336), (14336,4096), rotated across 32 seeded layer copies",
            "M": 1, "copies_per_gpu": args.copies, "layers_per_step": n_launch,
            "bytes_per_step": step_bytes, "packed_weight_bytes_per_step": code_bytes,
            "l2": "inputs larger than L2: %.0f MB of packed weights per step vs 126 MB L2" % (code_bytes / 1e6),
            "launch": ("one CUDA graph per step: sherry_linear per layer (activation quantiser fused "
                       "into the decode GEMM, one launch)") if fused else
                      "one CUDA graph per step: sherry_quant_act + GEMM per layer", "kernel": kernel,
            "parallelism": f"replicas x{world} (independent layer copies per GPU)",
        },
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 2), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
            "kernel": dom_name,
            "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
            "avg_launch_us": round(dom_launch_s * 1e6, 3),
            "algorithmic_bytes_per_launch": round(step_bytes / n_launch),
            "frac_of_8TBs_spec": round(achieved / 8000.0, 4),
        },
        "separate_kernels": {
            "quant_act_avg_launch_us": round(t_quant / (args.steps * n_launch) * 1e6, 3),
            "gemm_avg_launch_us": round(t_gemm / (args.steps * n_launch) * 1e6, 3),
            "gemm_gbs": round(step_bytes / (t_gemm / args.steps) / 1e9, 2),
            "two_launch_step_gbs": (round(step_bytes * args.steps / t_two / 1e9, 2) if fused else None),
        },
        "e2e": {"value": round(step_bytes * world * args.steps / t_e2e_pipe / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": ("per step: one H2D copy of the step's layer inputs from one pinned host buffer "
                         "(copy stream 1) -> "
                         + ("sherry_linear" if fused else f"sherry_quant_act -> sherry_gemm[{kernel}]")
                         + " per layer on device views (one CUDA graph) -> one D2H copy of the step's "
                         "outputs into pinned host memory (copy stream 2); two device buffer pairs, so "
                         "step k's copies overlap the compute of steps k - 1 and k + 1; timed from "
                         "before the first H2D to after the last D2H"),
                "serial_gbs": round(step_bytes * world * args.steps / t_e2e / 1e9, 2),
                "serial_path": ("H2D of the step's inputs, the layer calls, D2H of its outputs, all in one "
                                "CUDA graph per step, one step after another"),
                "per_layer_copies_gbs": round(step_bytes * world * args.steps / t_e2e_layer / 1e9, 2),
                "per_layer_copies_path": "H2D of x, the layer call, D2H of y, around every layer call"},
        "gpu_launches": (1 if fused else 2) * n_launch * args.steps,
        "clocks": clocks,
    }
    del g_step, g_gemm, g_quant, g_two, g_e2e, g_e2e_layer, g_comp
    if not args.no_extras:
        out["extra"] = extras(args, layers, kernel, peaks, peak_src, world,
                              sm_mhz=(clocks or {}).get("sm_mhz"))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        out["cpu_lut"] = cpu_lut_baseline(min(args.cpu_seconds, 3.0))
    return out


def load_traffic(kernel: str, avg_algorithmic_bytes: float):
    """DRAM bytes per launch of the dominant kernel: the committed ncu capture
    (profiles/traffic.json, one launch of one layer shape) scaled to the
    average launch of the step by algorithmic bytes.  None when the capture
    is not of the kernel this run times."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(kernel)
        if not e:
            return None
        return round(e["dram_bytes"] / e["algorithmic_bytes"] * avg_algorithmic_bytes)
    except Exception:
        return None


def timed_single_launches(fn, flush, reps: int = 5):
    """Median of `reps` single launches of fn, each after an L2 flush (CUDA
    events on the current stream)."""
    import torch
    for _ in range(3):
        fn()
    times = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(times)


def device_copies(native, alpha, count: int):
    """`count` weight copies on the device: the given ones first, then device
    clones of them (distinct memory, so every launch streams its own bytes)."""
    out = list(zip(native, alpha))
    i = 0
    while len(out) < count:
        nat, al = out[i % len(native)]
        out.append((nat.clone(), al))
        i += 1
    return out


def gemm_tops_line(M, K, N, cfg, flush, int8_peak, kernel):
    """One GEMM of config `cfg`'s distributions through sherry_gemm (int8
    activations already quantised): single launches after an L2 flush;
    int-TOPS counted as 2 M N K dense-equivalent operations."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    codes, alpha = sbm.pack(synth.config_weights(cfg, 0, K, N))
    native = sbm.repack(torch.from_numpy(codes).cuda(), N, K)
    al = torch.from_numpy(alpha).cuda()
    q, s = sbm.quant_act(torch.from_numpy(synth.config_activations(cfg, 0, M, K)).cuda())
    y = torch.empty((M, N), device="cuda")
    t = timed_single_launches(lambda: sbm.gemm(q, s, native, al, N, out=y, kernel=kernel), flush)
    tops = 2.0 * M * N * K / t / 1e12
    return {"us": round(t * 1e6, 2), "int_tops_dense_equiv": round(tops, 1),
            "frac_of_int8_peak": round(tops / int8_peak, 4), "frac_of_4500_spec": round(tops / 4500.0, 4),
            "algorithmic_add_tops": round(0.75 * M * N * K / t / 1e12, 1)}


def config4_m1_l2_resident(args, world, hbm_peak):
    """Config 4 at M = 1: one 36.7 MB weight matrix called back to back, so
    its codes stay in L2 (126 MB); labelled as such, not an HBM figure."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    K, N = 8192, 28672
    codes, alpha = sbm.pack(synth.config_weights(4, 0, K, N))
    native = sbm.repack(torch.from_numpy(codes).cuda(), N, K)
    al = torch.from_numpy(alpha).cuda()
    x = torch.from_numpy(synth.config_activations(4, 0, 1, K)).cuda()
    y = torch.empty((1, N), device="cuda")

    def fn():
        for _ in range(8):
            sbm.linear(x, native, al, N, out=y)
    g = capture(fn)
    reps = max(3, args.steps // 20)
    t = max_over_ranks(time_graph(g, reps, 2, world), world)
    call = t / (8 * reps)
    gbs = algorithmic_bytes(1, K, N) / call / 1e9
    return {"us_per_call": round(call * 1e6, 3), "gbs": round(gbs, 1),
            "l2_resident": "36.7 MB of codes called back to back: served from L2, not HBM",
            "frac_of_hbm_peak_for_context": round(gbs / hbm_peak, 4)}


def decode_per_shape(args, world, hbm_peak):
    """M = 1 through sherry_linear, one projection shape at a time, repeated
    over device copies of at least 600 MB per shape (every weight byte from
    HBM): us per call, GB/s and fraction of the HBM peak."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    out = {}
    for K, N in PROJ_SHAPES:
        per = N * K * 5 // 32
        count = max(16, -(-600_000_000 // per))
        base_n, base_a = [], []
        for c in range(4):
            codes, alpha = sbm.pack(synth.config_weights(1, c, K, N))
            base_n.append(sbm.repack(torch.from_numpy(codes).cuda(), N, K))
            base_a.append(torch.from_numpy(alpha).cuda())
        mats = device_copies(base_n, base_a, count)
        x = torch.from_numpy(synth.config_activations(1, 0, 1, K)).cuda()
        y = torch.empty((1, N), device="cuda")

        def fn():
            for nat, al in mats:
                sbm.linear(x, nat, al, N, out=y)
        g = capture(fn)
        reps = max(3, args.steps // 20)
        t = max_over_ranks(time_graph(g, reps, 2, world), world)
        call = t / (reps * count)
        gbs = algorithmic_bytes(1, K, N) / call / 1e9
        out[f"K{K}_N{N}"] = {"us_per_call": round(call * 1e6, 3), "gbs": round(gbs, 1),
                             "frac": round(gbs / hbm_peak, 4), "copies": count}
        del g, mats, base_n
        torch.cuda.empty_cache()
    return out


def long_call(args, world, hbm_peak, sm_mhz):
    """One long M = 1 call (K = 8192 -> N = 28672, 36.7 MB of codes) through
    sherry_linear, rotated over 16 device copies (587 MB > L2): the
    throughput the decode kernel sustains once per-call latency is a small
    part of the call.  groups_per_sm_clock = (N K / 4) / (time x SMs x SM
    clock), with the clock measured in the headline's timed window."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    K, N, copies = 8192, 28672, 16
    base_n, base_a = [], []
    for c in range(2):
        codes, alpha = sbm.pack(synth.config_weights(4, c, K, N))
        base_n.append(sbm.repack(torch.from_numpy(codes).cuda(), N, K))
        base_a.append(torch.from_numpy(alpha).cuda())
    mats = device_copies(base_n, base_a, copies)
    x = torch.from_numpy(synth.config_activations(4, 0, 1, K)).cuda()
    y = torch.empty((1, N), device="cuda")

    def fn():
        for nat, al in mats:
            sbm.linear(x, nat, al, N, out=y)
    g = capture(fn)
    reps = max(3, args.steps // 20)
    t = max_over_ranks(time_graph(g, reps, 2, world), world)
    call = t / (reps * copies)
    gbs = algorithmic_bytes(1, K, N) / call / 1e9
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    res = {"shape": "M=1, K=8192 -> N=28672 (config 4's projection), sherry_linear",
           "copies": copies, "bytes_per_pass": algorithmic_bytes(1, K, N) * copies,
           "us_per_call": round(call * 1e6, 3), "gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4)}
    if sm_mhz:
        res["groups_per_sm_clock"] = round((N * K / 4) / (call * sms * sm_mhz * 1e6), 2)
        res["sm_mhz_used"] = sm_mhz
    del g, mats, base_n
    torch.cuda.empty_cache()
    return res


def extras(args, layers, kernel, peaks, peak_src, world, sm_mhz=None):
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    res = {}
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # small-batch decode on the same weights (M = 4, 8, 16, 32): the public
    # call, sherry_linear from fp32 activations (or the named GEMM kernel)
    small = {}
    for M in (4, 8, 16, 32):
        xs, xf = {}, {}
        for L in layers:
            key = L["K"]
            if key not in xs:
                xf[key] = torch.from_numpy(synth.config_activations(2, 0, M, key)).cuda()
                xs[key] = sbm.quant_act(xf[key])
        ys = {L["N"]: torch.empty((M, L["N"]), device="cuda") for L in layers}

        def fn():
            for L in layers:
                if kernel == "auto":
                    sbm.linear(xf[L["K"]], L["native"], L["alpha"], L["N"], out=ys[L["N"]])
                else:
                    q, s = xs[L["K"]]
                    sbm.gemm(q, s, L["native"], L["alpha"], L["N"], out=ys[L["N"]], kernel=kernel)
        g = capture(fn)
        reps = max(3, args.steps // 4)
        t = max_over_ranks(time_graph(g, reps, 2, world), world)
        nb = sum(algorithmic_bytes(M, L["K"], L["N"]) for L in layers)
        gbs = nb * reps / t / 1e9
        small[str(M)] = {"gbs": round(gbs, 2), "frac": round(gbs / hbm_peak, 4),
                         "us_per_call": round(t / (reps * len(layers)) * 1e6, 3)}
        del g
    res["small_batch_decode"] = small
    res["small_batch_step"] = ("sherry_linear per layer call (fp32 activations in: the dispatch of the library)"
                               if kernel == "auto" else f"GEMM kernel {kernel} only")
    res["decode_per_shape_M1"] = decode_per_shape(args, world, hbm_peak)
    res["long_call_M1"] = long_call(args, world, hbm_peak, sm_mhz)
    # prefill GEMM, M = 2048 (L2 flushed between timed launches)
    int8_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * NOMINAL_INT8_OVER_BF16
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    pre = {}
    for K, N in [(4096, 14336), (14336, 4096)]:
        pre[f"K{K}_N{N}"] = gemm_tops_line(2048, K, N, 3, flush, int8_peak, kernel)
    res["prefill_M2048"] = pre
    # mid-size M on the tensor cores (64-, 128-token tiles), K = 4096 -> N = 14336
    res["prefill_mid_M"] = {str(M): gemm_tops_line(M, 4096, 14336, 3, flush, int8_peak, kernel)
                            for M in (64, 128, 512, 1024)}
    # the heavy-tailed stress shape (K = 8192 -> N = 28672): M = 1 keeps its
    # 36.7 MB of codes in the 126 MB L2 across back-to-back calls (labelled);
    # M = 128 and 4096 are single launches after an L2 flush
    c4 = {"M128": gemm_tops_line(128, 8192, 28672, 4, flush, int8_peak, kernel),
          "M4096": gemm_tops_line(4096, 8192, 28672, 4, flush, int8_peak, kernel)}
    c4["M1_l2_resident"] = config4_m1_l2_resident(args, world, hbm_peak)
    res["config4_K8192_N28672"] = c4
    res["int8_peak_tops"] = {"value": round(int8_peak, 1),
                             "source": f"{peak_src} bf16_tflops x nominal int8/bf16 ratio 2"}
    # practical dense INT8 tensor throughput of the library GEMM on this machine
    a = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device="cuda")
    b = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device="cuda").t()
    for _ in range(3):
        torch._int_mm(a, b)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(10):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize()
    lib_tops = 2.0 * 8192 ** 3 * 10 / (e0.elapsed_time(e1) / 1e3) / 1e12
    res["int8_library_gemm_tops"] = {"value": round(lib_tops, 1), "how": "torch._int_mm 8192^3, 10 launches"}
    for v in pre.values():
        v["frac_of_library_int8"] = round(v["int_tops_dense_equiv"] / lib_tops, 4)
    try:                                        # a second workload: its failure is reported, not fatal
        res["w4a8"] = w4a8_extras(args, flush, int8_peak, lib_tops, world)
    except Exception as e:
        res["w4a8"] = {"error": f"{type(e).__name__}: {e}"}
    return res


def w4a8_bytes(M: int, K: int, N: int) -> int:
    """SINT4 weights + fp32 channel scales + int8 activations + token scales."""
    return N * K // 2 + 4 * N + M * K + 4 * M


def w4a8_extras(args, flush, int8_peak, lib_tops, world):
    """W4A8 FastGEMM (SINT4 weights x int8 activations) on the tensor-core
    kernel: small M over a rotation of weight copies larger than twice L2,
    and prefill launches after an L2 flush."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    out = {"kernel": "sherry_w4a8_gemm: sherry_gemm_tc_kernel<BN, SC, int4 weights> for every M; "
                     "small M also timed on the CUDA-core comparison GEMV (sherry_w4a8_gemm_gemv)",
           "weights": "synthetic N(0, 0.02) quantised per channel to SINT4 (S = max|w| / 7)"}
    K, N = 4096, 14336
    copies = 9                                    # 9 x 29.4 MB = 264 MB > 2 x L2
    mats = []
    for c in range(copies):
        w4, scale = sbm.w4a8_pack(synth.config_weights(1, c, K, N))
        mats.append((sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K), torch.from_numpy(scale).cuda()))
    small = {}
    for M, kern in ((1, "auto"), (4, "auto"), (16, "auto"), (1, "gemv"), (4, "gemv")):
        q, s = sbm.quant_act(torch.from_numpy(synth.config_activations(2, 0, M, K)).cuda())
        y = torch.empty((M, N), device="cuda")

        def fn():
            for nat, sc in mats:
                sbm.w4a8_gemm(q, s, nat, sc, N, out=y, kernel=kern)
        g = capture(fn)
        reps = max(3, args.steps // 4)
        t = max_over_ranks(time_graph(g, reps, 2, world), world)
        gbs = w4a8_bytes(M, K, N) * copies * reps / t / 1e9
        key = str(M) if kern == "auto" else f"{M}_gemv"
        small[key] = {"gbs": round(gbs, 1), "us_per_call": round(t / (copies * reps) * 1e6, 2)}
        del g
    out[f"small_M_K{K}_N{N}_rotation{copies}"] = small
    pre = {}
    for K, N in [(4096, 14336), (14336, 4096)]:
        M = 2048
        w4, scale = sbm.w4a8_pack(synth.config_weights(3, 0, K, N))
        nat = sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K)
        sc = torch.from_numpy(scale).cuda()
        q, s = sbm.quant_act(torch.from_numpy(synth.config_activations(3, 0, M, K)).cuda())
        y = torch.empty((M, N), device="cuda")
        for _ in range(3):
            sbm.w4a8_gemm(q, s, nat, sc, N, out=y)
        times = []
        for _ in range(5):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            sbm.w4a8_gemm(q, s, nat, sc, N, out=y)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / 1e3)
        t = statistics.median(times)
        tops = 2.0 * M * N * K / t / 1e12
        pre[f"K{K}_N{N}"] = {"us": round(t * 1e6, 1), "int_tops": round(tops, 1),
                             "frac_of_int8_peak": round(tops / int8_peak, 4),
                             "frac_of_library_int8": round(tops / lib_tops, 4)}
    out["prefill_M2048"] = pre
    return out


def profile_case(args):
    """A few launches of one layer shape, small enough for a full ncu capture."""
    import torch
    import sparse_bit_matmul_b200 as sbm
    import synth
    torch.cuda.set_device(0)
    sbm.load()
    if args.profile_case == "w4a8":
        M, K, N = 2048, 4096, 14336
        w4, scale = sbm.w4a8_pack(synth.config_weights(3, 0, K, N))
        nat = sbm.w4a8_repack(torch.from_numpy(w4).cuda(), N, K)
        sc = torch.from_numpy(scale).cuda()
        q, s = sbm.quant_act(torch.from_numpy(synth.config_activations(3, 0, M, K)).cuda())
        y = torch.empty((M, N), device="cuda")
        for _ in range(4):
            sbm.w4a8_gemm(q, s, nat, sc, N, out=y)
        torch.cuda.synchronize()
        status = sbm.last_device_status()
        print(json.dumps({"profile_case": "w4a8", "M": M, "K": K, "N": N, "launches": 4,
                          "device_status": status}))
        return 0 if status == 0 else 1
    M = {"decode": 1, "small": 16, "prefill": 2048, "long": 1}[args.profile_case]
    K, N = (8192, 28672) if args.profile_case == "long" else (4096, 14336)
    copies = 2 if args.profile_case == "long" else (8 if M <= 16 else 1)
    layers = []
    for c in range(copies):
        codes, alpha = sbm.pack(synth.config_weights(1 if M <= 16 else 3, c, K, N))
        layers.append((sbm.repack(torch.from_numpy(codes).cuda(), N, K), torch.from_numpy(alpha).cuda()))
    x = torch.from_numpy(synth.config_activations(1 if M == 1 else (2 if M <= 16 else 3), 0, M, K)).cuda()
    q, s = sbm.quant_act(x)
    y = torch.empty((M, N), device="cuda")
    kernel = "auto" if args.impl == "reference" else args.impl
    for _ in range(4):
        for nat, al in layers:
            if kernel == "auto" and M == 1:
                sbm.linear(x, nat, al, N, out=y)
            else:
                sbm.gemm(q, s, nat, al, N, out=y, kernel=kernel)
    torch.cuda.synchronize()
    status = sbm.last_device_status()
    print(json.dumps({"profile_case": args.profile_case, "M": M, "K": K, "N": N, "copies": copies,
                      "launches": 4 * copies, "kernel": kernel, "device_status": status}))
    return 0 if status == 0 else 1


def main(argv=None):
    args = parse_args(argv)
    if args.profile_case:
        return profile_case(args)
    world, rank, local = dist_setup(args.gpus, need_cuda=(args.impl != "reference"))
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
            return 0
        out = run_gpu(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
