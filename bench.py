#!/usr/bin/env python
"""Benchmark of the fused MoE layer (forward + backward) on B200.

One step = one full pass of the layer's hot path: routing (top-k, histogram,
scan, permutation), the dispatch (x copied into the expert-sorted layout; under
MXFP8 gathered inside the GEMM), the gate/up grouped GEMM with the SwiGLU
epilogue, the down grouped GEMM and the slot-ordered combine, and the backward
(grad_out sorted, down dgrad + SwiGLU backward, both weight gradients, gate/up
dgrad and the slot-ordered scatter into dx, routing-score gradients), all
through the C ABI of libmoe.so on device-resident synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

N > 1 is launched by torchrun; every rank runs an independent replica of the
layer on its own GPU (the layer has no data-path exchange on one GPU), timing
is the max over ranks and ``value`` counts the work of all ranks.
``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).  Rank 0 prints one JSON line.
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
sys.path.insert(0, ROOT)

METRIC = "fused MoE layer fwd+bwd TFLOP/s & % of bf16 tensor peak (Qwen3-30B-A3B shape)"
UNIT = "TFLOP/s"
# workloads timed after the headline one and reported in the same JSON line
OTHER_WORKLOADS = ("qwen3_235b_a22b", "qwen3_30b_a3b_skew", "qwen3_30b_a3b_mxfp8", "tiny")
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="qwen3_30b_a3b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="skip sampling nvidia-smi during the timed region")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-recompute", action="store_true", help="skip the recompute-mode timing")
    ap.add_argument("--no-routing-sweep", action="store_true",
                    help="skip the routing-only timing over token counts")
    ap.add_argument("--cpu-tokens", type=int, default=0, help="oracle sample size (0 = auto)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other workloads (reported under 'configs')")
    ap.add_argument("--override", default="", help="comma list of size overrides, e.g. T=4096,E=32 "
                                                     "(smaller profiling cases; not a bench workload)")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(ms, pg, device):
    """The slowest rank's time (every rank calls this, in the same order)."""
    if pg is None:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step_per_rank, world, ms_per_step):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return flops_per_step_per_rank * world / (ms_per_step * 1e-3) / 1e12


def l2_note(cfg):
    wbytes = cfg["E"] * 3 * cfg["d"] * cfg["I"] * 2
    return f"inputs larger than L2 (expert weights {wbytes / 1e9:.2f} GB), no flush"


def routing_sweep(M, IN, dev, stream, peak_gbs, E, k, Ts=(16384, 65536, 262144, 524288, 1000000), reps=10):
    """Routing alone (moe_route: top-k, histogram, scan, permutation) at growing
    token counts, each call timed by itself with L2 flushed before it (a 256 MiB
    write), so that the logits come from HBM.  The largest count, 10^6 tokens,
    is near the most the library's 32-bit sorted-layout indices allow at k = 8.  The activation buffers that
    routing does not touch are left out (alloc_saved_routing) and the hidden
    sizes are small, so that the workspace stays small."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    for T in Ts:
        sh = M.make_shape(T, 128, E, k, 128)
        saved = M.alloc_saved_routing(sh, dev)
        f, _ = M.workspace_size(sh)
        ws = torch.empty(f, dtype=torch.uint8, device=dev)
        g = torch.Generator(device="cpu").manual_seed(1000 + T)
        logits = torch.randn(T, E, generator=g, dtype=torch.float32).to(dev)
        for _ in range(3):
            M.route(sh, logits, saved, ws, stream)
        times = []
        torch.cuda.nvtx.range_push(f"route_sweep_T{T}")  # for profilers: ncu --nvtx --nvtx-include route_sweep_T<T>/
        for _ in range(reps):
            flush.zero_()
            e0.record(stream)
            M.route(sh, logits, saved, ws, stream)
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        torch.cuda.nvtx.range_pop()
        if M.get_status(ws, stream) != 0:
            raise SystemExit(f"device status {M.get_status(ws, stream)} in the routing sweep (T={T})")
        us = statistics.median(times) * 1e3
        nbytes = IN.routing_bytes(T, E, k)
        out.append({"T": T, "us": us, "bytes": nbytes, "gbs": nbytes / (us * 1e-6) / 1e9,
                    "frac": nbytes / (us * 1e-6) / 1e9 / peak_gbs})
        del saved, ws, logits
    return out


def workload_config(name, cfg, extra=None):
    c = {"workload": name, "T": cfg["T"], "d": cfg["d"], "E": cfg["E"], "top_k": cfg["k"], "I": cfg["I"]}
    if "zipf_s" in cfg:
        c["zipf_s"] = cfg["zipf_s"]
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi samples of one GPU every 25 ms, each stamped with the host
    time it arrived; stop() keeps those inside the [mark_start, mark_end]
    window (the timed region), or, when the region is shorter than the
    sampling interval and none fell inside it, the sample nearest to it."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.reader = None
        self.t0 = self.t1 = None

    def start(self, wait_s=5.0):
        """Start sampling; returns once the first sample has arrived (or after wait_s)."""
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "25",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return

        def read():
            for line in self.proc.stdout:
                self.lines.append((time.time(), line))

        self.reader = threading.Thread(target=read, daemon=True)
        self.reader.start()
        t_end = time.time() + wait_s
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        if self.reader is not None:
            self.reader.join(timeout=5)
        stamped = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                stamped.append((t, dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                        hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8])))
            except ValueError:
                continue
        if not stamped:
            return None
        window = "timed region"
        if self.t0 is not None and self.t1 is not None:
            inside = [r for t, r in stamped if self.t0 <= t <= self.t1]
            if not inside:
                mid = 0.5 * (self.t0 + self.t1)
                inside = [min(stamped, key=lambda tr: abs(tr[0] - mid))[1]]
                window = "nearest sample to the timed region (shorter than the sampling interval)"
            rows = inside
        else:
            rows = [r for _, r in stamped]
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() in ("active", "1"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "samples": len(loaded), "power_w_max": max(r["power"] for r in rows), "reasons": sorted(reasons),
                "window": window}


# ----------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------
def oracle_threads(cfg):
    """Threads the oracle step uses: the C++ oracle splits the experts over the
    host's hardware threads; the numpy MXFP8 oracle uses the BLAS pool."""
    if cfg.get("dtype") == "mxfp8":
        try:
            from threadpoolctl import threadpool_info
            n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
            if n:
                return int(max(n))
        except Exception:
            pass
        return os.cpu_count() or 1
    from oracle import cpp_oracle as C
    return max(1, min(cfg["E"], C.hardware_threads()))


def oracle_kind(cfg):
    if cfg.get("dtype") == "mxfp8":
        return "fp64 numpy MXFP8 oracle"
    return "fp64 C++ oracle (experts split over std::threads; its backward recomputes h)"


def oracle_sample(cfg, inp, n_tokens):
    """Inputs of the first n_tokens tokens as float64 arrays (weights stay whole)."""
    import numpy as np
    sl = slice(0, n_tokens)
    x = inp["x"][sl].float().numpy().astype(np.float64)
    lg = inp["logits"][sl].numpy()
    gout = inp["gout"][sl].float().numpy().astype(np.float64)
    return x, lg, gout


def time_oracle_step(cfg, inp, wgu64, wd64, n_tokens):
    x, lg, gout = oracle_sample(cfg, inp, n_tokens)
    k = cfg["k"]
    if cfg.get("dtype") == "mxfp8":
        from oracle import moe_oracle as O
        t0 = time.perf_counter()
        f = O.forward_mx(x, lg, wgu64, wd64, k)
        O.backward_mx(x, lg, wgu64, wd64, k, gout, f)
        return time.perf_counter() - t0
    from oracle import cpp_oracle as C
    nt = oracle_threads(cfg)
    t0 = time.perf_counter()
    C.forward(x, lg, wgu64, wd64, k, nthreads=nt, keep_intermediates=False)
    C.backward(x, lg, wgu64, wd64, k, gout, nthreads=nt)
    return time.perf_counter() - t0


def oracle_weights(inp):
    import numpy as np
    return inp["wgu"].float().numpy().astype(np.float64), inp["wd"].float().numpy().astype(np.float64)


def cpu_baseline(cfg, inp, n_tokens=0, budget_s=15.0):
    """Oracle fwd+bwd throughput on the first n tokens; n grows until one pass takes ~budget_s/2."""
    from grouped_gemm_route_b200 import inputs as IN
    wgu64, wd64 = oracle_weights(inp)
    n = n_tokens or 256
    dt = time_oracle_step(cfg, inp, wgu64, wd64, n)
    while not n_tokens and dt < budget_s / 2 and n < cfg["T"]:
        n = min(cfg["T"], n * 2)
        dt = time_oracle_step(cfg, inp, wgu64, wd64, n)
    dims = {k: cfg[k] for k in ("d", "E", "k", "I")}
    flops = IN.flops_fwd(T=n, **dims) + IN.flops_bwd(T=n, **dims)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle_threads(cfg), "kind": "oracle",
            "sample": f"{oracle_kind(cfg)}, forward+backward of the first {n} of {cfg['T']} tokens "
                      f"(all experts' weights), {dt:.2f} s"}, n, dt


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    from grouped_gemm_route_b200 import inputs as IN
    cfg, inp = IN.make_workload(args.workload, seed=args.seed, device="cpu")
    wgu64, wd64 = oracle_weights(inp)
    # per-step sample sized so that warmup + steps finish in a few minutes
    probe = 64
    dt = time_oracle_step(cfg, inp, wgu64, wd64, probe)
    per_step_budget = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    n = args.cpu_tokens or int(min(cfg["T"], max(16, probe * per_step_budget / max(dt, 1e-3) * 0.8)))
    for _ in range(args.warmup):
        time_oracle_step(cfg, inp, wgu64, wd64, n)
    times = [time_oracle_step(cfg, inp, wgu64, wd64, n) for _ in range(args.steps)]
    total = sum(times)
    dims = {k: cfg[k] for k in ("d", "E", "k", "I")}
    flops = (IN.flops_fwd(T=n, **dims) + IN.flops_bwd(T=n, **dims)) * args.steps
    value = flops / total / 1e12
    sample = f"{oracle_kind(cfg)}, forward+backward of the first {n} of {cfg['T']} tokens per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.workload, cfg, {"oracle_tokens_per_step": n}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(cfg), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# timing helpers (our arm)
# ----------------------------------------------------------------------------
def timed_loop(step, n_steps, stream, dev, barrier, clocks=None):
    """Device time of n_steps calls of step(), CUDA events on the launching
    stream, a barrier and a synchronize on both sides; ms per step.  clocks
    (a ClockSampler) gets the host times between the two synchronizes."""
    import torch
    barrier()
    torch.cuda.synchronize(dev)
    if clocks is not None:
        clocks.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n_steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if clocks is not None:
        clocks.mark_end()
    barrier()
    return t0.elapsed_time(t1) / n_steps


def graph_loop(step_on, n_steps, dev, barrier):
    """The step captured once in a CUDA graph on a side stream (after an eager
    warm-up there) and replayed n_steps times: ms per step from CUDA events on
    that stream, or the reason the capture failed."""
    import torch
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    try:
        with torch.cuda.stream(s):
            step_on(s)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step_on(s)
        with torch.cuda.stream(s):
            graph.replay()
        torch.cuda.synchronize(dev)
    except Exception as exc:  # noqa: BLE001 -- reported, not hidden
        torch.cuda.synchronize(dev)
        return None, f"{type(exc).__name__}: {exc}"[:200]
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        t0.record(s)
        for _ in range(n_steps):
            graph.replay()
        t1.record(s)
    torch.cuda.synchronize(dev)
    barrier()
    del graph
    return t0.elapsed_time(t1) / n_steps, None


def profiled_loop(M, step, n_steps, stream, dev, barrier):
    """The same steps with the library's per-kernel events on: returns
    {kernel: (total ms, launches)} and the loop's ms per step."""
    M.profile_read()
    M.profile_enable(True)
    try:
        ms = timed_loop(step, n_steps, stream, dev, barrier)
    finally:
        M.profile_enable(False)
    return M.profile_read(), ms


def gemm_flops_per_launch(T, d, k, I):
    """Algorithmic FLOPs of one launch of each grouped GEMM (P = T*k pairs)."""
    P = T * k
    return {"gemm_gateup_fwd": 4.0 * P * d * I, "gemm_down_fwd_combine": 2.0 * P * I * d,
            "gemm_down_dgrad": 2.0 * P * d * I, "gemm_down_wgrad": 2.0 * P * d * I,
            "gemm_gateup_dgrad_scatter": 4.0 * P * d * I, "gemm_gateup_wgrad": 4.0 * P * d * I}


def kernel_breakdown(per_kernel, n_steps):
    total = sum(v[0] for v in per_kernel.values()) or 1.0
    return {n: {"ms_per_step": v[0] / n_steps, "share": v[0] / total, "launches": v[1]}
            for n, v in per_kernel.items() if v[1]}


def tensor_peaks(peaks, src, mx, clk):
    """The tensor peak a GEMM is compared with, and the other one.

    The measured burst figure (cuBLAS timed alone) applies when the timed
    region ran at the maximum SM clock; the sustained one (a seconds-long loop
    under the power cap) when the clock record shows the cap holding the clock
    down.  MXFP8 runs at twice the bf16 rate (derived, not measured)."""
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    at_max = bool(clk) and clk.get("sm_mhz", 0) >= 0.97 * clk.get("sm_max_mhz", 1e9)
    scale, tag = (2.0, "2 x ") if mx else (1.0, "")
    note = " (derived FP8 rate)" if mx else ""
    if at_max or not clk:
        return (scale * burst, f"{tag}{src} bf16_tflops (burst; timed region at max SM clock){note}",
                {"sustained": scale * sust})
    return (scale * sust, f"{tag}{src} bf16_tflops_sustained (clock held below max){note}",
            {"burst": scale * burst})


def time_other_config(M, IN, name, n_steps, n_warmup, dev, stream, barrier, peaks, peak_src, seed, clk_gpu):
    """ms per step, TFLOP/s, the GEMMs' share of the tensor peak and the clocks
    of one more workload, timed the same way as the headline one (events off),
    its breakdown from a second, profiled loop.  Frees its buffers on return."""
    import torch
    cfg = dict(IN.WORKLOADS[name])
    host = IN.make_inputs(seed=seed, device="cpu", **cfg)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    x, lg, wgu, wd, gout = (host[n].to(dev) for n in ("x", "logits", "wgu", "wd", "gout"))
    del host
    mx = cfg.get("dtype") == "mxfp8"
    layer = M.MoELayer(T, d, E, k, I, device=str(dev), dtype=M.MOE_MXFP8 if mx else M.MOE_BF16)

    def step():
        layer.forward(x, lg, wgu, wd, stream)
        layer.backward(gout, x, wgu, wd, True, stream)

    for _ in range(max(3, n_warmup)):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(clk_gpu)
    if clk_gpu is not None:
        clocks.start()
    ms = timed_loop(step, n_steps, stream, dev, barrier, clocks if clk_gpu is not None else None)
    clk = clocks.stop() if clk_gpu is not None else None
    per_kernel, _ = profiled_loop(M, step, n_steps, stream, dev, barrier)
    g_ms, g_err = graph_loop(lambda s: (layer.forward(x, lg, wgu, wd, s), layer.backward(gout, x, wgu, wd, True, s)),
                             n_steps, dev, barrier)
    status = layer.status(stream)
    if status != 0:
        raise SystemExit(f"device status {status} in workload {name}")
    flops = IN.flops_fwd(**cfg) + IN.flops_bwd(**cfg)
    gf = gemm_flops_per_launch(T, d, k, I)
    gemm_ms = sum(per_kernel.get(n, (0.0, 0))[0] for n in gf) / n_steps
    peak, note, _ = tensor_peaks(peaks, peak_src, mx, clk)
    tflops = flops / (ms * 1e-3) / 1e12
    out = {"ms_per_step": ms, "value": tflops, "unit": UNIT, "steps": n_steps,
           "frac_of_peak": tflops / peak,
           "gemm_only_frac": (flops / (gemm_ms * 1e-3) / 1e12) / peak if gemm_ms else None,
           "gemm_ms_per_step": gemm_ms, "peak": peak, "peak_source": note, "clocks": clk,
           "config": workload_config(name, cfg), "dtype": "mxfp8 (e4m3, ue8m0/32)" if mx else "bf16",
           "kernels": {n: v["ms_per_step"] for n, v in kernel_breakdown(per_kernel, n_steps).items()},
           "graph": ({"ms_per_step": g_ms, "value": flops / (g_ms * 1e-3) / 1e12} if g_ms else {"unavailable": g_err})}
    if "zipf_s" in cfg:
        counts = layer.saved["counts"].cpu()
        out["routing_skew"] = {"max_count": int(counts.max()), "empty_experts": int((counts == 0).sum())}
    del layer, x, lg, wgu, wd, gout
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch

    from grouped_gemm_route_b200 import inputs as IN
    from grouped_gemm_route_b200 import moe as M

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    cfg = dict(IN.WORKLOADS[args.workload])
    for item in filter(None, args.override.split(",")):
        key, val = item.split("=")
        cfg[key] = int(val)
    host = IN.make_inputs(seed=args.seed + rank, device="cpu", **cfg)
    T, d, E, k, I = (cfg[n] for n in ("T", "d", "E", "k", "I"))
    x, lg, wgu, wd, gout = (host[n].to(dev) for n in ("x", "logits", "wgu", "wd", "gout"))
    mx = cfg.get("dtype") == "mxfp8"
    dtype_code = M.MOE_MXFP8 if mx else M.MOE_BF16
    layer = M.MoELayer(T, d, E, k, I, device=str(dev), dtype=dtype_code)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(x, lg, wgu, wd, stream)
        layer.backward(gout, x, wgu, wd, True, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if layer.status(stream) != 0:
        raise SystemExit(f"device status {layer.status(stream)} after warm-up")

    def barrier():
        if pg is not None:
            pg.barrier()

    # ---- device-resident timed region: the layer alone, no per-kernel events ----
    clocks = ClockSampler(local)
    if not args.no_clocks:
        clocks.start()
    ms_per_step = timed_loop(step, args.steps, stream, dev, barrier, None if args.no_clocks else clocks)
    clk = clocks.stop()
    if layer.status(stream) != 0:
        raise SystemExit("device status error in the timed region")
    ms_per_step = max_over_ranks(ms_per_step, pg, dev)
    flops_step = IN.flops_fwd(**cfg) + IN.flops_bwd(**cfg)
    value = job_tflops(flops_step, world, ms_per_step)

    # ---- per-kernel breakdown: a second loop of the same steps, every launch
    # bracketed by CUDA events on its stream ----
    per_kernel, prof_ms = profiled_loop(M, step, args.steps, stream, dev, barrier)
    if layer.status(stream) != 0:
        raise SystemExit("device status error in the profiled loop")

    # ---- the same step captured once in a CUDA graph and replayed ----
    g_ms, g_err = graph_loop(lambda s: (layer.forward(x, lg, wgu, wd, s), layer.backward(gout, x, wgu, wd, True, s)),
                             args.steps, dev, barrier)
    if layer.status(stream) != 0:
        raise SystemExit("device status error in the graph replays")
    g_fail = max_over_ranks(0.0 if g_ms is not None else 1.0, pg, dev)  # every rank takes both collectives
    g_ms = max_over_ranks(g_ms if g_ms is not None else 0.0, pg, dev)
    if g_fail == 0.0:
        graph = {"ms_per_step": g_ms, "value": job_tflops(flops_step, world, g_ms), "unit": UNIT,
                 "note": "forward + backward captured once in a CUDA graph (routing's cooperative launch, "
                         "the persistent GEMMs, the second stream of the dx sum) and replayed; same work"}
    else:
        graph = {"unavailable": g_err or "the capture failed on another rank"}

    # ---- roofline of the dominant kernel ----
    peaks, peak_src = load_peaks()
    gemm_flops = gemm_flops_per_launch(T, d, k, I)
    dom = max(gemm_flops, key=lambda n: per_kernel.get(n, (0.0, 0))[0])
    dom_ms, dom_n = per_kernel[dom]
    dom_avg_ms = dom_ms / max(dom_n, 1)
    achieved = gemm_flops[dom] / (dom_avg_ms * 1e-3) / 1e12
    peak, peak_note, peak_alt = tensor_peaks(peaks, peak_src, mx, clk)
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if os.path.exists(tpath):
        try:
            from grouped_gemm_route_b200 import build as B
            with open(tpath) as f:
                tr = json.load(f)
            ent = tr.get(dom, {})
            if ent.get("source_hash") == B.source_hash(B.GEMM_SOURCES) and ent.get("workload") == args.workload:
                traffic = ent.get("dram_bytes_per_launch")
        except Exception:
            traffic = None
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_note,
                "frac_other_peak": {k_: achieved / v for k_, v in peak_alt.items()},
                "timing": "mean launch time from the per-kernel CUDA events of the profiled loop"}
    gemm_ms = sum(per_kernel.get(n, (0.0, 0))[0] for n in gemm_flops) / args.steps
    route_names = ("route_topk", "route_scan", "route_perm", "route_fused")
    route_ms = sum(per_kernel.get(n, (0.0, 0))[0] for n in route_names) / args.steps
    routing = {"bytes_per_step": IN.routing_bytes(T, E, k), "ms_per_step": route_ms,
               "achieved_gbs": IN.routing_bytes(T, E, k) / (route_ms * 1e-3) / 1e9 if route_ms else None,
               "peak_gbs": float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))}
    if not args.no_routing_sweep:
        routing["sweep"] = routing_sweep(M, IN, dev, stream, routing["peak_gbs"], E, k)
        routing["sweep_note"] = ("moe_route alone, E and top_k of this workload, one call per timing with L2 "
                                 "flushed before it; median of 10")
    breakdown = kernel_breakdown(per_kernel, args.steps)
    launches_per_step = sum(v[1] for v in per_kernel.values()) / args.steps
    launches = int(round(launches_per_step * args.steps))

    # ---- recompute mode: forward, h and aw regenerated, backward ----
    # (the layer cost under activation checkpointing: the gate/up GEMM runs
    # twice; same results as the plain step, tested bit for bit)
    recompute = None
    if not args.no_recompute:
        def step_recompute():
            layer.forward(x, lg, wgu, wd, stream)
            M.recompute(layer.shape, x, wgu, layer.saved, layer.ws, stream)
            layer.backward(gout, x, wgu, wd, True, stream)

        for _ in range(3):
            step_recompute()
        n_rc = max(3, args.steps // 4)
        barrier()
        torch.cuda.synchronize(dev)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(n_rc):
            step_recompute()
        r1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        rc_ms = max_over_ranks(r0.elapsed_time(r1), pg, dev) / n_rc
        if layer.status(stream) != 0:
            raise SystemExit("device status error in the recompute-mode loop")
        recompute = {"ms_per_step": rc_ms, "value": job_tflops(flops_step, world, rc_ms), "unit": UNIT,
                     "steps": n_rc, "note": "forward + moe_recompute (gate/up GEMM again) + backward; value counts "
                                            "the layer's fwd+bwd FLOPs only"}

    # ---- end-to-end through the public API with host buffers ----
    # Every step copies its inputs (x, logits, grad_out) from pinned host memory,
    # runs forward + backward, and copies its results (out, dx, dscore) back.
    # Two layer instances alternate so that the copies of one step overlap the
    # compute of the next (H2D and D2H on their own streams).
    e2e = None
    if not args.no_e2e:
        nb = 2
        layers = [layer] + [M.MoELayer(T, d, E, k, I, device=str(dev), dtype=dtype_code) for _ in range(nb - 1)]
        hx, hlg, hg = (host[n].pin_memory() for n in ("x", "logits", "gout"))
        hout = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
        hdx = [torch.empty(T, d, dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
        hds = [torch.empty(T, k, dtype=torch.float32).pin_memory() for _ in range(nb)]
        dins = [(torch.empty_like(x), torch.empty_like(lg), torch.empty_like(gout)) for _ in range(nb)]
        h2d = torch.cuda.Stream(dev)
        d2h = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event() for _ in range(nb)]
        computed = [torch.cuda.Event() for _ in range(nb)]
        drained = [torch.cuda.Event() for _ in range(nb)]

        def e2e_run(n_steps):
            for i in range(n_steps):
                b = i % nb
                with torch.cuda.stream(h2d):
                    h2d.wait_event(computed[b])  # step i - nb finished reading these inputs
                    for dst, src in zip(dins[b], (hx, hlg, hg)):
                        dst.copy_(src, non_blocking=True)
                    copied[b].record(h2d)
                stream.wait_event(copied[b])
                stream.wait_event(drained[b])  # step i - nb's results have left the device
                ly = layers[b]
                ly.forward(dins[b][0], dins[b][1], wgu, wd, stream)
                ly.backward(dins[b][2], dins[b][0], wgu, wd, True, stream)
                computed[b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(computed[b])
                    hout[b].copy_(ly.out, non_blocking=True)
                    hdx[b].copy_(ly.dx, non_blocking=True)
                    hds[b].copy_(ly.dscore, non_blocking=True)
                    drained[b].record(d2h)

        e2e_run(3)
        torch.cuda.synchronize(dev)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(h2d)
        stream.wait_event(e0)
        d2h.wait_event(e0)
        e2e_run(args.e2e_steps)
        stream.wait_stream(d2h)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
        bi = sum(t.numel() * t.element_size() for t in (hx, hlg, hg))
        bo = sum(t.numel() * t.element_size() for t in (hout[0], hdx[0], hds[0]))
        e2e = {"value": job_tflops(flops_step, world, e_ms / args.e2e_steps), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "steps": args.e2e_steps,
               "overlap": "copies of step i+1 / i-1 overlap compute of step i (two layer buffers); the first "
                          "step's inputs and the last step's results cross the bus with nothing to overlap",
               "note": "the step's result read back is out, dx and dscore; dW_gate_up and dW_down stay on the "
                       "device, as in a training loop whose optimizer runs on the GPU"}
        del layers

    # ---- CPU baseline (rank 0, N = 1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu, _, _ = cpu_baseline(cfg, host, args.cpu_tokens)

    # ---- the other workloads (N = 1 only): same warm-up and steps, events off,
    # breakdown from a profiled loop; the headline layer's buffers are freed first ----
    others = None
    if world == 1 and not args.no_configs:
        del layer, x, lg, wgu, wd, gout
        torch.cuda.empty_cache()
        others = {}
        for name in OTHER_WORKLOADS:
            if name == args.workload:
                continue
            others[name] = time_other_config(M, IN, name, args.steps, args.warmup, dev, stream, barrier, peaks,
                                             peak_src, args.seed, None if args.no_clocks else local)

    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "mxfp8 (e4m3, ue8m0/32)" if mx else "bf16", "data": "synthetic",
        "config": workload_config(args.workload, cfg, {"parallelism": f"replicas{world}", "l2": l2_note(cfg)}),
        "frac_of_peak": {"step": value / world / peak, "gemm_only": (flops_step / (gemm_ms * 1e-3) / 1e12) / peak
                              if gemm_ms else None, "peak": peak, "peak_source": roofline["peak_source"]},
        "roofline": roofline, "routing": routing, "kernels": breakdown, "gpu_launches": launches,
        "clocks": clk, "e2e": e2e, "graph": graph, "recompute": recompute, "cpu_baseline": cpu,
        "timing": "value and ms_per_step from a loop without per-kernel events; kernels and roofline from a "
                  f"second loop of the same steps with them ({prof_ms:.4f} ms per step there)",
        "configs": others,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
