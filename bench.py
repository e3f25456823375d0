#!/usr/bin/env python
"""Benchmark of the MoE routing hot path: gate -> route map -> expand -> reduce.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tk|reference] [--workload NAME]

One step = the four C-ABI calls (tk_gate_topk, tk_route_map, tk_expand, tk_reduce) over one
synthetic batch, inputs resident in HBM. The headline runs K such steps with two batches in
flight (the next batch's gate + route map on a second stream while this batch's expand + reduce
run); the JSON line also carries the serial time of the same K steps. Prints ONE JSON line (rank 0). For N > 1 run it under
torchrun: every rank routes its own batch (weak scaling, no data-path collective), time is the
max over ranks.

--impl reference times the CPU oracle (single-threaded C++) on bounded samples of the same
workload instead; under torchrun only rank 0 works.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed tokens/s + expand/reduce HBM GB/s vs peak @T=8192,E=256,k=8,H=7168"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["tk", "reference"], default="tk")
    p.add_argument("--workload", default="T8192_E256_k8_H7168_sigmoid_bias")
    p.add_argument("--tokens", type=int, default=None,
                   help="override T of the workload (smaller cases for profiling)")
    p.add_argument("--e2e-steps", type=int, default=None, help="end-to-end steps (default min(K, 20))")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time for cpu_baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--op", choices=["step", "backward", "stats", "ep", "boundary"], default="step",
                   help="step: the forward path (the benchmark's headline); backward: reduce and "
                        "expand backward; stats: load-balance statistics and the TP mask; ep: "
                        "expert-parallel dispatch/combine of the batch over --ep-ranks ranks run "
                        "on one GPU; boundary: reduce and expand each timed right after different "
                        "predecessors (itself, the other, a write that leaves L2 dirty, a read)")
    p.add_argument("--ep-ranks", type=int, default=8, help="ranks of the --op ep run")
    p.add_argument("--ep-tokens", type=int, default=None,
                   help="tokens per rank of the --op ep run (default: the workload's T, i.e. every "
                        "rank holds one 8K-token batch, the pages' EP setting)")
    p.add_argument("--ep-dtype", choices=["bf16", "fp8"], default="fp8",
                   help="dispatch format of the --op ep run (the pages' setting: FP8 dispatch)")
    return p.parse_args()


# ------------------------------------------------------------------ byte accounting
def algorithmic_bytes(wl, R=None):
    """Bytes each call must move at minimum (read + write), per launch over the whole batch."""
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    R = T * k if R is None else R
    pad_rows = R - T * k
    gate = T * E * 4 + (E * 4 if wl.bias else 0) + T * k * 8
    tiles = (T + 255) // 256
    route = T * k * 4 * 3 + tiles * E * 4 * 3 + wl.max_rows * 4 + T * k * 4 * 2 + (2 * E + 1) * 4
    if wl.out_dtype == "fp8":
        expand = T * H * 2 + T * k * 4 + T * k * H + T * k * (H // 128) * 4
        expand += pad_rows * (H + (H // 128) * 4)
    else:
        expand = T * H * 2 + T * k * 4 + T * k * H * 2 + pad_rows * H * 2
    if wl.align > 1:
        expand += R * 4
    reduce = T * k * H * 2 + T * k * 8 + T * H * 2
    return {"gate": gate, "route_map": route, "expand": expand, "reduce": reduce}


def per_token_bytes_text(wl):
    H, k = wl.H, wl.k
    if wl.out_dtype == "fp8":
        ex = f"2H + kH + 4k*H/128 + 4k = {2 * H + k * H + 4 * k * (H // 128) + 4 * k}"
    else:
        ex = f"2H(1+k) + 4k = {2 * H * (1 + k) + 4 * k}"
    return {"expand": ex, "reduce": f"2H(k+1) + 8k = {2 * H * (k + 1) + 8 * k}"}


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(kernel_file):
    """First 16 hex digits of the sha256 of a kernel's .cu file followed by the shared device
    header it includes (tk_device.cuh): a change to either makes stored counters stale."""
    csrc = os.path.join(ROOT, "token_routing_gate_b200", "csrc")
    h = hashlib.sha256()
    for name in (kernel_file, "tk_device.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_file, kernel_name, wl_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    source of the kernel; otherwise None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[wl_name][kernel_name]
        if e.get("source_sha") != source_sha(kernel_file):
            return None
        return float(e["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
             0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index, period_s=0.0005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001  (no NVML: report no clocks)
            self.nv = None

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self.nv is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in sorted(self.NAMES.items()) if self.reasons & b],
                "samples": len(self.samples)}


# ------------------------------------------------------------------ oracle (CPU) timing
def cpu_threads():
    return 1  # the oracle is single-threaded C++


def system_info(dev=None):
    """Host core count and CPU model, and the GPU's name when a device is given. Never raises:
    what cannot be read is None."""
    info = {"nproc": os.cpu_count(), "cpu_model": None, "gpu_name": None}
    try:
        with open("/proc/cpuinfo") as f:
            for row in f:
                if row.startswith("model name"):
                    info["cpu_model"] = row.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    if dev is not None:
        try:
            import torch
            info["gpu_name"] = torch.cuda.get_device_name(dev)
        except Exception:  # noqa: BLE001  (a name is context, never a reason to fail the run)
            pass
    return info


def oracle_buffers(wl):
    """Every output of the oracle's path for one batch of wl, allocated once (outside timing)."""
    import numpy as np
    import oracle
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    rmax = oracle.max_rows(T, E, k, wl.align)
    if wl.out_dtype == "fp8":
        xe = (np.zeros((rmax, H), np.uint8), np.zeros((rmax, H // 128), np.float32))
    else:
        xe = (np.zeros((rmax, H), np.uint16),)
    return {"gate": (np.empty((T, k), np.int32), np.empty((T, k), np.float32)),
            "route": (np.empty(E, np.int32), np.empty(E + 1, np.int32), np.empty((T, k), np.int32),
                      np.empty(rmax, np.int32)),
            "expand": xe, "reduce": np.empty((T, H), np.uint16)}


def oracle_step(wl, lg, b, x_bits, y_bits, bufs):
    """The whole path on the CPU oracle for one sample batch, into preallocated outputs."""
    import oracle
    fn = oracle.SOFTMAX if wl.score == "softmax" else oracle.SIGMOID
    idx, w = oracle.gate_topk(lg, b, wl.k, fn, out=bufs["gate"])
    counts, offsets, slot_of, token_of, _ = oracle.route_map(idx, wl.E, wl.align, out=bufs["route"])
    out_dtype = oracle.OUT_FP8_E4M3 if wl.out_dtype == "fp8" else oracle.OUT_BF16
    oracle.expand(x_bits, slot_of, offsets, wl.E, wl.align, out_dtype, out=bufs["expand"])
    return oracle.reduce(y_bits, slot_of, w, out=bufs["reduce"])


def oracle_sample_inputs(wl, Ts, seed):
    import numpy as np
    import torch
    from token_routing_gate_b200 import workloads as W
    sw = wl.with_(T=Ts, seed=seed)
    lg, b = W.gate_inputs(sw, "cpu")
    x = W.activations(sw, "cpu").view(torch.int16).numpy().view(np.uint16)
    y = W.expert_outputs(sw, "cpu").view(torch.int16).numpy().view(np.uint16)
    return sw, lg.numpy(), (b.numpy() if b is not None else None), x, y


def time_oracle(wl, seconds):
    """The oracle on the workload's whole batch (T tokens), outputs preallocated, repeated for
    about `seconds` (at least 3 runs)."""
    from oracle.build import build_oracle
    build_oracle()
    Ts = wl.T
    sw, lg, b, x, y = oracle_sample_inputs(wl, Ts, wl.seed)
    bufs = oracle_buffers(sw)
    oracle_step(sw, lg, b, x, y, bufs)  # warm (page in)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_step(sw, lg, b, x, y, bufs)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds and n >= 3:
            break
    return {"value": n * Ts / el, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n} runs of the full path on the whole {Ts}-token batch of {wl.name} "
                      f"(E={wl.E}, k={wl.k}, H={wl.H}) in {el:.1f} s, outputs preallocated, "
                      f"single-threaded C++ oracle"}


def run_reference(args, wl):
    from token_routing_gate_b200 import dist
    rank, world, _ = dist.rank_env()
    if rank != 0:
        return 0
    # size each step so the whole run stays within ~2 minutes of CPU time
    from oracle.build import build_oracle
    build_oracle()
    sw, lg, b, x, y = oracle_sample_inputs(wl, 128, wl.seed)
    bufs = oracle_buffers(sw)
    oracle_step(sw, lg, b, x, y, bufs)
    t0 = time.perf_counter()
    oracle_step(sw, lg, b, x, y, bufs)
    per_token = (time.perf_counter() - t0) / 128
    budget = 120.0 / max(1, args.steps + args.warmup)
    Ts = 64
    while Ts * 2 <= min(wl.T, 8192) and Ts * 2 * per_token <= budget:
        Ts *= 2
    sw, lg, b, x, y = oracle_sample_inputs(wl, Ts, wl.seed)
    bufs = oracle_buffers(sw)
    for _ in range(args.warmup):
        oracle_step(sw, lg, b, x, y, bufs)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(sw, lg, b, x, y, bufs)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = Ts * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "E": wl.E, "k": wl.k, "H": wl.H,
                   "score": wl.score, "bias": wl.bias, "align": wl.align, "out_dtype": wl.out_dtype,
                   "sample_tokens_per_step": Ts},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps, each the full path on {Ts} tokens of "
                                   f"{wl.name} (outputs preallocated), single-threaded C++ oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
        "system": system_info(),
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ the CUDA path
def run_tk(args, wl):
    import torch
    from token_routing_gate_b200 import dist, tk
    from token_routing_gate_b200 import workloads as W

    rank, world, local_rank = dist.rank_env()
    # Test hooks for the multi-rank path on a machine with fewer GPUs than ranks (the kernels of
    # one rank never wait on another, so ranks may share a GPU): TK_BENCH_DIST_BACKEND=gloo and
    # TK_BENCH_SAME_DEVICE=1. The numbers of such a run are not a measurement.
    if os.environ.get("TK_BENCH_SAME_DEVICE") == "1":
        local_rank = 0
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    backend = os.environ.get("TK_BENCH_DIST_BACKEND", "nccl")
    dist.init(backend if world > 1 else "gloo")
    if world > 1 and backend != "nccl":
        dev_for_collectives = None
    else:
        dev_for_collectives = dev
    stream = torch.cuda.current_stream(dev)

    swl = wl.with_(seed=dist.shard_seed(wl.seed, rank), param_seed=wl.seed)
    logits, bias = W.gate_inputs(swl, dev)
    x = W.activations(swl, dev)
    R_max = tk.max_rows(wl.T, wl.E, wl.k, wl.align)
    y = W.expert_outputs(swl, dev, rows=R_max)
    # outputs, preallocated once
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device=dev)
    w = torch.empty(wl.T, wl.k, dtype=torch.float32, device=dev)
    rm = tk.route_map(idx.zero_(), wl.E, wl.align)  # allocates the route-map buffers
    if wl.out_dtype == "fp8":
        xe = torch.empty(R_max, wl.H, dtype=torch.uint8, device=dev)
        xs = torch.empty(R_max, wl.H // 128, dtype=torch.float32, device=dev)
    else:
        xe = torch.empty(R_max, wl.H, dtype=torch.bfloat16, device=dev)
        xs = None
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tk.gate_topk(logits, wl.k, wl.score, bias, True, idx, w, stream)
        if ev is not None:
            ev[1].record(stream)
        tk.route_map(idx, wl.E, wl.align, out=rm, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        tk.expand(x, rm, wl.E, wl.k, wl.out_dtype, out=xe, out_scale=xs, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        tk.reduce(y, rm.slot_of, w, out=out, stream=stream)
        if ev is not None:
            ev[4].record(stream)

    # route map: count + fused scan/scatter while its count matrix (E rows of 128-token tiles,
    # padded to a multiple of 4) has at most 32K entries, else count, scan and scatter
    tiles = (wl.T + 127) // 128
    route_launches = 2 if (tiles + 3) // 4 * 4 * wl.E <= 32768 else 3
    launches_per_step = 1 + route_launches + 1 + (1 if wl.align > 1 else 0) + 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    R = int(rm.offsets[-1].item())

    K = args.steps
    from token_routing_gate_b200.pipeline import RoutingPipeline

    pipe = RoutingPipeline(wl.T, wl.E, wl.k, wl.score, wl.align, device=dev)

    def pipelined(n, step_ends=None):
        """n batches, two in flight: batch i+1's gate + route map on the pipeline's stream while
        batch i's expand + reduce run on `stream`. step_ends[i], when given, is recorded on
        `stream` right after batch i's reduce (next to the pipeline's own event there)."""
        pipe.stream.wait_stream(stream)
        h = pipe.route(logits, bias)
        for i in range(n):
            nxt = pipe.route(logits, bias) if i + 1 < n else None
            pipe.dispatch_combine(h, x, y, out, xe, wl.out_dtype, xs, stream=stream)
            if step_ends is not None:
                step_ends[i].record(stream)
            h = nxt

    for _ in range(args.warmup):
        pipelined(2)
    torch.cuda.synchronize(dev)

    def timed(run):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier(dev_for_collectives)
        torch.cuda.synchronize(dev)
        start.record(stream)
        run()
        end.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier(dev_for_collectives)
        return dist.max_over_ranks(start.elapsed_time(end) / 1e3, dev_for_collectives)

    clocks = ClockSampler(dev.index)   # sampled every 0.5 ms over all the passes below
    clocks.__enter__()
    # Pass 1 (the headline): K batches with two in flight (RoutingPipeline), nothing between the
    # calls, so each kernel's launch also overlaps the end of the previous one.
    max_s = timed(lambda: pipelined(K))
    # Pass 1b: the same K steps one after another on one stream (no batch overlap); this is the
    # routed tokens/s of all four calls timed as one stream sequence.
    serial_s = timed(lambda: [step() for _ in range(K)])
    # Pass 1c: the headline's K steps again with an event after every batch's reduce: the
    # distribution of single step times (median, best, p90) behind the headline's mean.
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    dist.barrier(dev_for_collectives)
    torch.cuda.synchronize(dev)
    ends[0].record(stream)
    pipelined(K, ends[1:])
    torch.cuda.synchronize(dev)
    dist.barrier(dev_for_collectives)
    step_ms = sorted(ends[i].elapsed_time(ends[i + 1]) for i in range(K))
    # Pass 2 (the per-kernel breakdown behind the roofline): the same K steps with events
    # between the calls; the events stop one call's launch from overlapping the previous one.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    dist.barrier(dev_for_collectives)
    torch.cuda.synchronize(dev)
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize(dev)
    dist.barrier(dev_for_collectives)
    clocks.__exit__(None, None, None)
    names = ["gate", "route_map", "expand", "reduce"]
    k_ms = {n: sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K)) / K for j, n in enumerate(names)}
    evented_ms = sum(evs[i][0].elapsed_time(evs[i][4]) for i in range(K)) / K

    peak, peak_kind = load_peak()
    ab = algorithmic_bytes(wl, R)
    kernels = {n: {"us": 1e3 * k_ms[n], "bytes": ab[n], "gbs": ab[n] / (k_ms[n] / 1e3) / 1e9}
               for n in names}
    dom = max(("expand", "reduce"), key=lambda n: k_ms[n])
    dom_file = {"expand": "expand.cu", "reduce": "reduce.cu"}[dom]
    dom_kernel = {"expand": "expand_fp8_kernel" if wl.out_dtype == "fp8" else "expand_bf16_kernel",
                  "reduce": "reduce_kernel"}[dom]
    achieved = kernels[dom]["gbs"]
    er_gbs = (ab["expand"] + ab["reduce"]) / ((k_ms["expand"] + k_ms["reduce"]) / 1e3) / 1e9
    value = dist.aggregate_rate(wl.T * K, world, max_s)
    serial_value = dist.aggregate_rate(wl.T * K, world, serial_s)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": 1e3 * max_s / K,
        "headline_form": "two batches in flight (gate + route map of the next batch overlap "
                         "expand + reduce of this one); 'serial' is the four calls of every step "
                         "timed as one stream sequence",
        "pairs_per_s": wl.k * value,
        "step_ms": {"mean": 1e3 * max_s / K, "median": statistics.median(step_ms),
                    "best": step_ms[0], "p90": step_ms[min(K - 1, int(0.9 * K))],
                    "note": "rank 0's single step times from a repeat of the headline pass with an "
                            "event after every batch's reduce; mean is the headline's"},
        "serial": {"value": serial_value, "pairs_per_s": wl.k * serial_value,
                   "ms_per_step": 1e3 * serial_s / K,
                   "note": "the same K steps one after another on one stream"},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "E": wl.E, "k": wl.k, "H": wl.H,
                   "score": wl.score, "bias": wl.bias, "align": wl.align,
                   "out_dtype": wl.out_dtype, "tokens_per_rank": wl.T, "rows_used": R,
                   "l2": "no flush: each step touches %.2f GB (> 126 MB L2)" % (sum(ab.values()) / 1e9),
                   "parallelism": f"dp{world} (independent token shards, no data-path collective)",
                   "pipelining": "two batches in flight: gate + route map of batch i+1 on a second "
                                 "stream overlap expand + reduce of batch i (RoutingPipeline); "
                                 "every batch runs all four calls"},
        "roofline": {"bound": "hbm", "kernel": dom_kernel, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": ncu_traffic(dom_file, dom_kernel, wl.name),
                     "algorithmic_bytes_per_launch": ab[dom],
                     "per_token_bytes": per_token_bytes_text(wl)[dom]},
        "expand_reduce": {"gbs": er_gbs, "frac": er_gbs / peak, "frac_of_8000": er_gbs / 8000.0},
        "kernels": kernels,
        "kernel_pass_ms_per_step": evented_ms,
        "clocks": clocks.summary(),
        "gpu_launches": launches_per_step * K,
        "system": system_info(dev),
    }

    if not args.no_e2e:
        line["e2e"] = run_e2e(args, wl, dev, stream, logits, bias, x, y, idx, w, rm, xe, xs, out,
                              world, dev_for_collectives)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_oracle(wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish()
    return 0


def run_e2e(args, wl, dev, stream, logits, bias, x, y, idx, w, rm, xe, xs, out, world, cdev):
    """Same step through the public calls, with every step's inputs copied in from pinned host
    memory and its result copied back, inside the timed region. Device inputs and outputs are
    double-buffered: step i+1's host-to-device copy and step i-1's device-to-host read run on
    their own streams while step i computes (PCIe carries both directions at once)."""
    import torch
    from token_routing_gate_b200 import dist, tk

    src = [t for t in (logits, bias, x, y) if t is not None]
    h_in = [t.cpu().pin_memory() for t in src]
    d_in = [[t, torch.empty_like(t)] for t in src]           # two device copies of each input
    d_out = [out, torch.empty_like(out)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out[0].numel() * h_out[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read_back = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(computed[b])                      # buffer b free (step i-2 done)
            for d, h in zip(d_in, h_in):
                d[b].copy_(h, non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        stream.wait_event(read_back[b])                       # out[b] read back (step i-2)
        lg, bi, xx, yy = (d_in[0][b], d_in[1][b] if bias is not None else None,
                          d_in[-2][b], d_in[-1][b])
        tk.gate_topk(lg, wl.k, wl.score, bi, True, idx, w, stream)
        tk.route_map(idx, wl.E, wl.align, out=rm, stream=stream)
        tk.expand(xx, rm, wl.E, wl.k, wl.out_dtype, out=xe, out_scale=xs, stream=stream)
        tk.reduce(yy, rm.slot_of, w, out=d_out[b], stream=stream)
        computed[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            h_out[b].copy_(d_out[b], non_blocking=True)
            read_back[b].record(s_out)

    n = args.e2e_steps if args.e2e_steps is not None else max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    dist.barrier(cdev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    s_in.wait_stream(stream)                                  # no copy starts before the clock
    for i in range(n):
        e2e_step(i)
    stream.wait_stream(s_out)
    e.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier(cdev)
    max_s = dist.max_over_ranks(s.elapsed_time(e) / 1e3, cdev)
    return {"value": dist.aggregate_rate(wl.T * n, world, max_s), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "ms_per_step": 1e3 * max_s / n,
            "pipelining": "double-buffered: H2D of step i+1 and D2H of step i-1 overlap step i"}


def run_op(args, wl):
    """Time one of the next-row ops on the workload (single GPU), one JSON line."""
    import torch
    from token_routing_gate_b200 import tk
    from token_routing_gate_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    logits, bias = W.gate_inputs(wl, dev)
    idx, w = tk.gate_topk(logits, wl.k, wl.score, bias)
    rm = tk.route_map(idx, wl.E, wl.align)
    T, E, k, H = wl.T, wl.E, wl.k, wl.H
    R = int(rm.offsets[-1].item())
    if args.op == "backward":
        y = W.expert_outputs(wl, dev)
        g = W.activations(wl.with_(seed=wl.seed + 7), dev)
        d_y = torch.empty_like(y)
        d_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        ws = tk._workspace(int(tk.lib.tk_reduce_backward_workspace_bytes(T, k)), dev)
        d_x = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        pad = (R - T * k) * H * 2 + (R * 4 if wl.align > 1 else 0)
        calls = {   # name: (call, algorithmic bytes, kernels it launches)
            "reduce_backward": (lambda: tk.reduce_backward(g, y, rm.slot_of, w, E, rm=rm, d_y=d_y, d_w=d_w,
                                                           workspace=ws, stream=stream),
                                T * H * 2 + 2 * T * k * H * 2 + T * k * (8 + 4 + 64) + pad, 2),
            "expand_backward": (lambda: tk.expand_backward(d_y, rm.slot_of, out=d_x, stream=stream),
                                T * k * H * 2 + T * k * 4 + T * H * 2, 1),
        }
        metric = "reduce + expand backward HBM GB/s vs peak"
    else:
        P = (torch.empty(E, device=dev), torch.empty(E, device=dev), torch.empty(1, device=dev))
        ws = tk._workspace(int(tk.lib.tk_balance_stats_workspace_bytes(T, E)), dev)
        masked = torch.empty_like(idx)
        rm_tp = tk.route_map(masked.zero_(), E // 8, 1)
        rm_win = tk.route_map_window(idx, E, 3 * (E // 8), E // 8, 1)
        calls = {
            "balance_stats": (lambda: tk.balance_stats(logits, rm.counts, k, wl.score, workspace=ws, out=P,
                                                       stream=stream),
                              T * E * 4 + E * 4 + ((T + 63) // 64) * E * 8 * 2 + 3 * E * 4, 2),
            "tp_mask": (lambda: tk.tp_mask(idx, E, 8, 3, out=masked, stream=stream), T * k * 8, 1),
            # one tensor-parallel rank's route map (8 ranks): the mask then the route map, and
            # the window route map doing both in one call
            "tp_mask_then_route_map": (lambda: (tk.tp_mask(idx, E, 8, 3, out=masked, stream=stream),
                                                tk.route_map(masked, E // 8, 1, out=rm_tp, stream=stream)),
                                       T * k * 8 + T * k * 12, 3),
            "route_map_window": (lambda: tk.route_map_window(idx, E, 3 * (E // 8), E // 8, 1, out=rm_win,
                                                             stream=stream), T * k * 12, 2),
        }
        metric = "load-balance statistics and TP mask us per call"
    peak, peak_kind = load_peak()
    # A call whose bytes fit twice in the 126 MB L2 would find its inputs there when launched back
    # to back, so such calls are timed one launch at a time after writing a 256 MB buffer; larger
    # ones run back to back (their own traffic evicts the previous launch's).
    flush_below = 256 << 20
    flush = torch.empty(flush_below, dtype=torch.uint8, device=dev)
    out, l2, launches = {}, {}, 0
    clocks = ClockSampler(0)
    with clocks:
        for name, (fn, nbytes, nk) in calls.items():
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize(dev)
            if nbytes < flush_below:
                pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                         for _ in range(args.steps)]
                for a, b in pairs:
                    flush.fill_(1)
                    a.record(stream)
                    fn()
                    b.record(stream)
                torch.cuda.synchronize(dev)
                us = 1e3 * sum(a.elapsed_time(b) for a, b in pairs) / args.steps
                l2[name] = "flushed (256 MB written) before each timed launch"
            else:
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                ev[0].record(stream)
                for _ in range(args.steps):
                    fn()
                ev[1].record(stream)
                torch.cuda.synchronize(dev)
                us = ev[0].elapsed_time(ev[1]) * 1e3 / args.steps
                l2[name] = "no flush: %.2f GB per launch (> 126 MB L2)" % (nbytes / 1e9)
            launches += nk * args.steps
            out[name] = {"us": us, "bytes": nbytes, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak}
    first = next(iter(out))
    line = {"metric": metric, "op": args.op, "value": out[first]["gbs"] if args.op == "backward" else out[first]["us"],
            "unit": "GB/s" if args.op == "backward" else "us", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": args.op == "backward", "dtype": "bf16",
            "data": "synthetic", "config": {"workload": wl.name, "T": T, "E": E, "k": k, "H": H,
                                             "align": wl.align, "rows_used": R, "l2": l2},
            "peak": peak, "peak_kind": peak_kind, "kernels": out, "clocks": clocks.summary(),
            "gpu_launches": launches, "system": system_info(dev)}
    if args.op == "backward":
        line["roofline"] = {"bound": "hbm", "kernel": "reduce_backward_kernel",
                            "achieved": out[first]["gbs"], "peak": peak, "peak_kind": peak_kind,
                            "unit": "GB/s", "frac": out[first]["frac"],
                            "traffic": ncu_traffic("backward.cu", "reduce_backward_kernel",
                                                   "backward_" + wl.name),
                            "algorithmic_bytes_per_launch": out[first]["bytes"]}
    print(json.dumps(line), flush=True)
    return 0


def run_ep(args, wl):
    """Expert-parallel dispatch -> experts' combine -> combine over G ranks that each hold
    --ep-tokens tokens of the workload's shape, all run on one GPU (VirtualRanks). The
    "transfers" are writes and reads of this GPU's own memory, so the numbers are HBM numbers of
    the EP kernels, not NVLink numbers."""
    import torch
    from token_routing_gate_b200 import ep, tk
    from token_routing_gate_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    G = args.ep_ranks
    Tr = args.ep_tokens or wl.T
    E, k, H = wl.E, wl.k, wl.H
    T = Tr * G
    if E % G:
        raise SystemExit(f"--ep-ranks {G} must divide E={E}")
    wl = wl.with_(T=T)
    logits, bias = W.gate_inputs(wl, dev)
    x = W.activations(wl, dev)
    idx, w = tk.gate_topk(logits, k, wl.score, bias)
    xs = [x[s * Tr:(s + 1) * Tr] for s in range(G)]
    idxs = [idx[s * Tr:(s + 1) * Tr].contiguous() for s in range(G)]
    ws = [w[s * Tr:(s + 1) * Tr].contiguous() for s in range(G)]
    vr = ep.VirtualRanks(G, E, k, H, Tr, args.ep_dtype, 1, dev)
    y = W.expert_outputs(wl, dev, rows=tk.max_rows(T, E // G, k, 1))   # shared by the ranks
    outs = [torch.empty(Tr, H, dtype=torch.bfloat16, device=dev) for _ in range(G)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def expert_fn(d, bufs, n, rm):
        return y

    names = ["layout", "dispatch", "experts", "combine"]

    def step(evs=None):
        if evs is None:
            return vr.step(xs, idxs, ws, expert_fn, outs, err, stream)
        evs["start"].record(stream)
        return vr.step(xs, idxs, ws, expert_fn, outs, err, stream, mark=lambda n: evs[n].record(stream))

    for _ in range(args.warmup):
        res = step()
    torch.cuda.synchronize(dev)
    if err.item() != 0:
        raise SystemExit(f"device error flag {err.item()}")
    recv = res["recv_rows"]
    K = args.steps
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in ["start"] + names} for _ in range(K)]
    with ClockSampler(dev.index) as clocks:
        for i in range(K):
            step(evs[i])
        torch.cuda.synchronize(dev)
    prev = ["start"] + names[:-1]
    phase_us = {n: 1e3 * sum(e[p].elapsed_time(e[n]) for e in evs) / K for p, n in zip(prev, names)}
    step_ms = sum(e["start"].elapsed_time(e["combine"]) for e in evs) / K
    # the dispatch and combine kernels on their own: rank 0's call launched back to back
    lay0 = res["layouts"][0]
    base0 = res["base"][0]
    peers0 = [vr.bufs[d].peer(int(base0[d])) for d in range(G)]
    # (one launch moves less than the 126 MB L2, so L2 is flushed before every timed launch by
    # writing a 256 MB buffer, and each launch is timed on its own)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    kernel_us = {}
    for name, fn in (("dispatch", lambda: tk.ep_dispatch(xs[0], idxs[0], ws[0], lay0, E, peers0,
                                                         args.ep_dtype, stream=stream)),
                     ("combine", lambda: tk.ep_combine([b.partial for b in vr.bufs], base0.tolist(),
                                                       recv.tolist(), lay0, H, out=outs[0],
                                                       stream=stream))):
        for _ in range(3):
            fn()
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(K)]
        torch.cuda.synchronize(dev)
        for a, b in pairs:
            flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        kernel_us[name] = 1e3 * sum(a.elapsed_time(b) for a, b in pairs) / K
    sent0 = int(lay0.send_counts.sum())
    sent_rows = int(recv.sum())
    row_out = H if args.ep_dtype == "fp8" else 2 * H
    scale_b = 4 * (H // 128) if args.ep_dtype == "fp8" else 0
    disp_bytes = T * 2 * H + sent_rows * (row_out + scale_b + 8 * k) + T * k * 8
    comb_bytes = sent_rows * 2 * H + T * 2 * H
    # destinations: every pair is a local choice on exactly one rank, so the experts' rows read
    # are T*k rows; each received row's choices and weights are read and its partial written
    # (the route maps' index traffic is small and not counted)
    dest_bytes = T * k * 2 * H + sent_rows * (k * 8 + 2 * H)
    peak, peak_kind = load_peak()
    line = {"metric": f"expert-parallel dispatch + combine tokens/s, {G} ranks on one GPU",
            "op": "ep", "value": T / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": K,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "dtype": args.ep_dtype, "data": "synthetic",
            "config": {"workload": f"ep{G}_T{Tr}_per_rank_E{E}_k{k}_H{H}_{wl.score}"
                                   + ("_bias" if wl.bias else ""), "T": T, "E": E, "k": k, "H": H, "ranks": G,
                       "tokens_per_rank": Tr, "rows_sent": sent_rows,
                       "emulated": "all ranks on one GPU: transfers are local HBM traffic"},
            "phases_us": phase_us,
            "kernel_us": kernel_us,
            "kernel_gbs": {"dispatch": (Tr * 2 * H + sent0 * (row_out + scale_b + 8 * k) + Tr * k * 8)
                           / (kernel_us["dispatch"] * 1e3),
                           "combine": (sent0 * 2 * H + Tr * 2 * H) / (kernel_us["combine"] * 1e3)},
            "hbm_gbs": {"dispatch": disp_bytes / (phase_us["dispatch"] * 1e3),
                        "experts": dest_bytes / (phase_us["experts"] * 1e3),
                        "combine": comb_bytes / (phase_us["combine"] * 1e3)},
            "experts_frac": {"value": dest_bytes / (phase_us["experts"] * 1e3) / peak, "peak": peak,
                             "peak_kind": peak_kind,
                             "note": "destination phase (route maps + tk_reduce_masked of every "
                                     "rank's received rows) against the HBM peak"},
            "bytes": {"dispatch": disp_bytes, "experts": dest_bytes, "combine": comb_bytes},
            "clocks": clocks.summary(), "gpu_launches": None, "system": system_info(dev)}
    print(json.dumps(line), flush=True)
    return 0


def run_boundary(args, wl):
    """tk_reduce and tk_expand of the workload, each launch timed on its own (events around it)
    right after a predecessor: the same call, the other call, a 256 MB or 64 MB write that leaves
    L2 full of dirty lines, a 256 MB read that leaves it clean. Median of K launches each. Shows
    what the step's order costs: the reduce follows expand, whose last writes are still dirty in
    L2 and are written back while the reduce reads."""
    import torch
    from token_routing_gate_b200 import tk
    from token_routing_gate_b200 import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = torch.cuda.current_stream(dev)
    logits, bias = W.gate_inputs(wl, dev)
    x = W.activations(wl, dev)
    R = tk.max_rows(wl.T, wl.E, wl.k, wl.align)
    y = W.expert_outputs(wl, dev, rows=R)
    idx, w = tk.gate_topk(logits, wl.k, wl.score, bias)
    rm = tk.route_map(idx, wl.E, wl.align)
    xe = torch.empty(R, wl.H, dtype=torch.bfloat16, device=dev)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    big = torch.empty(256 << 18, dtype=torch.float32, device=dev)   # 256 MB
    src = torch.ones_like(big)

    def reduce():
        tk.reduce(y, rm.slot_of, w, out=out, stream=s)

    def expand():
        tk.expand(x, rm, wl.E, wl.k, "bf16", out=xe, stream=s)

    preds = {"itself": None, "reduce": reduce, "expand": expand,
             "dirty_write_256MB": lambda: big.fill_(1.0),
             "dirty_write_64MB": lambda: big[: 64 << 18].fill_(1.0),
             "clean_read_256MB": lambda: torch.sum(src)}
    K = max(args.steps, 5)
    res = {}
    with ClockSampler(dev.index) as clocks:
        for name, op in (("reduce", reduce), ("expand", expand)):
            res[name] = {}
            for pname, prep in preds.items():
                prep = prep or op
                ts = []
                for i in range(K + args.warmup):
                    prep()
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(s)
                    op()
                    b.record(s)
                    torch.cuda.synchronize(dev)
                    if i >= args.warmup:
                        ts.append(a.elapsed_time(b) * 1e3)
                res[name][pname] = statistics.median(ts)
    ab = algorithmic_bytes(wl, int(rm.offsets[-1].item()))
    line = {"metric": "reduce / expand us after different predecessors", "op": "boundary",
            "value": res["reduce"]["expand"], "unit": "us", "n_gpus": 1, "steps": K,
            "warmup": args.warmup, "higher_is_better": False, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "E": wl.E, "k": wl.k, "H": wl.H},
            "median_us": res,
            "bytes": {"reduce": ab["reduce"], "expand": ab["expand"]},
            "clocks": clocks.summary(), "gpu_launches": None, "system": system_info(dev)}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    from token_routing_gate_b200 import workloads as W
    wl = W.BY_NAME[args.workload]
    if args.tokens is not None:
        wl = wl.with_(T=args.tokens, name=f"{wl.name}_T{args.tokens}")
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.op == "ep":
        return run_ep(args, wl)
    if args.op == "boundary":
        return run_boundary(args, wl)
    if args.op != "step":
        return run_op(args, wl)
    return run_tk(args, wl)


if __name__ == "__main__":
    sys.exit(main())
