#!/usr/bin/env python
"""Benchmark of the TTQ linear layer on B200: statistics + re-quantization + tensor-core
projection for each prompt (one "step" = one prompt through the layer), on the Qwen3-32B
query projection 5120 -> 8192 with 4-bit codes, group 128 (the runtime table of the
paper-daily.com deep reading of TTQ, section 4, measures this module).

Prints ONE JSON line (rank 0). ``value`` is whole-job prefill throughput in k tokens/s
with inputs resident in HBM; ``e2e`` is the same metric through the public Python API
with the prompt copied in from pinned host memory and Y copied back every step.
Per-stage times come from CUDA events the library records between its launches.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""

from __future__ import annotations

import argparse
import ctypes
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

from online_activation_aware_b200 import dist as D  # noqa: E402
from online_activation_aware_b200 import synthetic  # noqa: E402
from online_activation_aware_b200.lowrank_setup import lowrank_factors  # noqa: E402

METRIC = "TTQ linear k tokens/s (stats+requant+GEMM), 5120→8192 4-bit; requant GB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_32b_qproj")
    ap.add_argument("--T", type=int, default=None, help="prompt length (default: the workload's)")
    ap.add_argument("--r", type=int, default=None, help="low-rank r (default: the workload's)")
    ap.add_argument("--no-extras", action="store_true", help="skip the T sweep, decode and e2e legs")
    ap.add_argument("--no-decoder", action="store_true", help="skip the chained decoder-stack leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle baseline")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def requant_bytes(d, d_out, q, g):
    # read bf16 W and fp32 s; write packed codes and fp16 scale + zero
    return d_out * d * 2 + d * 4 + d_out * d * q // 8 + d_out * (d // g) * 4


def stats_bytes(T, d):
    return T * d * 2 + d * 4


def fold_bytes(T, d):
    return T * d * 4 + d * 4


def gemm_flops(T, d, d_out, r):
    return 2.0 * T * d * d_out + (2.0 * T * r * d_out if r else 0.0)


def input_sets(T, d, d_out):
    """Number of input buffer sets the timed steps rotate over, so that no step finds its
    operands in the 126 MB L2, and the bytes of one set."""
    import math

    set_bytes = (T * d + d_out * d) * 2
    return min(6, max(2, int(math.ceil(3 * 126e6 / set_bytes)) + 1)), set_bytes


def bench_config(wl, T, r, world):
    """The workload description both arms print (identical for the same arguments)."""
    lin = wl.layers[0]
    nsets, set_bytes = input_sets(T, lin.d, lin.d_out)
    return {"workload": f"{wl.name} {lin.d}->{lin.d_out} q={wl.q} g={wl.g} T={T}", "T": T, "d": lin.d,
            "d_out": lin.d_out, "q": wl.q, "g": wl.g, "alpha": wl.alpha, "lambda": wl.lam, "p": wl.p, "r": r,
            "parallelism": f"replicas{world}",
            "l2": f"{nsets} rotating input sets of {set_bytes / 1e6:.0f} MB (> 126 MB L2)"}


def whole_job_ktoks(T, steps, world, t_max_ms):
    """Whole-job throughput: every rank processed `steps` prompts of T tokens; the job
    took as long as its slowest rank."""
    return T * steps * world / (t_max_ms / 1e3) / 1e3


def decode_bytes(b, d, d_out, q, g):
    return d_out * d * q // 8 + d_out * (d // g) * 4 + b * d * 2 + b * d_out * 2 + d * 4


class ClockSampler:
    """Samples SM clock, power and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, mx, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "t0", -1e30), getattr(self, "t1", 1e30)
        for ts, ln in self.lines:
            if ts < t0 or ts > t1:
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockSampler:
    """Samples the SM clock, power and clock-event reasons every ~2 ms through NVML
    (read-only queries) on a background thread, so that even a timed region of a few
    milliseconds gets samples. Falls back to the nvidia-smi sampler when NVML is absent."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, gpu_id: str, period_s: float = 0.002):
        self.gpu_id = gpu_id
        self.period = period_s
        self.samples = []
        self._stop = threading.Event()
        self._fallback = None

    def start(self):
        try:
            import pynvml as N

            N.nvmlInit()
            self.N = N
            self.h = N.nvmlDeviceGetHandleByUUID(self.gpu_id)
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM))
            self.bits = [(name, getattr(N, attr, 0)) for name, attr in self.REASONS]
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self._fallback = ClockSampler(self.gpu_id)
            self._fallback.start()

    def _run(self):
        N, h = self.N, self.h
        while not self._stop.is_set():
            try:
                t = time.perf_counter()
                sm = float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM))
                rs = int(N.nvmlDeviceGetCurrentClocksEventReasons(h))
                pw = N.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((t, sm, rs, pw))
            except Exception:
                pass
            time.sleep(self.period)

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1
        if self._fallback is not None:
            self._fallback.window(t0, t1)

    def stop(self):
        if self._fallback is not None:
            out = self._fallback.stop()
            out["source"] = "nvidia-smi"
            return out
        self._stop.set()
        self._t.join(timeout=2)
        t0, t1 = getattr(self, "t0", -1e30), getattr(self, "t1", 1e30)
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        out = {"source": "nvml", "period_ms": self.period * 1e3, "samples": len(inside)}
        if not inside:
            # the region was shorter than one period: the nearest sample on each side
            before = [x for x in self.samples if x[0] < t0][-1:]
            after = [x for x in self.samples if x[0] > t1][:1]
            inside = before + after
            out["window"] = "no sample inside the timed region; the nearest one on each side"
        sm = [x[1] for x in inside]
        reasons = sorted({name for x in inside for name, bit in self.bits if bit and (x[2] & bit)})
        out.update({"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                    "power_w_max": max((x[3] for x in inside), default=None), "reasons": reasons})
        try:
            self.N.nvmlShutdown()
        except Exception:
            pass
        return out


def gpu_uuid(torch, dev):
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return str(dev)


def kernel_hash():
    h = hashlib.sha256()
    for name in ("gemm.cu", "gemm2sm.cu", "ttq_common.cuh"):
        with open(os.path.join(ROOT, "online_activation_aware_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload_key: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/ (null when the
    kernel source changed since the capture, or no capture exists)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    cur = kernel_hash()
    with open(path) as f:
        for line in f:
            parts = [p.strip() for p in line.strip().strip("|").split("|")]
            if len(parts) >= 4 and parts[0] == kernel and parts[1] == workload_key and parts[3] == cur:
                try:
                    return float(parts[2])
                except ValueError:
                    return None
    return None


# ------------------------------------------------------------------ CPU oracle legs


def oracle_sample(X, W, wl, T_tok: int, rows: int, seed: int = 0):
    """Times the oracle on a slice (T_tok tokens, `rows` output rows) and extrapolates
    the whole prompt (T tokens, all rows). Returns (seconds for the whole layer, info)."""
    import numpy as np

    from oracle import ttq_oracle as O

    T, d = X.shape
    d_out = W.shape[0]
    rng = np.random.default_rng(seed)
    t0 = rng.integers(0, max(1, T - T_tok + 1))
    r0 = rng.integers(0, max(1, d_out - rows + 1))
    Xs = X[t0:t0 + T_tok]
    Ws = W[r0:r0 + rows]
    a = time.perf_counter()
    s64, s32 = O.act_stats(Xs, wl.alpha, wl.lam, wl.p)
    b = time.perf_counter()
    codes, scale, zero = O.requant(Ws, s32, wl.q, wl.g)
    c = time.perf_counter()
    O.linear(Xs, s32, codes, scale, zero, wl.g)
    e = time.perf_counter()
    full = (b - a) * (T / T_tok) + (c - b) * (d_out / rows) + (e - c) * (T / T_tok) * (d_out / rows)
    return full, {"stats_s": b - a, "requant_s": c - b, "linear_s": e - c}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def host_inputs(wl, T, seed):
    lin = wl.layers[0]
    X, W = synthetic.draw_layer(T, lin.d, lin.d_out, seed)
    Xb, Wb = synthetic.as_bf16(X), synthetic.as_bf16(W)
    return Xb, Wb


def cpu_baseline(Xv, Wv, wl, budget_s):
    """The oracle, as it stands, on a bounded sample of the workload: 512 tokens x 256
    rows per sample, repeated on fresh slices until the budget is spent."""
    T = Xv.shape[0]
    T_tok = min(T, 512)
    rows = min(Wv.shape[0], 256)
    ests = []
    t_start = time.perf_counter()
    n = 0
    while time.perf_counter() - t_start < budget_s or n == 0:
        full, _ = oracle_sample(Xv, Wv, wl, T_tok, rows, seed=n)
        ests.append(full)
        n += 1
        if n >= 64:
            break
    full = statistics.median(ests)
    return {"value": round(T / full / 1e3, 6), "unit": "k tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} samples of {T_tok} tokens x {rows} output rows, each extrapolated to the full "
                      f"{T}-token prompt and {Wv.shape[0]} rows; median",
            "seconds": round(time.perf_counter() - t_start, 2)}


def run_reference(args, wl, T, r):
    rank, world, _ = D.env()
    if rank != 0:
        return 0
    import numpy as np

    Xb, Wb = host_inputs(wl, T, wl.seed)
    Xv, Wv = synthetic.bf16_values(Xb), synthetic.bf16_values(Wb)
    # size each step so the whole run stays within about two minutes
    nsteps = args.steps + args.warmup
    per_step = max(0.01, 120.0 / max(1, nsteps))
    T_tok, rows = 256, 64
    if per_step > 1.0:
        T_tok, rows = 512, 256
    times = []
    for i in range(nsteps):
        full, _ = oracle_sample(Xv, Wv, wl, T_tok, rows, seed=i)
        if i >= args.warmup:
            times.append(full)
    t = statistics.median(times)
    value = T / t / 1e3
    lin = wl.layers[0]
    cores = blas_threads()
    out = {"metric": METRIC, "value": round(value, 6), "unit": "k tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference", "extrapolated": True,
           "config": bench_config(wl, T, r, args.gpus),
           "cpu_baseline": {"value": round(value, 6), "unit": "k tokens/s", "cores": cores, "kind": "oracle",
                            "sample": f"each step: {T_tok} tokens x {rows} output rows, extrapolated to "
                                      f"{T} tokens x {lin.d_out} rows; median over {args.steps} steps"},
           "e2e": {"value": round(value, 6), "unit": "k tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ------------------------------------------------------------------ GPU legs


def main():
    args = parse()
    wl = synthetic.WORKLOADS[args.workload]
    T = args.T or wl.T
    r = wl.r if args.r is None else args.r
    if args.impl == "reference":
        return run_reference(args, wl, T, r)

    import numpy as np
    import torch

    import online_activation_aware_b200 as ttq

    rank, world, local_rank = D.env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    D.init("nccl")
    ttq.load_library()
    hbm_peak, tc_peak, tc_sust, peak_src = peaks()
    lin = wl.layers[0]
    d, d_out, q, g = lin.d, lin.d_out, wl.q, wl.g
    cfg = ttq.make_config(q, g, wl.alpha, wl.lam, wl.p, r)

    # inputs: this rank's own prompt and weight, copied into several buffer sets so that
    # consecutive steps never find their operands in the 126 MB L2
    Xb, Wb = host_inputs(wl, T, D.rank_seed(wl.seed, rank))
    A = B = None
    if r > 0:
        Bh, Ah, Rh = lowrank_factors(Wb, r)
        A, B = Ah.to(dev), Bh.to(dev)
        Wb = Rh
    nsets, set_bytes = input_sets(T, d, d_out)
    Xs = [Xb.to(dev) for _ in range(nsets)]
    Ws = [Wb.to(dev) for _ in range(nsets)]
    outs = [{"s": torch.empty(d, dtype=torch.float32, device=dev),
             "codes": torch.empty(ttq.codes_words(d_out, d, q), dtype=torch.int32, device=dev),
             "scale": torch.empty(d_out, d // g, dtype=torch.float16, device=dev),
             "zero": torch.empty(d_out, d // g, dtype=torch.float16, device=dev),
             "Y": torch.empty(T, d_out, dtype=torch.bfloat16, device=dev)} for _ in range(nsets)]
    ws = ttq.alloc_workspace(T, d, d_out, cfg, dev)
    stream = torch.cuda.current_stream()

    def step(i):
        k = i % nsets
        ttq.linear_prefill(Xs[k], Ws[k], cfg, A, B, out=outs[k], ws=ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert ttq.device_status() == 0

    # stage split: a separate run of the same steps with the library's stage events (each
    # stage then starts only when the one before it has finished), right after the warm-up
    # and before the timed region, with its own clock samples: the GEMM's roofline comes
    # from it
    Ks = max(3, min(args.steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(Ks)]
    tsampler = NvmlClockSampler(gpu_uuid(torch, dev))
    tsampler.start()
    time.sleep(0.02)
    tw0 = time.perf_counter()
    for i in range(Ks):
        ttq.set_trace_events(evs[i])
        step(i)
    torch.cuda.synchronize()
    tsampler.window(tw0, time.perf_counter())
    trace_clocks = tsampler.stop()
    ttq.set_trace_events(None)
    stage_names = ["stats", "lowrank_u", "fold_requant", "gemm", "reduce"]
    stage_ms = {n: statistics.median(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(Ks))
                for j, n in enumerate(stage_names)}

    # timed region: K prefill steps back to back (no stage events inside it: an event
    # between two kernels would stop the next one from starting early as a programmatic
    # dependent)
    K = args.steps
    sampler = NvmlClockSampler(gpu_uuid(torch, dev))
    sampler.start()
    time.sleep(0.05)
    D.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    start.record()
    for i in range(K):
        step(i)
    end.record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    sampler.window(wall0, wall0 + wall)
    D.barrier()
    clocks = sampler.stop()
    assert ttq.device_status() == 0
    t_ms = start.elapsed_time(end)
    t_max_ms = D.max_over_ranks(t_ms, dev)

    value = whole_job_ktoks(T, K, world, t_max_ms)

    plan_split = stage_ms["reduce"] > 0.002
    # kernels of ours per step: statistic, (low-rank X A^T partial products and their
    # reduction), fold + requant, tensor-core GEMM, (split-K reduce)
    launches_per_step = 3 + (2 if r > 0 else 0) + (1 if plan_split else 0)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB read flushes L2
    sink = torch.empty((), dtype=torch.float32, device=dev)

    # the statistic's kernel timed on its own (graph difference, L2 flushed): the traced
    # stage adds the gap that the event between two launches opens
    stats_sa = act_stats_leg(torch, ttq, Xs, outs, wl, hbm_peak, flush, sink)
    kern = {
        "stats": {"ms": stats_sa["us"] / 1e3, "bound": "hbm", "bytes": stats_bytes(T, d),
                  "method": "ttq_act_stats alone, graph difference, L2 flushed"},
        "fold_requant": {"ms": stage_ms["fold_requant"], "bound": "hbm",
                         "bytes": fold_bytes(T, d) + requant_bytes(d, d_out, q, g)},
        **({"lowrank_u": {"ms": stage_ms["lowrank_u"], "bound": "hbm", "bytes": T * d * 2 + r * d * 2 + T * 128}}
           if r > 0 else {}),
        "gemm": {"ms": stage_ms["gemm"] + stage_ms["reduce"], "bound": "tensor", "flops": gemm_flops(T, d, d_out, r)},
    }
    for k_, v in kern.items():
        sec = v["ms"] / 1e3
        if v["bound"] == "hbm":
            v["GBps"] = round(v["bytes"] / sec / 1e9, 1)
            v["frac"] = round(v["GBps"] / hbm_peak, 4)
        else:
            v["TFLOPs"] = round(v["flops"] / sec / 1e12, 1)
            v["frac"] = round(v["TFLOPs"] / tc_peak, 4)
        v["ms"] = round(v["ms"], 5)
    # the GEMM's stage time comes from the traced steps: against the sustained bf16 peak
    # when the SM clock fell under the power cap there, else the burst
    sm, smax = trace_clocks.get("sm_mhz"), trace_clocks.get("sm_max_mhz")
    long_run = bool(sm and smax and sm < 0.95 * smax)  # the clock fell (power cap) during the traced steps
    tc_ref = tc_sust if long_run else tc_peak
    kern["gemm"]["frac"] = round(kern["gemm"]["TFLOPs"] / tc_ref, 4)
    dom = max(kern, key=lambda k_: kern[k_]["ms"])
    dk = kern[dom]
    wkey = f"{wl.name}_T{T}_r{r}"
    if dk["bound"] == "tensor":
        roof = {"kernel": "ttq_gemm2sm_kernel" if T > 128 else "ttq_gemm_kernel", "bound": "tensor",
                "achieved": dk["TFLOPs"], "peak": tc_ref, "unit": "TFLOP/s", "frac": dk["frac"],
                "frac_of_burst": round(dk["TFLOPs"] / tc_peak, 4),
                "traffic": profiled_traffic("ttq_gemm2sm_kernel" if T > 128 else "ttq_gemm_kernel", wkey),
                "algorithmic": f"2*T*d*d_out flops per launch = {dk['flops']:.4g}",
                "peak_source": f"{peak_src} bf16 {'sustained (power-capped clock)' if long_run else 'burst'} "
                               "(MEASURED_PEAKS.json)"}
    else:
        roof = {"kernel": {"fold_requant": "requant_kernel", "stats": "stats_tma_kernel",
                           "lowrank_u": "lowrank_u_kernel"}[dom],
                "bound": "hbm", "achieved": dk["GBps"], "peak": hbm_peak, "unit": "GB/s", "frac": dk["frac"],
                "traffic": profiled_traffic(dom, wkey), "algorithmic": f"{dk['bytes']} bytes per launch",
                "peak_source": f"{peak_src} HBM copy (MEASURED_PEAKS.json)"}

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": "k tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t_max_ms / K, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(wl, T, r, world),
        "requant_gbs": requant_leg(torch, ttq, Ws, outs, d, d_out, q, g, flush, sink),
        "stage_trace_ms": {k_: round(v, 5) for k_, v in stage_ms.items()},
        "stage_trace_clocks": trace_clocks,
        "act_stats_standalone": stats_sa,
        "requant_batched": requant_batched_leg(torch, ttq, Ws, outs, d, d_out, q, g),
        "roofline": roof,
        "kernels": kern,
        "rho_measured": round((stage_ms["stats"] + stage_ms["fold_requant"]) / (stage_ms["gemm"] + stage_ms["reduce"]), 4),
        "gpu_launches": K * launches_per_step,
        "clocks": clocks,
        "wall_s_timed": round(wall, 3),
    }

    # ---- end to end through the public API: pinned host X in, Y back out, every step.
    # Three streams overlap step i's host->device copy, step i-1's prefill and step i-2's
    # device->host copy (two device buffers each for X and Y, events for the hand-offs),
    # as a serving loop would; every step still moves its own input and result over PCIe.
    if not args.no_extras:
        Xh = Xb.pin_memory()
        Yh = [torch.empty(T, d_out, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        layer_ = ttq.TTQLinear(Ws[0], q, g, wl.alpha, wl.lam, wl.p, r, A, B)
        Xd = [torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        Yd = [torch.empty(T, d_out, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        x_ready, x_free, y_ready, y_free = ([ev() for _ in range(2)] for _ in range(4))
        for k in range(2):  # every buffer starts free
            x_free[k].record(s_cmp)
            y_free[k].record(s_out)

        def e2e_step(i):
            k = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(x_free[k])
                Xd[k].copy_(Xh, non_blocking=True)
                x_ready[k].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(x_ready[k])
                s_cmp.wait_event(y_free[k])
                layer_.prefill(Xd[k], Y=Yd[k], stream=s_cmp)
                x_free[k].record(s_cmp)
                y_ready[k].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(y_ready[k])
                Yh[k].copy_(Yd[k], non_blocking=True)
                y_free[k].record(s_out)

        Ke = max(3, min(K, 50))
        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        D.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        e0.record(cur)
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(cur)
        for i in range(Ke):
            e2e_step(i)
        for st in (s_in, s_cmp, s_out):
            cur.wait_stream(st)
        e1.record(cur)
        torch.cuda.synchronize()
        te = D.max_over_ranks(e0.elapsed_time(e1), dev)
        result["e2e"] = {"value": round(T * Ke * world / (te / 1e3) / 1e3, 3), "unit": "k tokens/s",
                         "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d_out * 2,
                         "steps": Ke, "api": "TTQLinear.prefill",
                         "overlap": "copies of neighbouring steps overlap the prefill (three streams)"}
    else:
        result["e2e"] = None

    # ---- rank 0 extras: oracle baseline, decode steps, prompt-length sweep
    if world == 1 and not args.no_extras:
        Xv, Wv = synthetic.bf16_values(Xb), synthetic.bf16_values(Wb)
        result["cpu_baseline"] = cpu_baseline(Xv, Wv, wl, args.cpu_seconds)
        result["decode"] = decode_leg(torch, ttq, wl, cfg, Xs[0], Ws[0], A, B, dev, hbm_peak)
        result["decode_batched"] = decode_batched_leg(torch, ttq, wl, cfg, Ws[0], outs, dev, hbm_peak)
        result["sweep"] = sweep_leg(torch, ttq, wl, cfg, Wb, A, B, dev, r)
        if r == 0:
            result["rho_sweep"] = rho_sweep_leg(torch, ttq, wl, cfg, Wb, dev, hbm_peak)
        sets = {"single_512": workload_set_leg(torch, ttq, "single_512", dev, hbm_peak, tc_peak),
                "opt125m_set": workload_set_leg(torch, ttq, "opt125m_set", dev, hbm_peak, tc_peak)}
        for g_ in synthetic.WORKLOADS["qwen3_1p7b_set"].g_sweep:
            sets[f"qwen3_1p7b_set_g{g_}"] = workload_set_leg(torch, ttq, "qwen3_1p7b_set", dev, hbm_peak, tc_peak,
                                                             g=g_)
        result["workloads"] = sets
        if r == 0:
            result["lowrank_r16"] = lowrank_leg(torch, ttq, wl, Xs, Ws, dev)
            result["prefill_batched"] = prefill_batched_leg(torch, ttq, wl, cfg, Xs, Ws, dev)
        if not args.no_decoder:
            result["decoder_stack"] = decoder_leg(torch, ttq, dev)
    if rank == 0:
        print(json.dumps(result), flush=True)
    D.barrier()
    D.finalize()
    return 0


def graph_step_us(torch, step, flush, sink, n=32):
    """Device time of one `step` with L2 flushed before it, from two CUDA graphs replayed
    once each: n x (flush read, step) and n x (flush read); the difference over n is the
    step (no host launch latency inside either measurement)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    ga, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(ga, stream=s):
            for _ in range(n):
                torch.sum(flush, dim=0, out=sink)
                step(s)
        with torch.cuda.graph(gb, stream=s):
            for _ in range(n):
                torch.sum(flush, dim=0, out=sink)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()

    def run(g_):
        ts = []
        for _ in range(5):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            g_.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    ta, tb = run(ga), run(gb)
    del ga, gb
    return (ta - tb) * 1e3 / n


def requant_leg(torch, ttq, Ws, outs, d, d_out, q, g, flush, sink):
    """GB/s of the re-quantization alone (the ttq_requant entry point: read W and s, write
    codes, scale and zero) with L2 flushed before each launch, device time from the
    difference of two CUDA graphs (no host launch latency)."""
    n = len(Ws)
    ctr = [0]

    def one(st):
        i = ctr[0]
        ctr[0] += 1
        o = outs[i % n]
        ttq.requant(Ws[i % n], o["s"], q, g, codes=o["codes"], scale=o["scale"], zero=o["zero"], stream=st)

    for _ in range(3):
        one(torch.cuda.current_stream())
    torch.cuda.synchronize()
    us = graph_step_us(torch, one, flush, sink)
    return round(requant_bytes(d, d_out, q, g) / (us * 1e-6) / 1e9, 1)


def act_stats_leg(torch, ttq, Xs, outs, wl, hbm_peak, flush, sink):
    """The statistic alone (the ttq_act_stats entry point: read X, write s) with L2 flushed
    before each launch, device time from the difference of two CUDA graphs (launches with
    flushes, flushes alone), so host launch latency does not enter."""
    n = len(Xs)
    T, d = Xs[0].shape
    ctr = [0]

    def one(st):
        i = ctr[0]
        ctr[0] += 1
        ttq.act_stats(Xs[i % n], wl.alpha, wl.lam, wl.p, s=outs[i % n]["s"], stream=st)

    for _ in range(3):
        one(torch.cuda.current_stream())
    torch.cuda.synchronize()
    us = graph_step_us(torch, one, flush, sink)
    gbs = stats_bytes(T, d) / (us * 1e-6) / 1e9
    # the same kernel over prompts of 1/4, 1 and 4 times T tokens: a fixed cost per launch
    # plus a streaming rate (the least-squares line through time against bytes)
    pts = []
    for f in (0.25, 1.0, 4.0):
        Tf = int(T * f)
        Xf = Xs[0] if Tf == T else torch.randn(Tf, d, device=Xs[0].device).to(torch.bfloat16)
        sf = torch.empty(d, dtype=torch.float32, device=Xs[0].device)
        u = graph_step_us(torch, lambda st: ttq.act_stats(Xf, wl.alpha, wl.lam, wl.p, s=sf, stream=st), flush, sink)
        pts.append((stats_bytes(Tf, d), u))
        del Xf
    n = len(pts)
    mb = sum(b for b, _ in pts) / n
    mu = sum(u for _, u in pts) / n
    slope = sum((b - mb) * (u - mu) for b, u in pts) / sum((b - mb) ** 2 for b, _ in pts)  # us per byte
    return {"us": round(us, 2), "GBps": round(gbs, 1), "frac": round(gbs / hbm_peak, 4),
            "method": "graph difference, L2 flushed before each launch",
            "size_sweep_us": {f"{b / 1e6:.0f}MB": round(u, 2) for b, u in pts},
            "streaming_GBps": round(1e-3 / slope, 1), "fixed_us": round(mu - slope * mb, 2)}


def requant_batched_leg(torch, ttq, Ws, outs, d, d_out, q, g, P=4, reps=50):
    """One weight re-quantized for P prompts per launch (ttq_requant_batched: W read once,
    P sets of codes / scale / zero written), rotating weight sets; compared with P
    single-prompt launches (ttq_requant) over the same sets."""
    n = len(Ws)
    S = torch.stack([outs[i % n]["s"] for i in range(P)]).contiguous()
    dev = Ws[0].device
    res_ = [ttq.requant_batched(Ws[0], S, q, g) for _ in range(2)]

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps

    def batched(i):
        c, s_, z = res_[i % 2]
        ttq.requant_batched(Ws[i % n], S, q, g, codes=c, scale=s_, zero=z)

    def singles(i):
        c, s_, z = res_[i % 2]
        for p in range(P):
            ttq.requant(Ws[i % n], S[p], q, g, codes=c[p], scale=s_[p], zero=z[p])

    tb = timed(batched)
    ts = timed(singles)
    by = d_out * d * 2 + P * (d * 4 + d_out * d * q // 8 + d_out * (d // g) * 4)
    del res_, S
    return {"prompts": P, "us_per_launch": round(tb * 1e6, 2), "us_per_prompt": round(tb * 1e6 / P, 2),
            "GBps": round(by / tb / 1e9, 1), "single_prompt_launches_us": round(ts * 1e6, 2),
            "speedup_vs_single": round(ts / tb, 3)}


def decode_batched_leg(torch, ttq, wl, cfg, W, outs, dev, hbm_peak, P=8, b=1):
    """Decode steps of P requests with their own prefill parameters (statistic and codes
    from one weight re-quantized per request), b tokens each, in one call
    (ttq_linear_decode_batched), L2 flushed by a read of 256 MB before each step, timed
    as in decode_leg."""
    lin = wl.layers[0]
    d, d_out = lin.d, lin.d_out
    n = len(outs)
    S = torch.stack([outs[i % n]["s"] * (1.0 + 0.01 * i) for i in range(P)]).contiguous()
    codes, scale, zero = ttq.requant_batched(W, S, cfg.q, cfg.g)
    xt = synthetic.as_bf16(synthetic.draw_tokens(P * b, d, seed=77)).reshape(P, b, d).to(dev)
    Y = torch.empty(P, b, d_out, dtype=torch.bfloat16, device=dev)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    nws = ctypes.c_size_t(0)
    assert ttq.load_library().ttq_decode_batched_workspace_size(P, b, d, d_out, ctypes.byref(cfg),
                                                                ctypes.byref(nws)) == 0
    ws = torch.empty(max(int(nws.value), 256), dtype=torch.uint8, device=dev)
    for _ in range(3):
        ttq.linear_decode_batched(xt, S, codes, scale, zero, cfg, d_out, Y=Y, ws=ws)
    torch.cuda.synchronize()
    t = graph_step_us(torch, lambda st: ttq.linear_decode_batched(xt, S, codes, scale, zero, cfg, d_out, Y=Y, ws=ws,
                                                                  stream=st), flush, sink) / 1e6
    by = P * decode_bytes(b, d, d_out, cfg.q, cfg.g)
    assert ttq.device_status() == 0
    return {"requests": P, "tokens_per_request": b, "us_per_step": round(t * 1e6, 2),
            "k_tokens_per_s": round(P * b / t / 1e3, 2), "GBps": round(by / t / 1e9, 1),
            "frac_hbm": round(by / t / 1e9 / hbm_peak, 4)}


def decode_leg(torch, ttq, wl, cfg, X, W, A, B, dev, hbm_peak):
    """Decode steps reusing one prefill's codes, b tokens per step, with L2 flushed by a
    read of 256 MB before each step; timed as the difference of two CUDA graphs (steps
    with flushes, flushes alone)."""
    lin = wl.layers[0]
    d, d_out = lin.d, lin.d_out
    layer_ = ttq.TTQLinear(W, cfg.q, cfg.g, cfg.alpha, cfg.lambda_, cfg.p, cfg.r, A, B)
    layer_.prefill(X)
    # L2 flush by reading a 256 MB buffer: it evicts the codes without leaving dirty lines
    # whose write-back would be charged to the timed step
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    out = {}
    for b in wl.decode_batches or (1,):
        xt = synthetic.as_bf16(synthetic.draw_tokens(b, d, seed=1234 + b)).to(dev)
        Y = torch.empty(b, d_out, dtype=torch.bfloat16, device=dev)
        layer_.workspace(b)
        for _ in range(3):
            layer_.decode(xt, Y=Y)
        torch.cuda.synchronize()
        t = graph_step_us(torch, lambda st: layer_.decode(xt, Y=Y, stream=st), flush, sink) / 1e6
        by = decode_bytes(b, d, d_out, cfg.q, cfg.g)
        out[f"b{b}"] = {"us_per_step": round(t * 1e6, 2), "k_tokens_per_s": round(b / t / 1e3, 2),
                        "GBps": round(by / t / 1e9, 1), "frac_hbm": round(by / t / 1e9 / hbm_peak, 4)}
    assert ttq.device_status() == 0
    return out


def lowrank_leg(torch, ttq, wl, Xs, Ws, dev, r=16, K=30):
    """The same prefill with the low-rank side path (rank r): seeded random bf16 factors
    B [d_out, r], A [r, d] of the right shapes stand in for the SVD factors (the kernels'
    time does not depend on their values); rotating buffer sets as in the main run."""
    lin = wl.layers[0]
    d, d_out, T = lin.d, lin.d_out, Xs[0].shape[0]
    g_ = torch.Generator(device="cpu").manual_seed(16)
    A = (torch.randn(r, d, generator=g_) * 0.02).to(torch.bfloat16).to(dev)
    B = (torch.randn(d_out, r, generator=g_) * 0.02).to(torch.bfloat16).to(dev)
    cfg = ttq.make_config(wl.q, wl.g, wl.alpha, wl.lam, wl.p, r)
    ws = ttq.alloc_workspace(T, d, d_out, cfg, dev)
    n = len(Xs)
    outs = [ttq.linear_prefill(Xs[i], Ws[i], cfg, A, B, ws=ws) for i in range(n)]
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(K):
        ttq.linear_prefill(Xs[i % n], Ws[i % n], cfg, A, B, out=outs[i % n], ws=ws)
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / 1e3 / K
    assert ttq.device_status() == 0
    return {"r": r, "T": T, "k_tokens_per_s": round(T / t / 1e3, 2), "us_per_prompt": round(t * 1e6, 1),
            "factors": "seeded random bf16 of the SVD factors' shapes"}


def prefill_batched_leg(torch, ttq, wl, cfg, Xs, Ws, dev, P=4, Tp=1024, K=20):
    """P prompts of Tp tokens, each with its own statistic and codes, through one
    ttq_linear_prefill_batched call (one read of W re-quantized for all, one grouped
    projection) against P single-prompt prefills; rotating weight sets."""
    d = Xs[0].shape[1]
    d_out = Ws[0].shape[0]
    Xb = Xs[0][: P * Tp].contiguous()
    n = len(Ws)
    T = [Tp] * P
    nb = ctypes.c_size_t(0)
    Ta = (ctypes.c_int64 * P)(*T)
    assert ttq.load_library().ttq_prefill_batched_workspace_size(Ta, P, d, d_out, ctypes.byref(cfg),
                                                                 ctypes.byref(nb)) == 0
    wsb = torch.empty(int(nb.value), dtype=torch.uint8, device=dev)
    wss = ttq.alloc_workspace(Tp, d, d_out, cfg, dev)
    outs = [ttq.linear_prefill(Xb[:Tp], Ws[0], cfg, ws=wss) for _ in range(P)]

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(K):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / K

    tb = timed(lambda i: ttq.linear_prefill_batched(Xb, T, Ws[i % n], cfg, ws=wsb))
    ts = timed(lambda i: [ttq.linear_prefill(Xb[p * Tp:(p + 1) * Tp], Ws[i % n], cfg, out=outs[p], ws=wss)
                          for p in range(P)])
    assert ttq.device_status() == 0
    return {"prompts": P, "tokens_per_prompt": Tp, "k_tokens_per_s": round(P * Tp / tb / 1e3, 2),
            "us_per_call": round(tb * 1e6, 1), "single_prompt_calls_us": round(ts * 1e6, 1),
            "speedup_vs_single": round(ts / tb, 3)}


def sweep_leg(torch, ttq, wl, cfg, Wb, A, B, dev, r):
    """Prefill throughput across prompt lengths (k tokens/s), rotating buffer sets."""
    import numpy as np

    lin = wl.layers[0]
    d, d_out = lin.d, lin.d_out
    res = {}
    for T in (wl.T_sweep or ()):
        Xb = synthetic.as_bf16(synthetic.draw_layer(T, d, 8, seed=500 + T)[0])
        nsets = 3 if T <= 4096 else 2
        Xs = [Xb.to(dev) for _ in range(nsets)]
        Ws = [Wb.to(dev) for _ in range(nsets)]
        ws = ttq.alloc_workspace(T, d, d_out, cfg, dev)
        outs = [None] * nsets
        for i in range(3):
            outs[i % nsets] = ttq.linear_prefill(Xs[i % nsets], Ws[i % nsets], cfg, A, B, ws=ws)
        torch.cuda.synchronize()
        K = 30 if T <= 4096 else 8
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(K):
            k = i % nsets
            ttq.linear_prefill(Xs[k], Ws[k], cfg, A, B, out=outs[k], ws=ws)
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / K
        res[f"T{T}"] = {"k_tokens_per_s": round(T / t / 1e3, 2), "us_per_prompt": round(t * 1e6, 1)}
        del Xs, Ws, outs, ws
        torch.cuda.empty_cache()
    assert ttq.device_status() == 0
    return res

def rho_sweep_leg(torch, ttq, wl, cfg, Wb, dev, hbm_peak, Ts=(128, 1024, 2048, 4096, 8192, 16384), reps=20):
    """The overhead ratio across prompt lengths: per T, the stage split of the prefill from
    the library's stage events (median over `reps` prompts, rotating buffer sets larger
    than L2), rho = (statistic + fold and re-quantization) / projection, next to the
    pages' count rho_model = 1/d' + 3/T (gist.science French summary, section 2A:
    O(dT + 3d'd) extra against O(d'dT)). The count's structure, as times: the overhead is a
    constant (requant) plus a term linear in T (statistic, fold), the projection is
    proportional to T (checked from T = 2048, where it runs at its tensor-core rate)."""
    lin = wl.layers[0]
    d, d_out = lin.d, lin.d_out
    res = {}
    for T in Ts:
        Xb = synthetic.as_bf16(synthetic.draw_layer(T, d, 8, seed=600 + T)[0])
        nsets = 3 if T <= 4096 else 2
        Xs = [Xb.to(dev) for _ in range(nsets)]
        Ws = [Wb.to(dev) for _ in range(nsets)]
        ws = ttq.alloc_workspace(T, d, d_out, cfg, dev)
        outs = [ttq.linear_prefill(Xs[i], Ws[i], cfg, ws=ws) for i in range(nsets)]
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(reps)]
        for i in range(reps):
            ttq.set_trace_events(evs[i])
            k = i % nsets
            ttq.linear_prefill(Xs[k], Ws[k], cfg, out=outs[k], ws=ws)
        torch.cuda.synchronize()
        ttq.set_trace_events(None)
        med = lambda a, b: statistics.median(e[a].elapsed_time(e[b]) for e in evs) * 1e3  # noqa: E731
        t_stats, t_req, t_gemm = med(0, 1), med(2, 3), med(3, 5)
        rho = (t_stats + t_req) / t_gemm
        rho_model = 1.0 / d_out + 3.0 / T
        res[f"T{T}"] = {"stats_us": round(t_stats, 2), "fold_requant_us": round(t_req, 2),
                        "gemm_us": round(t_gemm, 2), "rho": round(rho, 5), "rho_model": round(rho_model, 6),
                        "rho_over_model": round(rho / rho_model, 2), "rho_T": round(rho * T, 1)}
        del Xs, Ws, outs, ws
        torch.cuda.empty_cache()
    # the count's structure as times (T >= 2048, the projection at its tensor-core rate):
    # overhead = a + b T, projection time per token constant, rho falling
    import numpy as np

    big = [T for T in Ts if T >= 2048]
    y = np.array([res[f"T{T}"]["stats_us"] + res[f"T{T}"]["fold_requant_us"] for T in big])
    x = np.array(big, dtype=np.float64)
    A = np.stack([np.ones_like(x), x], axis=1) / y[:, None]
    (a_, b_), *_ = np.linalg.lstsq(A, np.ones_like(y), rcond=None)
    per_tok = [res[f"T{T}"]["gemm_us"] / T for T in big]
    res["overhead_fit"] = {"constant_us": round(float(a_), 2), "per_token_ns": round(float(b_) * 1e3, 3),
                           "max_rel_residual": round(float(np.max(np.abs(a_ + b_ * x - y) / y)), 4),
                           "projection_per_token_spread": round(max(per_tok) / min(per_tok), 3),
                           "T": big}
    res["rho_decreasing"] = all(res[f"T{a}"]["rho"] > res[f"T{b}"]["rho"] for a, b in zip(Ts, Ts[1:]))
    assert ttq.device_status() == 0
    return res


def set_roofline_us(layers, T, hbm_peak, tc_peak):
    """Lower bound of one prompt through a set of TTQ linears, stage by stage (the stages
    of a linear depend on each other): statistic 2 B per X element; fold and
    re-quantization 4 B per X element plus 2 + q/8 + 4/g B per weight; low-rank U = X A^T
    2 B per X element; projection the larger of 2 T d d' (+ 2 T r (d + d')) flops at the
    tensor peak and its bytes (X' 2 B per element, codes and scale/zero q/8 + 4/g B per
    weight, Y 2 B per element) at the HBM peak. Peaks in GB/s and TFLOP/s."""
    t = 0.0
    for d, d_out, q, g, r in layers:
        hb = 2 * T * d + 4 * T * d + (2 + q / 8 + 4 / g) * d * d_out + (2 * T * d if r else 0)
        t += hb / (hbm_peak * 1e3)
        fl = 2.0 * T * d * d_out + 2.0 * T * r * (d + d_out)
        gb = 2 * T * d + (q / 8 + 4 / g) * d * d_out + 2 * T * d_out
        t += max(fl / (tc_peak * 1e6), gb / (hbm_peak * 1e3))
    return t


def workload_set_leg(torch, ttq, name, dev, hbm_peak, tc_peak, g=None, n=8):
    """One prompt of T tokens through every linear of a workload's layer set (each linear
    with its own seeded X and W, not chained; statistic, re-quantization and projection
    per linear), L2 flushed before each prompt, timed as the difference of two CUDA graphs
    (n x (flush, set) and n x flush). With r > 0 the static factors are the top-r fp64 SVD
    of each weight (set-up, untimed) and the residual is re-quantized."""
    wl = synthetic.WORKLOADS[name]
    g = g or wl.g
    T = wl.T
    Ls = []
    need = 0
    for i, lin in enumerate(wl.layers):
        X, W = synthetic.draw_layer(T, lin.d, lin.d_out, wl.layer_seed(i))
        Xb, Wb = synthetic.as_bf16(X), synthetic.as_bf16(W)
        A = B = None
        if wl.r > 0:
            B, A, Wb = lowrank_factors(Wb, wl.r, device=dev)
        cfg = ttq.make_config(wl.q, g, wl.alpha, wl.lam, wl.p, wl.r)
        need = max(need, ttq.workspace_size(T, lin.d, lin.d_out, cfg))
        Ls.append({"X": Xb.to(dev), "W": Wb.to(dev), "A": A, "B": B, "cfg": cfg, "out": None})
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    for L in Ls:
        L["out"] = ttq.linear_prefill(L["X"], L["W"], L["cfg"], L["A"], L["B"], ws=ws)
    torch.cuda.synchronize()

    def step(st):
        for L in Ls:
            ttq.linear_prefill(L["X"], L["W"], L["cfg"], L["A"], L["B"], out=L["out"], ws=ws, stream=st)

    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    t_us = graph_step_us(torch, step, flush, sink, n=n)
    assert ttq.device_status() == 0
    roof = set_roofline_us([(lin.d, lin.d_out, wl.q, g, wl.r) for lin in wl.layers], T, hbm_peak, tc_peak)
    flops = sum(2.0 * T * lin.d * lin.d_out for lin in wl.layers)
    del Ls, ws, flush
    torch.cuda.empty_cache()
    return {"linears": [f"{lin.name} {lin.d}->{lin.d_out}" for lin in wl.layers], "T": T, "q": wl.q, "g": g,
            "alpha": wl.alpha, "r": wl.r, "us_per_prompt": round(t_us, 2), "k_tokens_per_s": round(T / t_us * 1e3, 2),
            "projection_TFLOPs": round(flops / (t_us * 1e-6) / 1e12, 1), "roofline_us": round(roof, 2),
            "frac_of_roofline": round(roof / t_us, 4), "l2": "flushed (256 MB read) before each prompt"}


def decoder_leg(torch, ttq, dev, K=3):
    """The chained decoder stack (Qwen3-8B shapes: 36 layers, 4 TTQ linears each, random
    weights): one prompt of T tokens through every layer (each layer re-quantized from its
    own activations), then 128 decode steps reusing the codes, replayed from one captured
    CUDA graph. Weights (14 GB) and codes stream from HBM on every pass (> L2)."""
    from online_activation_aware_b200.decoder import TTQDecoder

    wl = synthetic.WORKLOADS["qwen3_8b_stack"]
    shape = synthetic.QWEN3_SHAPES["8B"]
    T, steps = wl.T, wl.decode_steps
    W = synthetic.device_decoder_weights(shape, wl.r, seed=wl.seed, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed + 1)
    fn = (1.0 + 0.1 * torch.randn(shape["hidden"], generator=gen, device=dev)).to(torch.bfloat16)
    x = torch.randn(T + steps, shape["hidden"], generator=gen, device=dev).to(torch.bfloat16)
    dec = TTQDecoder(shape, W, fn, wl.q, wl.g, wl.alpha, wl.lam, r=wl.r, max_len=T + steps, device=dev)
    for _ in range(2):
        dec.prefill(x[:T])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(K):
        e0.record()
        dec.prefill(x[:T])
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    # the prompt attention alone (layer 0's caches after the prefill), as the difference of
    # two CUDA graphs: causal flops 4 * D * H * T (T + 1) / 2
    H, Hkv, D = shape["heads"], shape["kv_heads"], shape["head_dim"]
    qkv0 = torch.randn(T, (H + 2 * Hkv) * D, generator=gen, device=dev).to(torch.bfloat16)
    aout = torch.empty(T, H * D, dtype=torch.bfloat16, device=dev)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    t_attn = graph_step_us(torch, lambda st: ttq.prompt_attention(qkv0, H, Hkv, D, dec.k_cache[0], dec.v_cache[0],
                                                                   out=aout, stream=st), flush, sink, n=8)
    attn_flops = 4.0 * D * H * T * (T + 1) / 2
    del qkv0, aout, flush
    dec.capture_decode()
    for i in range(4):              # warm the replay, then start over from a fresh prefill
        dec.decode(x[T + i: T + i + 1])
    dec.prefill(x[:T])
    torch.cuda.synchronize()
    e0.record()
    for i in range(steps):
        out = dec.decode(x[T + i: T + i + 1])
    e1.record()
    torch.cuda.synchronize()
    td = e0.elapsed_time(e1)
    ok = bool(torch.isfinite(out.float()).all())
    tp = sorted(ts)[len(ts) // 2]
    flops = 2.0 * T * sum(lin.d * lin.d_out + (lin.cfg.r * (lin.d + lin.d_out))
                          for L in dec.layers for lin in L["lin"].values())
    res = {"model": "Qwen3-8B shapes (architecture table), random-init weights", "layers": shape["layers"],
           "T": T, "decode_steps": steps, "q": wl.q, "g": wl.g, "r": wl.r,
           "linears_per_layer": "qkv (stacked), o, gate_up (stacked), down",
           "prefill_ms": round(tp, 3), "prefill_k_tokens_per_s": round(T / tp, 2),
           "prefill_linear_TFLOPs": round(flops / (tp / 1e3) / 1e12, 1),
           "decode_ms_per_step": round(td / steps, 4), "decode_tokens_per_s": round(steps / (td / 1e3), 1),
           "prompt_plus_decode_ms": round(tp + td, 2), "finite": ok,
           "attention": "the library's own kernels: prompt on the tensor cores, decode split over positions",
           "prompt_attention_us": round(t_attn, 1), "prompt_attention_TFLOPs": round(attn_flops / (t_attn * 1e-6) / 1e12, 1),
           "decode_launch": "one captured CUDA graph per step (device-held position)"}
    del dec, W, x
    torch.cuda.empty_cache()
    return res



if __name__ == "__main__":
    sys.exit(main())
