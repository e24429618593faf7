#!/usr/bin/env python
"""Benchmark of the attention hot path: one step = forward (fa_fwd) + backward (fa_bwd) of
exact attention on one batch of seeded synthetic bf16 inputs, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--dropout P]
                    [--impl reference]

Prints ONE JSON line (rank 0). ``value`` is whole-job attention TFLOP/s (fwd + bwd) with
inputs resident in device memory; ``e2e`` is the same metric with pinned-host inputs copied in
and every output copied back inside the timed region. Multi-GPU runs (torchrun) are
independent replicas of the same workload, one per GPU (weak scaling); the only collectives
are the barrier and the max-over-ranks of the timing.

FLOP accounting: forward 4 B H N^2 d, backward 2.5x forward, both halved when causal.
``--fp8`` times the FP8 (E4M3) forward of the workload instead (fa_fwd_fp8, forward only, its
FLOPs counted as for bf16, the roofline against twice the measured bf16 peak — the nominal
FP8/bf16 ratio). ``--dropout P`` runs the same step with dropout probability P on the attention probabilities
(fa_fwd_ex / fa_bwd_ex, a new Philox offset every step); the FLOP count is unchanged.
``--impl reference`` times the fp64 CPU oracle on the host instead, on bounded samples of the
same workload. A single-GPU run of the default workload also times, after the headline, the
metric's other N >= 4096 configurations (B1 H16 N16384 d128 causal forward + backward, B1 H8
N131072 d128 causal forward; 5 steps each after 3 warm-up, L2 flushed) and reports them under
``per_config`` (``--no-per-config`` skips this).
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from exact_io_aware_66_b200.workloads import WORKLOADS, workload_inputs  # noqa: E402

DEFAULT_WORKLOAD = "causal_train_b4h16n4096d128"
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 512 * 1024 * 1024
KERNEL_SOURCES = ["exact_io_aware_66_b200/csrc/fa_bwd.cuh", "exact_io_aware_66_b200/csrc/fa_fwd.cuh",
                  "exact_io_aware_66_b200/csrc/fa_bwd_q128.cuh",
                  "exact_io_aware_66_b200/csrc/fa_fwd_d256.cuh",
                  "exact_io_aware_66_b200/csrc/fa_bwd_d256.cuh",
                  "exact_io_aware_66_b200/csrc/sm100.cuh", "exact_io_aware_66_b200/csrc/fa_api.cu",
                  "exact_io_aware_66_b200/csrc/dropout.cuh",
                  "exact_io_aware_66_b200/csrc/fa_fwd_fp8.cuh"]


# The headline metric: attention TFLOP/s of the forward and forward+backward passes in bf16
# for N = 4k..128k, and their fraction of the B200's dense bf16 peak.
METRIC = "attention TFLOP/s (fwd, fwd+bwd) bf16 N=4k\u2013128k; % of B200 dense BF16 peak"


def load_metric() -> str:
    return METRIC


def load_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"bf16_burst": float(d["bf16_tflops"]),
                "bf16_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_burst": 1590.0, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0,
                "source": "fallback"}


def peak_label(peaks: dict, kind: str) -> str:
    if peaks["source"] == "measured":
        return f"measured bf16 {kind} (MEASURED_PEAKS.json)"
    return f"fallback bf16 {kind} (no MEASURED_PEAKS.json)"


def _code_only(src: str) -> str:
    """The source without comments and blank lines: what the compiler sees."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def sources_hash() -> str:
    """Fingerprint of the kernel and host sources (comments excluded), recorded with each ncu
    capture so that bench.py reports its traffic only while the code is unchanged."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was taken on the
    current kernel sources (same source hash); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("sources_hash") != sources_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# --------------------------------------------------------------------------------------------
# Clock sampling (nvidia-smi) during the timed region
# --------------------------------------------------------------------------------------------
REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """SM clocks and clock-event reasons during the timed region, read-only.

    nvidia-smi samples every 200 ms; a short timed region can end before its first sample, so
    an NVML polling thread (10 ms) runs beside it and its samples are reported when nvidia-smi
    has none."""

    NVML_BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                 "sw_power_cap": 0x4}

    def __init__(self, device: int):
        self.proc = None
        self.thread = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(device)

    def _nvml_loop(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu)
                maxmhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
                reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
                while not self.stop_evt.is_set():
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    bits = reasons_fn(h)
                    self.nvml.append((time.time(), float(mhz), float(maxmhz), int(bits)))
                    self.stop_evt.wait(0.01)
            finally:
                pynvml.nvmlShutdown()
        except Exception:
            pass

    def start(self):
        import threading

        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.nvml = []
        self.stop_evt = threading.Event()
        self.thread = threading.Thread(target=self._nvml_loop, daemon=True)
        self.thread.start()
        t0 = time.time()  # let the NVML thread take its first sample before the region starts
        while not self.nvml and self.thread.is_alive() and time.time() - t0 < 2.0:
            time.sleep(0.002)
        self.t_region = time.time()

    def stop(self) -> dict | None:
        out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
        mhz, maxmhz, reasons = [], [], set()
        for line in (out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                mhz.append(float(parts[1]))
                maxmhz.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(REASONS, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        source = "nvidia-smi"
        if not mhz and self.thread is not None:
            source = "nvml"
            inside = [x for x in self.nvml if x[0] >= self.t_region] or self.nvml
            for _, m, mx, bits in inside:
                mhz.append(m)
                maxmhz.append(mx)
                reasons.update(n for n, b in self.NVML_BITS.items() if bits & b)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxmhz),
                "reasons": sorted(reasons), "samples": len(mhz), "source": source}


# --------------------------------------------------------------------------------------------
# Distributed plumbing (replicas only)
# --------------------------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------------------------
# CPU baseline: the fp64 oracle, as it stands
# --------------------------------------------------------------------------------------------
def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_head_step(x, w, heads, prefix: int | None = None, dropout: float = 0.0,
                     fp8: bool = False):
    """Oracle fwd+bwd of the given (b, h) heads, optionally restricted to the first `prefix`
    rows and keys (a self-contained sub-problem under the causal mask). Returns FLOPs done."""
    import numpy as np

    import oracle

    n = w.N if prefix is None else prefix
    if fp8:
        from oracle.fp8 import attention_forward_fp8

        for b, h in heads:
            codes = [x[t][b, h, :n].view(torch.uint8).numpy() for t in ("q8", "k8", "v8")]
            attention_forward_fp8(*codes, *x["descale"], w.scale, w.causal)
        f = 4.0 * n * n * w.d * len(heads)
        return f / 2 if w.causal else f
    for b, h in heads:
        q, k, v = (x[t][b, h, :n].float().numpy().astype(np.float64) for t in ("q", "k", "v"))
        dr = (dropout, 1, 0) if dropout > 0 else None
        if w.backward:
            do = x["do"][b, h, :n].float().numpy().astype(np.float64)
            oracle.attention_backward(q, k, v, do, w.scale, w.causal, dropout=dr)
        else:
            oracle.attention_forward(q, k, v, w.scale, w.causal, dropout=dr)
    f = 4.0 * n * n * w.d * (3.5 if w.backward else 1.0) * len(heads)
    return f / 2 if w.causal else f


def cpu_baseline(w, x, budget_s: float = 12.0, dropout: float = 0.0, fp8: bool = False) -> dict:
    heads_all = [(b, h) for b in range(w.B) for h in range(w.H)]
    t0 = time.perf_counter()
    flops = oracle_head_step(x, w, heads_all[:1], prefix=min(w.N, 4096), dropout=dropout, fp8=fp8)
    one = time.perf_counter() - t0
    prefix = min(w.N, 4096)
    nh = max(1, min(len(heads_all), int(budget_s / max(one, 1e-3))))
    heads = heads_all[:nh]
    t0 = time.perf_counter()
    flops = oracle_head_step(x, w, heads, prefix=prefix, dropout=dropout, fp8=fp8)
    dt = time.perf_counter() - t0
    bwd = w.backward and not fp8
    sample = (f"oracle {'fp8 ' if fp8 else ''}fwd{'+bwd' if bwd else ''} (fp64 NumPy) of {nh} of "
              f"{len(heads_all)} "
              f"heads" + (f", first {prefix} rows/keys of each" if prefix < w.N else "")
              + f"; {dt:.1f} s")
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(),
            "kind": "oracle", "sample": sample}


def run_reference(args, w, world, rank):
    """The reference arm: the fp64 CPU oracle on bounded samples of the same workload."""
    if rank != 0:
        return 0
    if args.fp8:
        from exact_io_aware_66_b200.workloads import make_inputs_fp8

        x = make_inputs_fp8(w.B, w.H, w.H, w.N, w.N, w.d, seed=w.seed)
    else:
        x = workload_inputs(w)
    steps, warm = args.steps, args.warmup
    budget_per_step = max(0.05, 150.0 / (steps + warm))
    # calibrate a causal-prefix length (multiple of 128) so one step takes about the budget
    t0 = time.perf_counter()
    oracle_head_step(x, w, [(0, 0)], prefix=min(w.N, 1024), fp8=args.fp8)
    t1024 = time.perf_counter() - t0
    n = int(min(w.N, 1024 * (budget_per_step / max(t1024, 1e-4)) ** 0.5))
    n = max(128, n // 128 * 128)
    heads = [(0, 0)]
    for _ in range(warm):
        oracle_head_step(x, w, heads, prefix=n, dropout=args.dropout, fp8=args.fp8)
    t0 = time.perf_counter()
    flops = 0.0
    for s in range(steps):
        b, h = divmod(s % (w.B * w.H), w.H)
        flops += oracle_head_step(x, w, [(b, h)], prefix=n, dropout=args.dropout, fp8=args.fp8)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    bwd = w.backward and not args.fp8
    sample = (f"per step: oracle {'fp8 ' if args.fp8 else ''}fwd{'+bwd' if bwd else ''} "
              f"(fp64 NumPy) of one head, "
              f"first {n} of {w.N} rows/keys")
    line = {"impl": "reference", "metric": load_metric(), "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": dt * 1000 / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1), bf16-rounded, widened to fp64)",
            "config": workload_config(w, world, args.dropout, args.fp8),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world, dropout: float = 0.0, fp8: bool = False) -> dict:
    bwd = w.backward and not fp8
    return {"workload": w.name + (f"+dropout{dropout:g}" if dropout > 0 else "")
                        + ("+fp8fwd" if fp8 else ""),
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "pass": "fwd (E4M3 Q, K, V)" if fp8 else ("fwd+bwd" if bwd else "fwd"),
            "scale": "1/sqrt(d)", "dropout": dropout,
            "flops_per_step": w.fwd_flops() + (w.bwd_flops() if bwd else 0.0),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"{FLUSH_BYTES >> 20} MiB buffer written before every timed step "
                  f"(L2 is {L2_BYTES >> 20} MiB)"}


# --------------------------------------------------------------------------------------------
# The other target configurations of the metric's N range, timed beside the headline
# --------------------------------------------------------------------------------------------
PER_CONFIG = ("causal_train_b1h16n16384d128", "causal_fwd_b1h8n131072d128")


def time_config(name: str, dev, steps: int, warmup: int, peaks: dict) -> dict:
    """Forward (and backward, if the workload has one) of workload `name` through the C ABI,
    inputs resident, L2 flushed before every step; per-pass device time from the library's own
    per-kernel events. Returns TFLOP/s and fractions of the measured burst peak."""
    from exact_io_aware_66_b200 import fa

    w = WORKLOADS[name]
    x = workload_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    if w.backward:
        do = x["do"].to(dev)
        ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                         device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    del x
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        fa.fa_fwd(q, k, v, o, lse, w.causal, None, stream)
        if w.backward:
            fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, w.causal, None, stream)

    for _ in range(warmup):
        step()
    fa.fa_check_status(stream)
    fa.fa_profile_read()
    fa.fa_profile_enable(True)
    for _ in range(steps):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    fa.fa_profile_enable(False)
    prof = fa.fa_profile_read()
    fa.fa_check_status(stream)
    fwd_ms = prof["fa_fwd_kernel"][1] / steps
    out = {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "steps": steps,
           "fwd_tflops": w.fwd_flops() / (fwd_ms / 1e3) / 1e12}
    out["fwd_frac_of_peak"] = out["fwd_tflops"] / peaks["bf16_burst"]
    if w.backward:
        bwd_ms = sum(prof[n][1] for n in ("fa_bwd_preprocess", "fa_bwd_main",
                                           "fa_bwd_dq_convert")) / steps
        out["bwd_tflops"] = w.bwd_flops() / (bwd_ms / 1e3) / 1e12
        out["fwd_bwd_tflops"] = (w.fwd_flops() + w.bwd_flops()) / ((fwd_ms + bwd_ms) / 1e3) / 1e12
        out["fwd_bwd_frac_of_peak"] = out["fwd_bwd_tflops"] / peaks["bf16_burst"]
    out["peak_source"] = peak_label(peaks, "burst")
    return out


# --------------------------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dropout", type=float, default=0.0)
    ap.add_argument("--fp8", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other N >= 4096 configurations beside the headline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if not 0.0 <= args.dropout < 1.0:
        ap.error("--dropout must be in [0, 1)")
    if args.fp8 and args.dropout > 0:
        ap.error("--fp8 has no dropout")
    w = WORKLOADS[args.workload]
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, w, world, rank)
    if world > 1:  # each replica computes its own units: inputs seeded per rank
        import dataclasses

        w = dataclasses.replace(w, seed=w.seed + 7919 * rank)

    from exact_io_aware_66_b200 import fa

    fa.lib()  # fails loudly if the CUDA library is missing: there is no fallback
    dev = torch.device("cuda", local)
    backward = w.backward and not args.fp8
    if args.fp8:
        from exact_io_aware_66_b200.workloads import make_inputs_fp8

        x = make_inputs_fp8(w.B, w.H, w.H, w.N, w.N, w.d, seed=w.seed)
        in_names = ("q8", "k8", "v8")
        q, k, v = (x[n].to(dev) for n in in_names)
        o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
        ws8 = torch.empty(max(16, fa.fa_fwd_fp8_workspace_size(w.B, w.H, w.H, w.N, w.N, w.d,
                                                                 w.causal)),
                          dtype=torch.uint8, device=dev)
    else:
        x = workload_inputs(w)
        in_names = ("q", "k", "v", "do") if backward else ("q", "k", "v")
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
    do = x["do"].to(dev) if backward else None
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    if backward:
        ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                         device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)
    counter = [0]

    def step(q_, k_, v_, do_):
        if args.fp8:
            fa.fa_fwd_fp8(q_, k_, v_, x["descale"], o, lse, w.causal, None, stream, ws8)
            return
        if args.dropout > 0:
            dr = (args.dropout, 0x5EED, counter[0])  # a fresh Philox offset every step
            counter[0] += 1
            fa.fa_fwd_ex(q_, k_, v_, o, lse, w.causal, None, stream, dr)
            if backward:
                fa.fa_bwd_ex(q_, k_, v_, o, do_, lse, dq, dk, dv, ws, w.causal, None, stream, dr)
            return
        fa.fa_fwd(q_, k_, v_, o, lse, w.causal, None, stream)
        if backward:
            fa.fa_bwd(q_, k_, v_, o, do_, lse, dq, dk, dv, ws, w.causal, None, stream)

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step(q, k, v, do)
    fa.fa_check_status(stream)
    cfg = workload_config(w, world, args.dropout, args.fp8)
    flops_step = cfg["flops_per_step"]

    # ---- timed region: K steps, L2 flushed before each (outside the event pairs) ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    fa.fa_profile_read()
    fa.fa_profile_enable(True)
    for s in range(args.steps):
        flush.zero_()
        starts[s].record(stream)
        step(q, k, v, do)
        ends[s].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop()
    fa.fa_profile_enable(False)
    prof = fa.fa_profile_read()
    fa.fa_check_status(stream)
    ms_total = sum(a.elapsed_time(b) for a, b in zip(starts, ends))
    ms_total = max_over_ranks(ms_total, world)
    value = flops_step * args.steps * world / (ms_total / 1e3) / 1e12
    ms_step = ms_total / args.steps

    # per-kernel device time from the library's own event pairs
    kern = {name: {"launches": n, "ms": t} for name, (n, t) in prof.items() if n}
    fwd_ms = sum(kern.get(n, {}).get("ms", 0.0)
                 for n in ("fa_fwd_kernel", "fa_fwd_d256_kernel", "fa_fwd_fp8_kernel",
                           "fa_fp8_transpose_v")) / args.steps
    bwd_ms = sum(kern.get(n, {}).get("ms", 0.0)
                 for n in ("fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_dq_convert",
                           "fa_bwd_d256_dv", "fa_bwd_d256_dkdq")) / args.steps
    peaks = load_peaks()
    dom = max(kern, key=lambda n: kern[n]["ms"])
    # algorithmic FLOPs per launch of each main kernel; the d = 256 backward splits its five
    # products over two passes (the dV pass: dV; the dK/dQ pass: dP, dK, dQ; S in both), so each
    # is credited with its share of the backward's 2.5 x forward
    dom_flops = {"fa_fwd_kernel": w.fwd_flops(), "fa_bwd_main": w.bwd_flops(),
                 "fa_fwd_fp8_kernel": w.fwd_flops(), "fa_fwd_d256_kernel": w.fwd_flops(),
                 "fa_bwd_d256_dv": w.bwd_flops() * 1.0 / 5.0,
                 "fa_bwd_d256_dkdq": w.bwd_flops() * 4.0 / 5.0}.get(dom)
    avg_ms = kern[dom]["ms"] / kern[dom]["launches"]
    sustained = ms_total > 1000
    peak = peaks["bf16_sustained"] if sustained else peaks["bf16_burst"]
    peak_source = peak_label(peaks, "sustained" if sustained else "burst")
    if dom == "fa_fwd_fp8_kernel":  # E4M3 contraction: nominal FP8/bf16 dense ratio 4.5/2.25
        peak *= 2.0
        peak_source += " x 2 (nominal fp8/bf16 dense ratio)"
    achieved = dom_flops / (avg_ms / 1e3) / 1e12 if dom_flops else None
    roofline = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak if achieved else None,
                "traffic": ncu_traffic(dom, cfg["workload"]),
                "peak_source": peak_source, "per_launch_flops": dom_flops, "avg_launch_ms": avg_ms}

    # ---- end-to-end: pinned host inputs in, every output back, inside the timed region ----
    # As an input pipeline would run it: three streams (host-to-device copies, the library's
    # kernels, device-to-host copies) and two sets of device buffers, so that step k's inputs
    # travel while step k-1 computes and step k-2's outputs come back. Every step still copies
    # its own inputs in and all of its outputs out.
    host_in = {n: x[n].pin_memory() for n in in_names}
    outs = [o, lse] + ([dq, dk, dv] if backward else [])
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    dev_in = [{n: torch.empty_like(t, device=dev) for n, t in host_in.items()} for _ in range(2)]
    dev_out = [[torch.empty_like(t) for t in outs] for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
                for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def compute_into(b):
        d_in, d_out = dev_in[b], dev_out[b]
        q_, k_, v_ = (d_in[n] for n in in_names[:3])
        if args.fp8:
            fa.fa_fwd_fp8(q_, k_, v_, x["descale"], d_out[0], d_out[1], w.causal, None, stream,
                          ws8)
            return
        dr = None
        if args.dropout > 0:
            dr = (args.dropout, 0x5EED, counter[0])
            counter[0] += 1
        fa.fa_fwd_ex(q_, k_, v_, d_out[0], d_out[1], w.causal, None, stream, dr)
        if backward:
            fa.fa_bwd_ex(q_, k_, v_, d_out[0], d_in["do"], d_out[1], d_out[2], d_out[3],
                         d_out[4], ws, w.causal, None, stream, dr)

    def e2e_step(k_step):
        b = k_step % 2
        s_in.wait_event(ev_cmp[b])  # the kernels of step k-2 are done with dev_in[b]
        with torch.cuda.stream(s_in):
            for n, t in host_in.items():
                dev_in[b][n].copy_(t, non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # step k-2's outputs have left dev_out[b]
        compute_into(b)
        ev_cmp[b].record(stream)
        s_out.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_out):
            for t, h in zip(dev_out[b], host_out[b]):
                h.copy_(t, non_blocking=True)
        ev_out[b].record(s_out)

    for k_step in range(3):
        e2e_step(k_step)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k_step in range(args.e2e_steps):
        e2e_step(k_step)
    s_out.wait_event(ev_cmp[(args.e2e_steps - 1) % 2])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(world)
    fa.fa_check_status(stream)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e = {"value": flops_step * args.e2e_steps * world / (e2e_ms / 1e3) / 1e12,
           "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": args.e2e_steps,
           "pipeline": "h2d / kernels / d2h on three streams, two device buffer sets"}

    # the metric's other target configurations (N = 16384 fwd+bwd, N = 131072 fwd), timed on
    # rank 0 of a single-GPU run of the default workload
    per_config = None
    if (rank == 0 and world == 1 and not args.no_per_config and args.workload == DEFAULT_WORKLOAD
            and not args.fp8 and args.dropout == 0):
        del host_in, dev_in, dev_out, host_out
        per_config = {name: time_config(name, dev, 5, 3, peaks) for name in PER_CONFIG}
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x, dropout=args.dropout, fp8=args.fp8)

    if rank == 0:
        line = {
            "metric": load_metric(), "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if args.fp8 else "bf16",
            "data": "synthetic (seeded N(0,1)" + (f" x{w.mult}" if w.mult != 1 else "")
                    + (", E4M3 with per-tensor descale" if args.fp8 else ", bf16")
                    + "), inputs resident in device memory",
            "config": cfg,
            "fwd_tflops": w.fwd_flops() / (fwd_ms / 1e3) / 1e12 if fwd_ms else None,
            "bwd_tflops": (w.bwd_flops() / (bwd_ms / 1e3) / 1e12) if bwd_ms else None,
            "frac_of_peak": {"fwd+bwd": value / world / peaks["bf16_burst"],
                             "fwd": (w.fwd_flops() / (fwd_ms / 1e3) / 1e12) / peaks["bf16_burst"]
                             if fwd_ms else None,
                             "peak": peaks["bf16_burst"],
                             "peak_source": peak_label(peaks, "burst")},
            "roofline": roofline,
            "kernels": kern,
            "per_config": per_config,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": sum(v["launches"] for v in kern.values()),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
