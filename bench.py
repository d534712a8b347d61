#!/usr/bin/env python
"""Throughput of the routing-weighted SiTU-GLU forward + fused backward on B200.

One step = one forward (situ_glu_fwd) and one backward (situ_glu_bwd, with the
routing-weight gradient) over one synthetic workload resident in HBM.  The
metric is achieved HBM bandwidth from ALGORITHMIC bytes (what the two passes
must move: read gate_up and w, write Y; read gate_up, grad_out and w, write
d_gate_up and d_w), plus rows/s.

    python bench.py [--gpus N --steps K --warmup W] [--config 0..4] [--impl reference]

For N > 1 launch one process per GPU with torchrun; every rank runs the same
per-GPU workload (weak scaling, no collective on the data path), the step
time is the max over ranks, and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "SiTU-GLU fwd/bwd achieved HBM GB/s (% of B200 peak) and rows/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCE = os.path.join(ROOT, "ffn_gated_activation_b200", "csrc", "situ_glu.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=2, help="workload index (default: routed MoE rows)")
    p.add_argument("--beta", type=float, default=None, help="gate beta (default: the workload's first)")
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-oracle sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--flush", choices=["auto", "always", "never"], default="auto",
                   help="flush L2 before every step (auto: when the inputs fit in L2)")
    return p.parse_args(argv)


# ---- helpers ------------------------------------------------------------------

def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_digest() -> str:
    with open(KERNEL_SOURCE, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def recorded_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; None otherwise."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(kernel, {}).get(workload_name)
    if not entry or entry.get("source_sha256") != source_digest():
        return None
    return float(entry["bytes_per_launch"])


def workload_config(wl, beta, l2_note, world):
    rw = {"uniform": "U(0,1) per row", "ones": "1.0 per row",
          "topk_softmax": f"top-{wl.topk} softmax weights of N(0,1) logits over {wl.experts} experts"}[wl.rw_kind]
    return {
        "workload": wl.describe(),
        "name": wl.name,
        "tokens": wl.tokens,
        "inter": wl.inter,
        "storage_dtype": wl.dtype,
        "beta": beta,
        "linear_beta": wl.linear_beta,
        "routing_weights": rw,
        "inputs": f"G~N(0,{wl.g_std}), U~N(0,{wl.u_std})"
                  + (f", {wl.outlier_p:.0%} outliers +-U({wl.outlier_lo:g},{wl.outlier_hi:g})" if wl.outlier_p else "")
                  + f", grad_out~N(0,{wl.go_std}), seed {wl.seed}",
        "l2": l2_note,
        "parallelism": f"replicas x{world} (weak scaling; rows independent, no collective)",
    }


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while the
    timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML unavailable: record why
            self.nvml, self.err = None, f"{type(e).__name__}: {e}"

    def _reasons(self):
        n = self.nvml
        fn = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or n.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.handle)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                mask = self._reasons()
                watts = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.samples.append((mhz, mask, watts))
            except Exception as e:
                self.err = f"{type(e).__name__}: {e}"
                return
            time.sleep(0.001)

    def start(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no sample"}
        mask = 0
        for _, m, _ in self.samples:
            mask |= m
        names = sorted(v for k, v in self.REASONS.items() if mask & k and v != "gpu_idle")
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1), "source": "nvml"}


def cpu_oracle_rate(wl, beta, x, seconds: float):
    """The fp64 oracle (single thread, as it stands) on the first rows of the
    workload, fwd then bwd per chunk of rows, until ``seconds`` have passed.
    Returns (GB/s of algorithmic bytes, rows done, elapsed)."""
    import oracle
    o = oracle.load()
    per_row = (wl.fwd_bytes() + wl.bwd_bytes()) / wl.tokens
    chunk = max(1, min(64, int(2 ** 20 // wl.inter)))
    done, t0 = 0, time.perf_counter()
    while done < wl.tokens:
        rows = np.arange(done, min(wl.tokens, done + chunk), dtype=np.int64)
        o.fwd(x["gate_up"], x["routing_weights"], beta, wl.linear_beta, rows=rows)
        o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], beta, wl.linear_beta, rows=rows)
        done += rows.size
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return per_row * done / dt / 1e9, done, dt


# ---- the reference arm: the fp64 oracle on the host cores -------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0  # the CPU arm runs once, on rank 0
    wl = workloads.workload(args.config)
    beta = args.beta if args.beta is not None else wl.betas[0]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rows_per_step = max(1, min(wl.tokens, (1 << 17) // wl.inter))
    x = workloads.inputs(wl, tokens=rows_per_step)
    import oracle
    o = oracle.load()
    per_row = (wl.fwd_bytes() + wl.bwd_bytes()) / wl.tokens

    def step():
        o.fwd(x["gate_up"], x["routing_weights"], beta, wl.linear_beta)
        o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], beta, wl.linear_beta)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_row * rows_per_step * args.steps / dt / 1e9
    sample = (f"{rows_per_step} of {wl.tokens} rows per step (fwd + bwd), {args.steps} steps, "
              f"single-threaded fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(wl, beta, "n/a (host)", 1),
        "rows_per_s": rows_per_step * args.steps / dt,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- our arm -----------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    import ffn_gated_activation_b200 as pkg

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and not (world == 1 and args.gpus == 1):
        if world == 1:
            raise SystemExit(f"--gpus {args.gpus}: launch one process per GPU with torchrun")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = workloads.workload(args.config)
    beta = args.beta if args.beta is not None else wl.betas[0]
    lb = wl.linear_beta
    T, I = wl.tokens, wl.inter
    x = workloads.inputs(wl)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def upload(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.pin_memory()

    gu_h, go_h = upload(x["gate_up"]), upload(x["grad_out"])
    rw_h = torch.from_numpy(x["routing_weights"]).reshape(T, 1).pin_memory()
    gu = gu_h.to(dev)
    go = go_h.to(dev)
    rw = rw_h.to(dev)
    y = torch.empty(T, I, dtype=tdt, device=dev)
    d_gu = torch.empty(T, 2 * I, dtype=tdt, device=dev)
    d_rw = torch.empty(T, 1, dtype=torch.float32, device=dev)

    input_bytes = gu.numel() * gu.element_size() + go.numel() * go.element_size() + rw.numel() * 4
    flush = args.flush == "always" or (args.flush == "auto" and input_bytes < 2 * L2_BYTES)
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    l2_note = (f"L2 flushed before every step by writing {2 * L2_BYTES >> 20} MB (flush not timed)" if flush
               else f"inputs ({input_bytes / 1e6:.0f} MB) exceed the {L2_BYTES >> 20} MB L2; no flush")

    def fwd():
        pkg.situ_glu_fwd(gu, rw, beta, lb, out=y)

    def bwd():
        pkg.situ_glu_bwd(gu, rw, go, beta, lb, d_gate_up=d_gu, d_rw=d_rw)

    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        if flush:
            flush_buf.zero_()
        fwd()
        bwd()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    outer0, outer1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    outer0.record(stream)
    for k in range(K):
        if flush:
            flush_buf.zero_()
        ev[k][0].record(stream)
        fwd()
        ev[k][1].record(stream)
        bwd()
        ev[k][2].record(stream)
    outer1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    bwd_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(K)]
    total_ms = sum(fwd_ms) + sum(bwd_ms) if flush else outer0.elapsed_time(outer1)
    times = torch.tensor([total_ms, sum(fwd_ms), sum(bwd_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    total_ms, fwd_sum, bwd_sum = times.tolist()
    ms_per_step = total_ms / K
    step_bytes = wl.fwd_bytes() + wl.bwd_bytes()
    value = step_bytes * world / (ms_per_step / 1e3) / 1e9
    peak, peak_src = measured_peak()
    fwd_us, bwd_us = fwd_sum / K * 1e3, bwd_sum / K * 1e3
    fwd_gbs, bwd_gbs = wl.fwd_bytes() / fwd_us / 1e3, wl.bwd_bytes() / bwd_us / 1e3
    traffic = recorded_traffic("situ_glu_bwd_kernel", wl.name)

    # End to end through the public API with host buffers: every step copies the
    # inputs from pinned host memory, runs both passes and reads all outputs back.
    e2e = None
    if not args.no_e2e:
        y_h = torch.empty(T, I, dtype=tdt).pin_memory()
        d_gu_h = torch.empty(T, 2 * I, dtype=tdt).pin_memory()
        d_rw_h = torch.empty(T, 1, dtype=torch.float32).pin_memory()
        K2 = args.e2e_steps or max(1, min(K, 20))

        def e2e_step():
            gu.copy_(gu_h, non_blocking=True)
            go.copy_(go_h, non_blocking=True)
            rw.copy_(rw_h, non_blocking=True)
            fwd()
            bwd()
            y_h.copy_(y, non_blocking=True)
            d_gu_h.copy_(d_gu, non_blocking=True)
            d_rw_h.copy_(d_rw, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K2):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        t = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item() / K2
        h2d = input_bytes
        d2h = y_h.numel() * y_h.element_size() + d_gu_h.numel() * d_gu_h.element_size() + d_rw_h.numel() * 4
        e2e = {"value": step_bytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": K2,
               "api": "ffn_gated_activation_b200.situ_glu_fwd/situ_glu_bwd on pinned host copies"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows_done, secs = cpu_oracle_rate(wl, beta, x, args.cpu_seconds)
        cpu = {"value": rate, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"first {rows_done} of {T} rows, fwd + bwd, {secs:.1f} s, single-threaded fp64"}

    launches_per_step = 2
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, beta, l2_note, world),
            "rows_per_s": T * world / (ms_per_step / 1e3),
            "pct_of_nominal_hbm": value / world / NOMINAL_HBM_GBS * 100.0,
            "kernels": {
                "situ_glu_fwd_kernel": {"us": fwd_us, "bytes": wl.fwd_bytes(), "GB/s": fwd_gbs,
                                        "pct_of_nominal_8TBs": fwd_gbs / NOMINAL_HBM_GBS * 100,
                                        "frac_of_measured_copy": fwd_gbs / peak,
                                        "rows_per_s": T / (fwd_us / 1e6)},
                "situ_glu_bwd_kernel": {"us": bwd_us, "bytes": wl.bwd_bytes(), "GB/s": bwd_gbs,
                                        "pct_of_nominal_8TBs": bwd_gbs / NOMINAL_HBM_GBS * 100,
                                        "frac_of_measured_copy": bwd_gbs / peak,
                                        "rows_per_s": T / (bwd_us / 1e6)},
            },
            "roofline": {"bound": "hbm", "kernel": "situ_glu_bwd_kernel", "achieved": bwd_gbs, "peak": peak,
                         "unit": "GB/s", "frac": bwd_gbs / peak, "peak_source": f"{peak_src} copy bandwidth",
                         "traffic": traffic},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * K,
            "clocks": clocks.summary(),
            "device_status": pkg.abi.situ_glu_device_status(0),
            "device": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
