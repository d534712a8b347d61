#!/usr/bin/env python
"""Throughput of the routing-weighted SiTU-GLU forward + fused backward on B200.

One step = one forward (situ_glu_fwd) and one backward (situ_glu_bwd, with the
routing-weight gradient) over one synthetic workload resident in HBM.  The
metric is achieved HBM bandwidth from ALGORITHMIC bytes (what the two passes
must move: read gate_up and w, write Y; read gate_up, grad_out and w, write
d_gate_up and d_w), plus rows/s.

    python bench.py [--gpus N --steps K --warmup W] [--config 0..4] [--impl reference]
                    [--variant row|col|full|mxfp8|nvfp4|fc1|fc2|attn_res]

--variant picks the form timed (default: per-row routing weights, the routed
MoE form): per-column [I] or per-element [T, I] weights, or MXFP8 outputs
(E4M3 codes + E8M0 scales for Y and d_gate_up, OCP rule), or an NVFP4 Y
and d_gate_up (E2M1 codes + E4M3 scales per 16 + the tensor maximum; the
quantising kernels are also timed alone, and the backward's is the roofline).  Algorithmic
bytes follow the form (weights read, weight gradients written, one byte per
code plus one per 32 codes).  --variant fc1 times the fused FC1 grouped GEMM
+ SiTU-GLU forward on the routed-MoE rows (hidden 7168, 8 local experts) in
TFLOP/s against the tensor-core peak, with the unfused cuBLAS GEMMs +
SiTU-GLU kernel timed beside it; --variant fc2 the fused FC2 data gradient
+ SiTU-GLU backward on the same rows (against cuBLAS GEMMs + situ_glu_bwd).
--variant attn_res times the
attention-residual mixing core (16384 tokens, 8 stored sums + the current
sum, hidden 7168, bf16) in GB/s of algorithmic bytes (every source value read
once, the output written once).

For N > 1 launch one process per GPU with torchrun; every rank runs the same
per-GPU workload (weak scaling, no collective on the data path), the step
time is the max over ranks, and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
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
KERNEL_SOURCES = [os.path.join(ROOT, "ffn_gated_activation_b200", "csrc", n)
                  for n in ("situ_glu.cu", "situ_fused_gemm.cuh")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=4,
                   help="workload index (default: the large one, bf16 [131072, 8192])")
    p.add_argument("--tokens", type=int, default=None,
                   help="rows of the workload (default: its own); for small profiler captures")
    p.add_argument("--no-sub", action="store_true",
                   help="skip the per-workload records of the other target workloads")
    p.add_argument("--beta", type=float, default=None, help="gate beta (default: the workload's first)")
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-oracle sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--variant", choices=["row", "col", "full", "mxfp8", "nvfp4", "fc1", "fc2", "attn_res"],
                   default="row",
                   help="routing-weight form or output format timed (default: per-row weights)")
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


def link_bandwidth(torch, dev, host_in, dev_in, dev_out, host_out, reps: int = 2) -> dict:
    """PCIe between pinned host memory and the device, measured in this run
    with the bench's own buffers: host_in -> dev_in alone, dev_out -> host_out
    alone, then both at once on two streams (CUDA events; the best of
    ``reps``; GB/s per direction)."""
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    nb_up = host_in.numel() * host_in.element_size()
    nb_down = host_out.numel() * host_out.element_size()

    def timed(streams_ops):
        torch.cuda.synchronize()
        marks = []
        for s, op in streams_ops:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s)
            with torch.cuda.stream(s):
                op()
            b.record(s)
            marks.append((a, b))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in marks]

    h2d = lambda: dev_in.copy_(host_in, non_blocking=True)
    d2h = lambda: host_out.copy_(dev_out, non_blocking=True)
    alone_up = min(timed([(up, h2d)])[0] for _ in range(reps))
    alone_down = min(timed([(down, d2h)])[0] for _ in range(reps))
    both = [timed([(up, h2d), (down, d2h)]) for _ in range(reps)]
    both_up, both_down = min(b[0] for b in both), min(b[1] for b in both)
    rate = lambda nb, ms: nb / (ms / 1e3) / 1e9
    return {"h2d_GB/s": rate(nb_up, alone_up), "d2h_GB/s": rate(nb_down, alone_down),
            "both_h2d_GB/s": rate(nb_up, both_up), "both_d2h_GB/s": rate(nb_down, both_down),
            "bytes_h2d": nb_up, "bytes_d2h": nb_down,
            "how": "copy_ between pinned host and device buffers of this run, CUDA events, best of %d" % reps}


class L2Flush:
    """Leaves the L2 cold and clean before a timed kernel: writes a buffer of
    twice the L2 (which evicts whatever the last kernel left there), then reads
    another of the same size, so the written lines are written back here and
    not inside the next timed kernel.  Neither buffer is timed."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.dirty = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.clean = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.dirty.zero_()
        self.torch.amax(self.clean)


def copy_bandwidth(torch, dev, stream, nbytes: int = 1 << 31, reps: int = 10) -> dict:
    """A device-to-device copy measured in this run: ``dst.copy_(src)`` of
    ``nbytes`` (one read and one write of every byte) on ``stream``, 3 untimed
    copies, then ``reps`` timed one by one with CUDA events.  GB/s count
    2 * nbytes; the median is the figure, the best beside it."""
    src = torch.ones(nbytes // 2, dtype=torch.bfloat16, device=dev)
    dst = torch.empty_like(src)
    with torch.cuda.stream(stream):
        for _ in range(3):
            dst.copy_(src)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in evs:
            e0.record(stream)
            dst.copy_(src)
            e1.record(stream)
    torch.cuda.synchronize()
    ms = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
    del src, dst
    torch.cuda.empty_cache()
    rate = lambda m: 2 * nbytes / (m / 1e3) / 1e9
    return {"GB/s": rate(ms[len(ms) // 2]), "GB/s_best": rate(ms[0]), "bytes_per_copy": nbytes, "copies": reps,
            "how": "torch copy_ between two device buffers (read + write counted), CUDA events, median of the copies"}


def add_copy_fractions(copy: dict, *records) -> None:
    """Each record with a GB/s figure gains its fraction of the same-run copy."""
    for rec in records:
        if isinstance(rec, dict) and "GB/s" in rec:
            rec["frac_of_copy_same_run"] = rec["GB/s"] / copy["GB/s"]


def host_info() -> dict:
    """The host the CPU figures were taken on: CPU model and core counts."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count()
    return {"cpu_model": model, "host_cores": os.cpu_count(), "cores_available": avail}


class PinnedCore:
    """Runs the calling thread on one core of its affinity set (the first),
    and puts the set back on exit; ``core`` is None where affinity cannot be
    set."""

    def __enter__(self):
        self.saved, self.core = None, None
        try:
            self.saved = os.sched_getaffinity(0)
            self.core = min(self.saved)
            os.sched_setaffinity(0, {self.core})
        except (AttributeError, OSError):
            self.core = None
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            try:
                os.sched_setaffinity(0, self.saved)
            except OSError:
                pass
        return False


def cpu_record(value, unit, sample, cores=1, **extra) -> dict:
    """A cpu_baseline object: the oracle's rate on ``cores`` threads, with the host it ran on."""
    return {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample, **host_info(),
            **extra}


def source_digest() -> str:
    """sha256 over the kernel sources, in order: a recorded ncu traffic figure
    is used only while the kernels are the ones it was taken on."""
    h = hashlib.sha256()
    for path in KERNEL_SOURCES:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


E2E_CHUNK_ROWS = 4096  # rows per chunk of the host pipeline in the end-to-end measurement


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


def workload_config(wl, beta, l2_note, world, variant="row"):
    rw = {"uniform": "U(0,1) per row", "ones": "1.0 per row",
          "topk_softmax": f"top-{wl.topk} softmax weights of N(0,1) logits over {wl.experts} experts"}[wl.rw_kind]
    if variant == "col":
        rw = "U(0,1) per column ([I], shared by every row)"
    elif variant == "full":
        rw = "U(0,1) per element ([T, I])"
    return {
        "variant": {"row": "per-row routing weights, bf16/fp32 outputs",
                    "col": "per-column routing weights [I]", "full": "per-element routing weights [T, I]",
                    "mxfp8": "per-row routing weights, MXFP8 Y and d_gate_up (E4M3 + E8M0 per 32, OCP rule)",
                    "nvfp4": "per-row routing weights, NVFP4 Y and d_gate_up (E2M1 + E4M3 per 16, each tensor "
                             "scale from its call's own amax pass)"}[variant],
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
        self.power_limit_w = None
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
            try:
                self.power_limit_w = pynvml.nvmlDeviceGetEnforcedPowerLimit(self.handle) / 1000.0
            except Exception:
                self.power_limit_w = None
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
                "power_w_max": round(max(s[2] for s in self.samples), 1), "power_limit_w": self.power_limit_w,
                "source": "nvml"}


# The fused FC1 workload: the routed-MoE token rows (32768 rows, I = 2048) fed
# by a hidden size of 7168, grouped over 8 local experts with an uneven split.
FC1_HIDDEN = 7168
FC1_EXPERTS = 8
FC1_METRIC = "fused FC1 grouped GEMM + SiTU-GLU forward TFLOP/s"


def fc1_workload(wl):
    """Inputs of the fused FC1 bench: (x, w1, offsets, routing weights) on the
    host, from the routed-MoE rows' sizes and seed."""
    d = workloads.fc1_inputs(wl.tokens, FC1_HIDDEN, wl.inter, FC1_EXPERTS, wl.seed)
    d["offsets"] = workloads.expert_offsets(wl.tokens, FC1_EXPERTS, wl.seed, skew=2.0)
    d["routing_weights"] = workloads.routing_weights(wl)
    return d


def fc1_flops(wl) -> float:
    return 2.0 * wl.tokens * FC1_HIDDEN * 2 * wl.inter


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def fc1_cpu_rate(wl, beta, d, seconds: float):
    """The fp64 FC1 oracle on the first rows until ``seconds`` pass: TFLOP/s."""
    import oracle
    o = oracle.load()
    per_row = 2.0 * FC1_HIDDEN * 2 * wl.inter
    done, t0 = 0, time.perf_counter()
    while done < wl.tokens and time.perf_counter() - t0 < seconds:
        rows = np.arange(done, min(wl.tokens, done + 8), dtype=np.int64)
        o.fc1_fwd(d["x"], d["w1"], d["offsets"], wl.inter, d["routing_weights"], beta, wl.linear_beta, rows=rows)
        done += rows.size
    dt = time.perf_counter() - t0
    return per_row * done / dt / 1e12, done, dt


# The attention-residual mixing workload: 16384 tokens, 8 stored block sums
# plus the current sum (Kimi-K3 stores at most 8 sums), hidden 7168, bf16.
AR_TOKENS, AR_BLOCKS, AR_HIDDEN = 16384, 8, 7168
AR_METRIC = "attention-residual mixing core achieved HBM GB/s"


def ar_bytes() -> int:
    return AR_TOKENS * (AR_BLOCKS + 1) * AR_HIDDEN * 2 + AR_TOKENS * AR_HIDDEN * 2


def ar_config(l2_note, world):
    return {"workload": (f"attention-residual mix: {AR_BLOCKS} stored sums bf16 [{AR_TOKENS}, {AR_BLOCKS}, "
                         f"{AR_HIDDEN}] (source b ~ N(0, 1 + b/2)) + the current sum [{AR_TOKENS}, {AR_HIDDEN}], "
                         f"norm/proj weights fp32 [{AR_HIDDEN}], eps 1e-6, out bf16"),
            "name": "attn_res", "tokens": AR_TOKENS, "sources": AR_BLOCKS + 1, "hidden": AR_HIDDEN,
            "l2": l2_note, "parallelism": f"replicas x{world} (weak scaling; no collective)"}


def run_reference_attn_res(args, world):
    import oracle
    o = oracle.load()
    rows_per_step = 16
    d = workloads.attn_res_inputs(rows_per_step, AR_BLOCKS, AR_HIDDEN, seed=2)

    def step():
        o.attn_res(d["blocks"], d["prefix"], d["norm_weight"], d["proj_weight"], 1e-6)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = ar_bytes() / AR_TOKENS * rows_per_step * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": AR_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": ar_config("n/a (host)", 1),
            "cpu_baseline": cpu_record(value, "GB/s", f"{rows_per_step} rows per step, {args.steps} steps, "
                                                      f"single-threaded fp64"),
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_ours_attn_res(args, dev, world, rank, local, barrier):
    import torch
    import torch.distributed as dist

    import ffn_gated_activation_b200 as pkg

    d = workloads.attn_res_inputs(AR_TOKENS, AR_BLOCKS, AR_HIDDEN, seed=2)

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.pin_memory()

    blocks_h, prefix_h = pinned(d["blocks"]), pinned(d["prefix"])
    blocks, prefix = blocks_h.to(dev), prefix_h.to(dev)
    nw, pw = torch.from_numpy(d["norm_weight"]).to(dev), torch.from_numpy(d["proj_weight"]).to(dev)
    out = torch.empty(AR_TOKENS, AR_HIDDEN, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        pkg.apply_attn_res(prefix, blocks, pw, nw, 1e-6, out=out)

    for _ in range(max(3, args.warmup)):
        fwd()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for a, b in ev:
        a.record(stream)
        fwd()
        b.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    t = torch.tensor([sum(a.elapsed_time(b) for a, b in ev)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = t.item() / K
    gbs = ar_bytes() / (ms / 1e3) / 1e9
    peak, peak_src = measured_peak()

    # The same chain in plain PyTorch ops (eager, fp32), for context.
    def torch_chain():
        x = torch.cat([blocks, prefix.unsqueeze(1)], dim=1).float()
        k = torch.nn.functional.rms_norm(x, (AR_HIDDEN,), weight=nw, eps=1e-6)
        prob = torch.softmax(k @ pw, dim=-1)
        return (prob.unsqueeze(-1) * x).sum(dim=1).to(torch.bfloat16)

    for _ in range(2):
        torch_chain()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        torch_chain()
    b.record(stream)
    torch.cuda.synchronize()
    torch_ms = a.elapsed_time(b) / 3

    e2e = None
    if not args.no_e2e:
        out_h = torch.empty(AR_TOKENS, AR_HIDDEN, dtype=torch.bfloat16).pin_memory()
        K2 = args.e2e_steps or max(1, min(K, 10))

        def e2e_step():
            blocks.copy_(blocks_h, non_blocking=True)
            prefix.copy_(prefix_h, non_blocking=True)
            fwd()
            out_h.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K2):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        tt = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = tt.item() / K2
        e2e = {"value": ar_bytes() * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": blocks_h.numel() * 2 + prefix_h.numel() * 2,
               "d2h_bytes_per_step": out_h.numel() * 2, "ms_per_step": e2e_ms, "steps": K2,
               "api": "ffn_gated_activation_b200.apply_attn_res on pinned host copies"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        o = oracle.load()
        done, t0 = 0, time.perf_counter()
        per_row = ar_bytes() / AR_TOKENS
        while time.perf_counter() - t0 < args.cpu_seconds and done < AR_TOKENS:
            rows = np.arange(done, min(AR_TOKENS, done + 8), dtype=np.int64)
            o.attn_res(d["blocks"], d["prefix"], d["norm_weight"], d["proj_weight"], 1e-6, rows=rows)
            done += rows.size
        secs = time.perf_counter() - t0
        cpu = cpu_record(per_row * done / secs / 1e9, "GB/s",
                         f"first {done} of {AR_TOKENS} rows, {secs:.1f} s, single-threaded fp64 oracle")
    copy = copy_bandwidth(torch, dev, stream)
    if rank == 0:
        line = {"metric": AR_METRIC, "value": gbs * world, "unit": "GB/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": ar_config(f"inputs {ar_bytes() / 1e9:.1f} GB exceed the 126 MB L2; no flush", world),
                "kernels": {"situ_attn_res_staged_kernel": {"us": ms * 1e3, "GB/s": gbs,
                                                            "frac_of_measured_copy": gbs / peak,
                                                            "frac_of_copy_same_run": gbs / copy["GB/s"]}},
                "torch_eager_fp32_chain": {"ms": torch_ms, "GB/s": ar_bytes() / (torch_ms / 1e3) / 1e9},
                "roofline": {"bound": "hbm", "kernel": "situ_attn_res_staged_kernel", "achieved": gbs, "peak": peak,
                             "unit": "GB/s", "frac": gbs / peak, "peak_source": f"{peak_src} copy bandwidth",
                             "traffic": recorded_traffic("situ_attn_res_staged_kernel", "attn_res"),
                             "copy_same_run_gbs": copy["GB/s"], "frac_of_copy_same_run": gbs / copy["GB/s"]},
                "copy_same_run": copy, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": K, "clocks": clocks.summary(),
                "device_status": pkg.abi.situ_glu_device_status(0), "device": torch.cuda.get_device_name(dev)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def variant_bytes(wl, variant: str):
    """Algorithmic bytes (forward, backward) of one pass over the workload in
    the given form.  Per-row weights: read gate_up and w, write Y; read
    gate_up, grad_out and w, write d_gate_up and d_w.  Per-column weights move
    I weights and I gradients per pass; per-element weights T I of each.
    MXFP8 writes one byte per code and one scale byte per 32 codes; NVFP4
    half a byte per code and one scale byte per 16 (the tensor maximum's extra
    read of gate_up is not algorithmic: it counts against the kernels)."""
    T, I = wl.tokens, wl.inter
    es = 2 if wl.dtype == "bf16" else 4
    if variant == "col":
        return T * 3 * I * es + 4 * I, T * 5 * I * es + 8 * I
    if variant == "full":
        return T * (3 * I * es + 4 * I), T * (5 * I * es + 8 * I)
    if variant == "mxfp8":
        return T * (2 * I * es + I + I // 32 + 4), T * (3 * I * es + 2 * I + 2 * I // 32 + 8)
    if variant == "nvfp4":
        return T * (2 * I * es + I // 2 + I // 16 + 4), T * (3 * I * es + I + 2 * I // 16 + 8)
    return wl.fwd_bytes(), wl.bwd_bytes()


def variant_weights(wl, x, variant: str):
    """Host routing weights of the form (float32) and the oracle's mode."""
    import oracle
    if variant == "col":
        return workloads.column_weights(wl), oracle.RW_COL
    if variant == "full":
        return workloads.element_weights(wl), oracle.RW_FULL
    return x["routing_weights"], oracle.RW_ROW


def cpu_oracle_rate(wl, beta, x, seconds: float, variant: str = "row"):
    """The fp64 oracle (single thread, as it stands) on the first rows of the
    workload, fwd then bwd per chunk of rows (MXFP8: plus the oracle's block
    quantisation of Y and d_gate_up), until ``seconds`` have passed.
    Returns (GB/s of algorithmic bytes, rows done, elapsed, the core it was
    pinned to or None)."""
    import oracle
    o = oracle.load()
    fb, bb = variant_bytes(wl, variant)
    per_row = (fb + bb) / wl.tokens
    w, mode = variant_weights(wl, x, variant)
    chunk = max(1, min(64, int(2 ** 20 // wl.inter)))
    with PinnedCore() as pin:
        rate, done, dt = _oracle_loop(o, wl, beta, x, w, mode, chunk, seconds, variant, per_row)
    return rate, done, dt, pin.core


def _oracle_loop(o, wl, beta, x, w, mode, chunk, seconds, variant, per_row):
    import oracle
    done, t0 = 0, time.perf_counter()
    while done < wl.tokens:
        stop = min(wl.tokens, done + chunk)
        rows = np.arange(done, stop, dtype=np.int64)
        if mode == oracle.RW_FULL:  # the oracle reads [T, I] weights from row 0: pass the chunk's own rows
            gu, go, wr, rsel = x["gate_up"][done:stop], x["grad_out"][done:stop], w[done:stop], None
        else:
            gu, go, wr, rsel = x["gate_up"], x["grad_out"], w, rows
        y = o.fwd(gu, wr, beta, wl.linear_beta, rows=rsel, rw_mode=mode)
        r = o.bwd(gu, wr, go, beta, wl.linear_beta, rows=rsel, rw_mode=mode)
        if variant == "mxfp8":
            o.mxfp8_quantize(y)
            o.mxfp8_quantize(np.concatenate([r.dg, r.du], axis=1))
        elif variant == "nvfp4":
            o.nvfp4_quantize(y)
            o.nvfp4_quantize(np.concatenate([r.dg, r.du], axis=1))
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
    if args.tokens:
        wl = dataclasses.replace(wl, tokens=args.tokens)
    beta = args.beta if args.beta is not None else wl.betas[0]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.variant == "fc1":
        return run_reference_fc1(args, wl, beta, world)
    if args.variant == "fc2":
        return run_reference_fc2(args, wl, beta, world)
    if args.variant == "attn_res":
        return run_reference_attn_res(args, world)
    rows_per_step = max(1, min(wl.tokens, (1 << 17) // wl.inter))
    x = workloads.inputs(wl, tokens=rows_per_step)
    import oracle
    o = oracle.load()
    fb, bb = variant_bytes(wl, args.variant)
    per_row = (fb + bb) / wl.tokens
    w, mode = variant_weights(wl, x, args.variant)
    if mode == oracle.RW_FULL:
        w = w[:rows_per_step]

    def step():
        y = o.fwd(x["gate_up"], w, beta, wl.linear_beta, rw_mode=mode)
        r = o.bwd(x["gate_up"], w, x["grad_out"], beta, wl.linear_beta, rw_mode=mode)
        if args.variant == "mxfp8":
            o.mxfp8_quantize(y)
            o.mxfp8_quantize(np.concatenate([r.dg, r.du], axis=1))
        elif args.variant == "nvfp4":
            o.nvfp4_quantize(y)
            o.nvfp4_quantize(np.concatenate([r.dg, r.du], axis=1))

    with PinnedCore() as pin:
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
        "data": "synthetic", "config": workload_config(wl, beta, "n/a (host)", 1, args.variant),
        "rows_per_s": rows_per_step * args.steps / dt,
        "cpu_baseline": cpu_record(value, "GB/s", sample, pinned_core=pin.core),
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_fc1(args, wl, beta, world):
    d = fc1_workload(wl)
    import oracle
    o = oracle.load()
    rows_per_step = 4
    per_row = 2.0 * FC1_HIDDEN * 2 * wl.inter
    rows = np.arange(rows_per_step, dtype=np.int64)

    def step():
        o.fc1_fwd(d["x"], d["w1"], d["offsets"], wl.inter, d["routing_weights"], beta, wl.linear_beta, rows=rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_row * rows_per_step * args.steps / dt / 1e12
    sample = (f"{rows_per_step} of {wl.tokens} rows per step, {args.steps} steps, single-threaded fp64 FC1 oracle "
              f"(hidden {FC1_HIDDEN}, {FC1_EXPERTS} experts)")
    line = {
        "impl": "reference", "metric": FC1_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": fc1_config(wl, beta, "n/a (host)", 1),
        "cpu_baseline": cpu_record(value, "TFLOP/s", sample),
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def fc1_config(wl, beta, l2_note, world):
    return {
        "workload": (f"fused FC1: x bf16 [{wl.tokens}, {FC1_HIDDEN}] ~ N(0,1), w1 bf16 [{FC1_EXPERTS} x {2 * wl.inter},"
                     f" {FC1_HIDDEN}] ~ N(0, 3/sqrt({FC1_HIDDEN})), {FC1_EXPERTS} experts (Dirichlet(2) split), "
                     f"Y bf16 [{wl.tokens}, {wl.inter}]"),
        "name": f"{wl.name}/fc1",
        "tokens": wl.tokens, "hidden": FC1_HIDDEN, "inter": wl.inter, "experts": FC1_EXPERTS,
        "beta": beta, "linear_beta": wl.linear_beta,
        "routing_weights": f"top-{wl.topk} softmax weights per row",
        "l2": l2_note,
        "parallelism": f"replicas x{world} (weak scaling; no collective)",
    }


FC2_METRIC = "fused FC2 data-gradient GEMM + SiTU-GLU backward TFLOP/s"


def fc2_flops(wl) -> float:
    return 2.0 * wl.tokens * FC1_HIDDEN * wl.inter


def run_reference_fc2(args, wl, beta, world):
    d = workloads.fc2_inputs(wl.tokens, FC1_HIDDEN, wl.inter, FC1_EXPERTS, wl.seed)
    import oracle
    o = oracle.load()
    rows = np.arange(4, dtype=np.int64)

    def step():
        o.fc2_dgrad(d["dout"], d["w2t"], d["offsets"], d["gate_up"], d["routing_weights"], beta, wl.linear_beta,
                    rows=rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = 2.0 * FC1_HIDDEN * wl.inter * rows.size * args.steps / dt / 1e12
    cfg = fc1_config(wl, beta, "n/a (host)", 1)
    cfg["name"] = f"{wl.name}/fc2"
    line = {"impl": "reference", "metric": FC2_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": cpu_record(value, "TFLOP/s", f"{rows.size} rows per step, {args.steps} steps, "
                                                         f"single-threaded fp64"),
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_ours_fc2(args, wl, beta, dev, world, rank, local, barrier):
    import torch
    import torch.distributed as dist

    import ffn_gated_activation_b200 as pkg

    lb = wl.linear_beta
    T, I, H, E = wl.tokens, wl.inter, FC1_HIDDEN, FC1_EXPERTS
    d = workloads.fc2_inputs(T, H, I, E, wl.seed)
    d["offsets"] = workloads.expert_offsets(T, E, wl.seed, skew=2.0)

    def up(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    dout, w2t, gu = up(d["dout"]), up(d["w2t"]), up(d["gate_up"])
    off = torch.from_numpy(d["offsets"]).to(dev)
    rw = up(d["routing_weights"]).reshape(T, 1)
    dgu = torch.empty(T, 2 * I, dtype=torch.bfloat16, device=dev)
    d_rw = torch.empty(T, 1, dtype=torch.float32, device=dev)
    ws = torch.empty(max(1, pkg.abi.situ_glu_fc2_dgrad_workspace_bytes(T, I, 1)), dtype=torch.uint8, device=dev)
    flops = fc2_flops(wl)
    stream = torch.cuda.current_stream(dev)

    def bwd():
        pkg.situ_glu_fc2_dgrad_bwd(dout, w2t, off, gu, rw, beta, lb, d_gate_up=dgu, d_rw=d_rw, workspace=ws)

    for _ in range(max(3, args.warmup)):
        bwd()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for a, b in ev:
        a.record(stream)
        bwd()
        b.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    t = torch.tensor([sum(a.elapsed_time(b) for a, b in ev)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = t.item() / K
    tflops = flops / (ms / 1e3) / 1e12
    peak, peak_src = measured_tensor_peak()

    # unfused: cuBLAS dY = dOut W2_e per expert, then situ_glu_bwd
    offs = d["offsets"]
    dy = torch.empty(T, I, dtype=torch.bfloat16, device=dev)
    w2e = w2t.view(E, I, H)

    def unfused():
        for e in range(E):
            a0, a1 = int(offs[e]), int(offs[e + 1])
            if a1 > a0:
                torch.matmul(dout[a0:a1], w2e[e].t(), out=dy[a0:a1])
        pkg.situ_glu_bwd(gu, rw, dy, beta, lb, d_gate_up=dgu, d_rw=d_rw)

    for _ in range(3):
        unfused()
    torch.cuda.synchronize()
    ue = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(max(3, K // 2))]
    for a, b in ue:
        a.record(stream)
        unfused()
        b.record(stream)
    torch.cuda.synchronize()
    unfused_ms = statistics.median([a.elapsed_time(b) for a, b in ue])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        o = oracle.load()
        done, t0 = 0, time.perf_counter()
        while done < T and time.perf_counter() - t0 < args.cpu_seconds:
            rows = np.arange(done, min(T, done + 8), dtype=np.int64)
            o.fc2_dgrad(d["dout"], d["w2t"], d["offsets"], d["gate_up"], d["routing_weights"], beta, lb, rows=rows)
            done += rows.size
        secs = time.perf_counter() - t0
        cpu = cpu_record(2.0 * H * I * done / secs / 1e12, "TFLOP/s",
                         f"first {done} of {T} rows, {secs:.1f} s, single-threaded fp64 FC2-dgrad oracle")
    if rank == 0:
        cfg = fc1_config(wl, beta, "inputs 1.1 GB exceed the 126 MB L2; no flush", world)
        cfg["name"] = f"{wl.name}/fc2"
        cfg["workload"] = (f"fused FC2 data gradient: dOut bf16 [{T}, {H}] ~ N(0,1), W2 transposed bf16 "
                           f"[{E} x {I}, {H}] ~ N(0, 1/sqrt({H})), saved gate_up bf16 [{T}, {2 * I}] ~ N(0,3), "
                           f"{E} experts (Dirichlet(2) split), d_gate_up bf16, d_w fp32")
        line = {"metric": FC2_METRIC, "value": tflops * world, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
                "kernels": {"fc1::situ_fused_gemm_2sm_kernel<Fc2Epilogue>": {"us": ms * 1e3, "TFLOP/s": tflops,
                                                                         "frac_of_measured_bf16": tflops / peak}},
                "unfused": {"ms": unfused_ms, "TFLOP/s": flops / (unfused_ms / 1e3) / 1e12,
                            "what": "cuBLAS bf16 GEMM per expert (torch.matmul) into dY, then situ_glu_bwd"},
                "roofline": {"bound": "tensor", "kernel": "fc1::situ_fused_gemm_2sm_kernel<Fc2Epilogue>", "achieved": tflops,
                             "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                             "peak_source": f"{peak_src} cuBLAS bf16 (burst)",
                             "traffic": recorded_traffic("situ_fused_gemm_2sm_kernel<Fc2Epilogue>", f"{wl.name}/fc2")},
                "cpu_baseline": cpu, "e2e": None, "gpu_launches": 2 * K, "clocks": clocks.summary(),
                "device_status": pkg.abi.situ_glu_device_status(0), "device": torch.cuda.get_device_name(dev)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_ours_fc1(args, wl, beta, dev, world, rank, local, barrier):
    import torch
    import torch.distributed as dist

    import ffn_gated_activation_b200 as pkg

    lb = wl.linear_beta
    T, I = wl.tokens, wl.inter
    d = fc1_workload(wl)

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.pin_memory()

    x_h, w1_h = pinned(d["x"]), pinned(d["w1"])
    off_h = torch.from_numpy(d["offsets"]).pin_memory()
    rw_h = torch.from_numpy(d["routing_weights"]).reshape(T, 1).pin_memory()
    x, w1, off, rw = x_h.to(dev), w1_h.to(dev), off_h.to(dev), rw_h.to(dev)
    y = torch.empty(T, I, dtype=torch.bfloat16, device=dev)
    flops = fc1_flops(wl)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        pkg.situ_glu_fc1_fwd(x, w1, off, rw, beta, lb, out=y)

    for _ in range(max(3, args.warmup)):
        fwd()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for a, b in ev:
        a.record(stream)
        fwd()
        b.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    times = torch.tensor([sum(a.elapsed_time(b) for a, b in ev)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    ms = times.item() / K
    tflops = flops / (ms / 1e3) / 1e12
    peak, peak_src = measured_tensor_peak()

    # The unfused pipeline on the same data: one cuBLAS GEMM per expert into a
    # bf16 gate_up buffer, then the SiTU-GLU kernel over all rows.
    offs = d["offsets"]
    gu = torch.empty(T, 2 * I, dtype=torch.bfloat16, device=dev)
    w1e = w1.view(FC1_EXPERTS, 2 * I, FC1_HIDDEN)

    def unfused():
        for e in range(FC1_EXPERTS):
            a0, a1 = int(offs[e]), int(offs[e + 1])
            if a1 > a0:
                torch.matmul(x[a0:a1], w1e[e].t(), out=gu[a0:a1])
        pkg.situ_glu_fwd(gu, rw, beta, lb, out=y)

    for _ in range(3):
        unfused()
    torch.cuda.synchronize()
    ue = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(max(3, K // 2))]
    for a, b in ue:
        a.record(stream)
        unfused()
        b.record(stream)
    torch.cuda.synchronize()
    unfused_ms = statistics.median([a.elapsed_time(b) for a, b in ue])
    del gu

    e2e = None
    if not args.no_e2e:
        y_h = torch.empty(T, I, dtype=torch.bfloat16).pin_memory()
        K2 = args.e2e_steps or max(1, min(K, 10))

        def e2e_step():
            x.copy_(x_h, non_blocking=True)
            w1.copy_(w1_h, non_blocking=True)
            off.copy_(off_h, non_blocking=True)
            rw.copy_(rw_h, non_blocking=True)
            fwd()
            y_h.copy_(y, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
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
        h2d = sum(t_.numel() * t_.element_size() for t_ in (x_h, w1_h, off_h, rw_h))
        e2e = {"value": flops * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": y_h.numel() * 2, "ms_per_step": e2e_ms, "steps": K2,
               "api": "ffn_gated_activation_b200.situ_glu_fc1_fwd on pinned host copies"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows_done, secs = fc1_cpu_rate(wl, beta, d, args.cpu_seconds)
        cpu = cpu_record(rate, "TFLOP/s", f"first {rows_done} of {T} rows, {secs:.1f} s, single-threaded fp64 FC1 oracle")
    if rank == 0:
        line = {
            "metric": FC1_METRIC, "value": tflops * world, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": fc1_config(wl, beta, "inputs 940 MB exceed the 126 MB L2; no flush", world),
            "kernels": {"fc1::situ_fused_gemm_2sm_kernel<Fc1Epilogue>": {"us": ms * 1e3, "TFLOP/s": tflops,
                                                                     "frac_of_measured_bf16": tflops / peak}},
            "unfused": {"ms": unfused_ms, "TFLOP/s": flops / (unfused_ms / 1e3) / 1e12,
                        "what": "cuBLAS bf16 GEMM per expert (torch.matmul) into gate_up, then situ_glu_fwd"},
            "roofline": {"bound": "tensor", "kernel": "fc1::situ_fused_gemm_2sm_kernel<Fc1Epilogue>", "achieved": tflops,
                         "peak": peak,
                         "unit": "TFLOP/s", "frac": tflops / peak, "peak_source": f"{peak_src} cuBLAS bf16 (burst)",
                         "traffic": recorded_traffic("situ_fused_gemm_2sm_kernel<Fc1Epilogue>", f"{wl.name}/fc1")},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": K,
            "clocks": clocks.summary(),
            "device_status": pkg.abi.situ_glu_device_status(0),
            "device": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ---- our arm -----------------------------------------------------------------------

# The other workloads the 80 %-of-peak target names, each timed on its own
# after the headline workload: (workload index, gate beta).
SUB_CPU_SECONDS = 2.0  # oracle sample per sub-workload (one pinned core)
SUB_WORKLOADS = ((1, 4.0), (2, 4.0), (3, 1.0), (3, 4.0), (3, 16.0), (4, 4.0))


def step_stats(ms_list) -> dict:
    """Mean, median and minimum of per-launch times (microseconds)."""
    us = [v * 1e3 for v in ms_list]
    return {"us": sum(us) / len(us), "us_median": statistics.median(us), "us_min": min(us)}


def kernel_record(stats: dict, nbytes: int, rows: int, peak: float) -> dict:
    """Per-kernel figures: GB/s from the mean (the roofline's), the median and
    the fastest launch, each as a fraction of the measured copy and of 8 TB/s."""
    gbs = nbytes / stats["us"] / 1e3
    gbs_med = nbytes / stats["us_median"] / 1e3
    gbs_best = nbytes / stats["us_min"] / 1e3
    return {**stats, "bytes": nbytes, "GB/s": gbs, "GB/s_median": gbs_med, "GB/s_best": gbs_best,
            "pct_of_nominal_8TBs": gbs / NOMINAL_HBM_GBS * 100,
            "pct_of_nominal_8TBs_median": gbs_med / NOMINAL_HBM_GBS * 100,
            "frac_of_measured_copy": gbs / peak, "frac_of_measured_copy_median": gbs_med / peak,
            "rows_per_s": rows / (stats["us"] / 1e6)}


def row_kernels(wl):
    """The kernels the per-row forward and backward launch for this shape (the
    forward takes 32-byte vectors when a half row is a multiple of 64 vectors
    and at most 256 threads' worth, every pitch being 32-byte aligned here)."""
    vpr = wl.inter * wl.elem_bytes // 16
    fwd = "situ_glu_fwd_wide_kernel" if vpr % 64 == 0 and vpr // 2 <= 256 else "situ_glu_fwd_kernel"
    return fwd, "situ_glu_bwd_kernel"


def measure_workload(pkg, wl, beta, dev, K, warmup, local, allreduce_max, cpu_seconds=0.0):
    """One workload's forward and backward (per-row weights, native outputs),
    timed alone: K steps with CUDA events on the launching stream around each
    pass; with ``cpu_seconds`` > 0 also the fp64 oracle on one pinned core over
    the workload's first rows.  Returns the workload's record."""
    import torch
    x = workloads.inputs(wl)
    T, I = wl.tokens, wl.inter
    cpu = None
    if cpu_seconds > 0:
        rate, rows_done, secs, core = cpu_oracle_rate(wl, beta, x, cpu_seconds)
        cpu = cpu_record(rate, "GB/s", f"first {rows_done} of {T} rows, fwd + bwd, {secs:.1f} s, single-threaded "
                                       f"fp64", pinned_core=core)
    up = lambda a: (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
                    else torch.from_numpy(a)).to(dev)
    gu, go = up(x["gate_up"]), up(x["grad_out"])
    rw = torch.from_numpy(x["routing_weights"]).reshape(T, 1).to(dev)
    del x
    tdt = gu.dtype
    y = torch.empty(T, I, dtype=tdt, device=dev)
    d_gu = torch.empty(T, 2 * I, dtype=tdt, device=dev)
    d_rw = torch.empty(T, 1, dtype=torch.float32, device=dev)
    input_bytes = (gu.numel() + go.numel()) * gu.element_size() + T * 4
    flush_l2 = L2Flush(torch, dev) if input_bytes < 2 * L2_BYTES else None
    lb = wl.linear_beta
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, warmup)):
        if flush_l2 is not None:
            flush_l2()
        pkg.situ_glu_fwd(gu, rw, beta, lb, out=y)
        if flush_l2 is not None:
            flush_l2()
        pkg.situ_glu_bwd(gu, rw, go, beta, lb, d_gate_up=d_gu, d_rw=d_rw)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    for k in range(K):
        if flush_l2 is not None:
            flush_l2()
        ev[k][0].record(stream)
        pkg.situ_glu_fwd(gu, rw, beta, lb, out=y)
        ev[k][1].record(stream)
        if flush_l2 is not None:
            flush_l2()
        ev[k][2].record(stream)
        pkg.situ_glu_bwd(gu, rw, go, beta, lb, d_gate_up=d_gu, d_rw=d_rw)
        ev[k][3].record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    f = step_stats([e[0].elapsed_time(e[1]) for e in ev])
    b = step_stats([e[2].elapsed_time(e[3]) for e in ev])
    vals = allreduce_max([f["us"], f["us_median"], f["us_min"], b["us"], b["us_median"], b["us_min"]])
    f = dict(zip(("us", "us_median", "us_min"), vals[:3]))
    b = dict(zip(("us", "us_median", "us_min"), vals[3:]))
    peak, _ = measured_peak()
    fk, bk = row_kernels(wl)
    return {"workload": wl.describe(), "beta": beta, "steps": K,
            "l2": ("L2 left cold and clean before each kernel (a 2x-L2 buffer written, another read; not timed)"
                   if flush_l2 is not None
                   else f"inputs ({input_bytes / 1e6:.0f} MB) exceed the {L2_BYTES >> 20} MB L2; no flush"),
            "fwd": {"kernel": fk, **kernel_record(f, wl.fwd_bytes(), T, peak)},
            "bwd": {"kernel": bk, **kernel_record(b, wl.bwd_bytes(), T, peak)},
            "clocks": clocks.summary(), "cpu_baseline": cpu}


def cpu_oracle_rate_threads(wl, beta, x, seconds: float, threads: int):
    """The same oracle code as cpu_oracle_rate, with the rows split across
    ``threads`` threads (each takes the next chunk of rows; the C oracle
    releases the GIL), until ``seconds`` have passed.  Returns (GB/s, rows)."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    o = oracle.load()
    per_row = (wl.fwd_bytes() + wl.bwd_bytes()) / wl.tokens
    chunk = max(1, min(64, int(2 ** 20 // wl.inter)))
    nxt, lock, rows_done = [0], threading.Lock(), [0]
    t0 = time.perf_counter()

    def worker():
        while time.perf_counter() - t0 < seconds:
            with lock:
                r0 = nxt[0]
                if r0 >= wl.tokens:
                    return
                nxt[0] = min(wl.tokens, r0 + chunk)
            r1 = min(wl.tokens, r0 + chunk)
            rows = np.arange(r0, r1, dtype=np.int64)
            o.fwd(x["gate_up"], x["routing_weights"], beta, wl.linear_beta, rows=rows)
            o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], beta, wl.linear_beta, rows=rows)
            with lock:
                rows_done[0] += r1 - r0

    with ThreadPoolExecutor(max_workers=threads) as pool:
        for fut in [pool.submit(worker) for _ in range(threads)]:
            fut.result()
    dt = time.perf_counter() - t0
    return per_row * rows_done[0] / dt / 1e9, rows_done[0], dt


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

    def allreduce_max(vals):
        t = torch.tensor(list(vals), dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.tolist()

    wl = workloads.workload(args.config)
    if args.tokens:
        wl = dataclasses.replace(wl, tokens=args.tokens)
    beta = args.beta if args.beta is not None else wl.betas[0]
    if args.variant == "fc1":
        return run_ours_fc1(args, wl, beta, dev, world, rank, local, barrier)
    if args.variant == "fc2":
        return run_ours_fc2(args, wl, beta, dev, world, rank, local, barrier)
    if args.variant == "attn_res":
        return run_ours_attn_res(args, dev, world, rank, local, barrier)
    lb = wl.linear_beta
    T, I = wl.tokens, wl.inter
    x = workloads.inputs(wl)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32

    def upload(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.pin_memory()

    variant = args.variant
    gu_h, go_h = upload(x["gate_up"]), upload(x["grad_out"])
    w_np, _ = variant_weights(wl, x, variant)
    rw_h = torch.from_numpy(w_np).reshape({"col": (I,), "full": (T, I)}.get(variant, (T, 1))).pin_memory()
    gu = gu_h.to(dev)
    go = go_h.to(dev)
    rw = rw_h.to(dev)
    d_rw = torch.empty(rw.shape, dtype=torch.float32, device=dev)
    if variant == "mxfp8":
        y = torch.empty(T, I, dtype=torch.float8_e4m3fn, device=dev)
        y_sc = torch.empty(T, I // 32, dtype=torch.uint8, device=dev)
        d_gu = torch.empty(T, 2 * I, dtype=torch.float8_e4m3fn, device=dev)
        d_sc = torch.empty(T, 2 * I // 32, dtype=torch.uint8, device=dev)
        outputs = [y, y_sc, d_gu, d_sc, d_rw]
    elif variant == "nvfp4":
        y = torch.empty(T, I // 2, dtype=torch.uint8, device=dev)
        y_sc = torch.empty(T, I // 16, dtype=torch.float8_e4m3fn, device=dev)
        y_amax = torch.empty(1, dtype=torch.float32, device=dev)
        d_gu = torch.empty(T, I, dtype=torch.uint8, device=dev)
        d_sc = torch.empty(T, 2 * I // 16, dtype=torch.float8_e4m3fn, device=dev)
        d_amax = torch.empty(1, dtype=torch.float32, device=dev)
        outputs = [y, y_sc, y_amax, d_gu, d_sc, d_amax, d_rw]
    else:
        y = torch.empty(T, I, dtype=tdt, device=dev)
        d_gu = torch.empty(T, 2 * I, dtype=tdt, device=dev)
        outputs = [y, d_gu, d_rw]

    input_bytes = gu.numel() * gu.element_size() + go.numel() * go.element_size() + rw.numel() * 4
    flush = args.flush == "always" or (args.flush == "auto" and input_bytes < 2 * L2_BYTES)
    flush_l2 = L2Flush(torch, dev) if flush else None
    l2_note = (f"L2 left cold and clean before each kernel: {2 * L2_BYTES >> 20} MB written, another "
               f"{2 * L2_BYTES >> 20} MB read (not timed)" if flush
               else f"inputs ({input_bytes / 1e6:.0f} MB) exceed the {L2_BYTES >> 20} MB L2; no flush")

    if variant == "mxfp8":
        def fwd():
            pkg.situ_glu_fwd_mxfp8(gu, rw, beta, lb, rule="ocp", data=y, scale=y_sc)

        def bwd():
            pkg.situ_glu_bwd_mxfp8(gu, rw, go, beta, lb, rule="ocp", data=d_gu, scale=d_sc, d_rw=d_rw)
    elif variant == "nvfp4":
        def fwd():
            pkg.situ_glu_fwd_nvfp4(gu, rw, beta, lb, data=y, scale=y_sc, amax_out=y_amax)

        def bwd():
            pkg.situ_glu_bwd_nvfp4(gu, rw, go, beta, lb, data=d_gu, scale=d_sc, amax_out=d_amax, d_rw=d_rw)
    else:
        def fwd():
            pkg.situ_glu_fwd(gu, rw, beta, lb, out=y)

        def bwd():
            pkg.situ_glu_bwd(gu, rw, go, beta, lb, d_gate_up=d_gu, d_rw=d_rw)

    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        if flush:
            flush_l2()
        fwd()
        if flush:
            flush_l2()
        bwd()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    outer0, outer1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    outer0.record(stream)
    for k in range(K):
        if flush:
            flush_l2()
        ev[k][0].record(stream)
        fwd()
        ev[k][1].record(stream)
        if flush:
            flush_l2()
        ev[k][2].record(stream)
        bwd()
        ev[k][3].record(stream)
    outer1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(K)]
    bwd_ms = [ev[k][2].elapsed_time(ev[k][3]) for k in range(K)]
    total_ms = sum(fwd_ms) + sum(bwd_ms) if flush else outer0.elapsed_time(outer1)
    times = torch.tensor([total_ms, sum(fwd_ms), sum(bwd_ms)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    total_ms, fwd_sum, bwd_sum = times.tolist()
    quant_us = None
    if variant == "nvfp4":
        # the quantising kernels alone: the same calls with the tensor maxima given
        fgiven, bgiven = y_amax.clone(), d_amax.clone()
        qev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        torch.cuda.synchronize()
        for k in range(K):
            if flush:
                flush_l2()
            qev[k][0].record(stream)
            pkg.situ_glu_fwd_nvfp4(gu, rw, beta, lb, data=y, scale=y_sc, amax=fgiven)
            qev[k][1].record(stream)
            if flush:
                flush_l2()
            qev[k][2].record(stream)
            pkg.situ_glu_bwd_nvfp4(gu, rw, go, beta, lb, data=d_gu, scale=d_sc, amax=bgiven, d_rw=d_rw)
            qev[k][3].record(stream)
        torch.cuda.synchronize()
        qt = torch.tensor([sum(e[0].elapsed_time(e[1]) for e in qev), sum(e[2].elapsed_time(e[3]) for e in qev)],
                          dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(qt, op=dist.ReduceOp.MAX)
        quant_us = [v / K * 1e3 for v in qt.tolist()]
    ms_per_step = total_ms / K
    fwd_bytes, bwd_bytes = variant_bytes(wl, variant)
    step_bytes = fwd_bytes + bwd_bytes
    value = step_bytes * world / (ms_per_step / 1e3) / 1e9
    peak, peak_src = measured_peak()
    fwd_us, bwd_us = fwd_sum / K * 1e3, bwd_sum / K * 1e3
    fwd_gbs, bwd_gbs = fwd_bytes / fwd_us / 1e3, bwd_bytes / bwd_us / 1e3
    # median and fastest launch of each pass, max over ranks
    fs, bs = step_stats(fwd_ms), step_stats(bwd_ms)
    mm = allreduce_max([fs["us_median"], fs["us_min"], bs["us_median"], bs["us_min"]])
    fs = {"us": fwd_us, "us_median": mm[0], "us_min": mm[1]}
    bs = {"us": bwd_us, "us_median": mm[2], "us_min": mm[3]}
    # the kernels each pass launches for this form and shape
    fwd_kernel, bwd_kernel = {
        "row": row_kernels(wl),
        "col": ("situ_glu_fwd_ew_kernel", "situ_glu_bwd_ew_kernel"),
        "full": ("situ_glu_fwd_ew_kernel", "situ_glu_bwd_ew_kernel"),
        "mxfp8": ("situ_glu_fwd_quant_kernel<MxQuant>", "situ_glu_bwd_quant_kernel<MxQuant>"),
        "nvfp4": ("situ_glu_fwd_quant_kernel<AmaxOnly>+situ_glu_fwd_quant_kernel<Nvfp4Quant>",
                  "situ_glu_bwd_quant_kernel<AmaxOnly>+situ_glu_bwd_quant_kernel<Nvfp4Quant>"),
    }[variant]
    # per-column weights: plus the column finalize; NVFP4: an amax pass and a quantising pass each way
    launches_per_step = {"col": 3, "nvfp4": 4}.get(variant, 2)
    traffic_key = wl.name if variant == "row" else f"{wl.name}/{variant}"
    roof_kernel = "situ_glu_bwd_quant_kernel<Nvfp4Quant>" if variant == "nvfp4" else bwd_kernel
    traffic = recorded_traffic(roof_kernel, traffic_key)

    # End to end through the public API with host buffers: every step copies the
    # inputs from pinned host memory, runs both passes and reads all outputs back.
    e2e = None
    if not args.no_e2e:
        outputs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outputs]
        K2 = args.e2e_steps or max(1, min(K, 20))

        if variant == "row":
            # the public host-tensor API: row chunks streamed through the GPU,
            # uploads, kernels and downloads of successive chunks overlapped
            pipe = pkg.HostPipeline(I, tdt, chunk_rows=E2E_CHUNK_ROWS, device=dev)
            y_h, dgu_h, drw_h = outputs_h

            def e2e_step():
                pipe.run(gu_h, rw_h, go_h, beta, lb, y=y_h, d_gate_up=dgu_h, d_rw=drw_h)
        else:
            def e2e_step():
                gu.copy_(gu_h, non_blocking=True)
                go.copy_(go_h, non_blocking=True)
                rw.copy_(rw_h, non_blocking=True)
                fwd()
                bwd()
                for th, td in zip(outputs_h, outputs):
                    th.copy_(td, non_blocking=True)

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
        d2h = sum(t.numel() * t.element_size() for t in outputs_h)
        api = {"mxfp8": "situ_glu_fwd_mxfp8/situ_glu_bwd_mxfp8 on pinned host copies",
               "nvfp4": "situ_glu_fwd_nvfp4/situ_glu_bwd_nvfp4 on pinned host copies",
               "row": f"HostPipeline.run on pinned host tensors (chunks of {E2E_CHUNK_ROWS} rows; uploads, "
                      f"kernels and downloads of successive chunks overlapped on three streams)"}.get(
                   variant, "situ_glu_fwd/situ_glu_bwd on pinned host copies")
        e2e = {"value": step_bytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": K2,
               "api": f"ffn_gated_activation_b200.{api}"}
        if variant == "row":
            # the link the end-to-end step is bound by, measured with its own buffers
            link = link_bandwidth(torch, dev, gu_h, gu, d_gu, outputs_h[1])
            e2e["link_same_run"] = link
            e2e["h2d_GB/s"] = h2d / (e2e_ms / 1e3) / 1e9
            e2e["d2h_GB/s"] = d2h / (e2e_ms / 1e3) / 1e9
            # the time the link needs for the step's bytes at its both-ways rates, over the step's time
            link_ms = max(h2d / link["both_h2d_GB/s"], d2h / link["both_d2h_GB/s"]) / 1e6
            e2e["frac_of_link_both_ways"] = link_ms / e2e_ms

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows_done, secs, core = cpu_oracle_rate(wl, beta, x, args.cpu_seconds, variant)
        extra = {"pinned_core": core}
        if variant == "row":
            threads = host_info()["cores_available"] or 1
            prate, prows, psecs = cpu_oracle_rate_threads(wl, beta, x, args.cpu_seconds, threads)
            extra["all_cores"] = {"value": prate, "unit": "GB/s", "cores": threads,
                                  "sample": f"first {prows} of {T} rows, fwd + bwd, {psecs:.1f} s, the same fp64 "
                                            f"oracle code with the rows split across {threads} threads"}
        cpu = cpu_record(rate, "GB/s", f"first {rows_done} of {T} rows, fwd + bwd, {secs:.1f} s, "
                                       f"single-threaded fp64", **extra)
    del x

    # The other target workloads, each timed alone after the headline one.
    subs = None
    if variant == "row" and not args.no_sub and not args.tokens:
        del outputs, gu, go, rw, y, d_gu, d_rw, flush_l2
        torch.cuda.empty_cache()
        subs = {}
        for idx, b_ in SUB_WORKLOADS:
            if idx == args.config and b_ == beta:
                continue
            w_ = workloads.workload(idx)
            sub_cpu = SUB_CPU_SECONDS if rank == 0 and world == 1 and not args.no_cpu_baseline else 0.0
            subs[f"{w_.name} beta={b_:g}"] = measure_workload(pkg, w_, b_, dev, K, args.warmup, local, allreduce_max,
                                                              sub_cpu)
            torch.cuda.empty_cache()

    copy = copy_bandwidth(torch, dev, stream)
    kernels = {fwd_kernel: kernel_record(fs, fwd_bytes, T, peak), bwd_kernel: kernel_record(bs, bwd_bytes, T, peak)}
    roofline = {"bound": "hbm", "kernel": bwd_kernel, "achieved": bwd_gbs, "peak": peak,
                "unit": "GB/s", "frac": bwd_gbs / peak, "peak_source": f"{peak_src} copy bandwidth",
                "traffic": traffic}
    if quant_us is not None:
        es_ = 2 if wl.dtype == "bf16" else 4
        passes = [("fwd", fwd_us, fwd_bytes, quant_us[0], T * (2 * I * es_ + 4)),
                  ("bwd", bwd_us, bwd_bytes, quant_us[1], T * (3 * I * es_ + 4))]
        for d, call_us, q_bytes, q_us, a_bytes in passes:
            a_us = max(call_us - q_us, 1e-9)
            kernels[f"situ_glu_{d}_quant_kernel<AmaxOnly>"] = {
                "us": a_us, "bytes": a_bytes, "GB/s": a_bytes / a_us / 1e3,
                "frac_of_measured_copy": a_bytes / a_us / 1e3 / peak,
                "note": "the NVFP4 call's time less its quantising pass alone"}
            kernels[f"situ_glu_{d}_quant_kernel<Nvfp4Quant>"] = {
                "us": q_us, "bytes": q_bytes, "GB/s": q_bytes / q_us / 1e3,
                "frac_of_measured_copy": q_bytes / q_us / 1e3 / peak, "note": "timed alone, tensor maximum given"}
        q_gbs = bwd_bytes / quant_us[1] / 1e3
        roofline = {"bound": "hbm", "kernel": roof_kernel, "achieved": q_gbs, "peak": peak, "unit": "GB/s",
                    "frac": q_gbs / peak, "peak_source": f"{peak_src} copy bandwidth", "traffic": traffic}

    roofline["copy_same_run_gbs"] = copy["GB/s"]
    roofline["frac_of_copy_same_run"] = roofline["achieved"] / copy["GB/s"]
    add_copy_fractions(copy, *kernels.values())
    for sub in (subs or {}).values():
        add_copy_fractions(copy, sub.get("fwd"), sub.get("bwd"))
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(wl, beta, l2_note, world, variant),
            "rows_per_s": T * world / (ms_per_step / 1e3),
            "pct_of_nominal_hbm": value / world / NOMINAL_HBM_GBS * 100.0,
            "kernels": kernels,
            "roofline": roofline,
            "copy_same_run": copy,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * K,
            "clocks": clocks.summary(),
            "device_status": pkg.abi.situ_glu_device_status(0),
            "device": torch.cuda.get_device_name(dev),
        }
        if subs is not None:
            line["workloads"] = subs
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
