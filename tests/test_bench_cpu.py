"""CPU checks of the bench harness (bench.py): the algorithmic byte counts the
roofline divides by, the reference arm's JSON line for every variant, its
rank handling under torchrun, the single-core pinning of the CPU baseline
and the traffic record's source check.  Nothing here needs a GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


@pytest.mark.parametrize("index", [0, 1, 2, 3, 4])
def test_algorithmic_bytes(index):
    """Per row: forward 2I s + 4 + I s (read gate_up and w, write Y); backward
    2I s + I s + 4 + 2I s + 4 (read gate_up, go and w, write d_gate_up, d_w)."""
    wl = workloads.workload(index)
    s = 2 if wl.dtype == "bf16" else 4
    T, I = wl.tokens, wl.inter
    fwd, bwd = bench.variant_bytes(wl, "row")
    assert fwd == wl.fwd_bytes() == T * (2 * I * s + 4 + I * s)
    assert bwd == wl.bwd_bytes() == T * (2 * I * s + I * s + 4 + 2 * I * s + 4)


def test_form_bytes():
    """The other forms' bytes, from their layouts: per-column weights are read
    once and their gradient written once; per-element weights and gradients
    move 4I bytes a row each way; MXFP8 writes one byte per element plus a
    scale byte per 32; NVFP4 half a byte per element plus a scale byte per 16."""
    wl = workloads.workload(2)
    T, I = wl.tokens, wl.inter
    row_f, row_b = bench.variant_bytes(wl, "row")
    col_f, col_b = bench.variant_bytes(wl, "col")
    assert col_f == row_f - 4 * T + 4 * I and col_b == row_b - 8 * T + 8 * I
    full_f, full_b = bench.variant_bytes(wl, "full")
    assert full_f == row_f - 4 * T + 4 * T * I and full_b == row_b - 8 * T + 8 * T * I
    mx_f, mx_b = bench.variant_bytes(wl, "mxfp8")
    assert mx_f == T * (2 * I * 2 + 4 + I + I // 32)
    assert mx_b == T * (3 * I * 2 + 2 * I + 2 * I // 32 + 8)
    nv_f, nv_b = bench.variant_bytes(wl, "nvfp4")
    assert nv_f == T * (2 * I * 2 + 4 + I // 2 + I // 16)
    assert nv_b == T * (3 * I * 2 + 4 + I + 2 * I // 16 + 4)


def _reference_line(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    return lines


@pytest.mark.parametrize("variant", ["row", "col", "full", "mxfp8", "nvfp4", "fc1", "fc2", "attn_res"])
def test_reference_arm_line(variant):
    """One JSON line with the contract's keys; the CPU baseline describes the
    run (one pinned core where affinity can be set) and e2e repeats the value
    with no host-device bytes."""
    lines = _reference_line(["--config", "2", "--variant", variant, "--steps", "1", "--warmup", "0"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["gpu_launches"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["host_cores"] >= 1


def test_reference_arm_other_ranks_are_silent():
    """Under torchrun only rank 0 runs the CPU arm; the others exit 0 at once."""
    assert _reference_line(["--steps", "1", "--warmup", "0"], {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_pinned_core_restores_the_affinity():
    if not hasattr(os, "sched_getaffinity"):
        pytest.skip("no affinity control on this host")
    before = os.sched_getaffinity(0)
    with bench.PinnedCore() as pin:
        assert pin.core == min(before)
        assert os.sched_getaffinity(0) == {pin.core}
    assert os.sched_getaffinity(0) == before


def test_traffic_record_needs_the_current_source(tmp_path, monkeypatch):
    """A recorded DRAM figure is used only while the kernel source it was taken
    on is the current one."""
    rec = {"situ_glu_bwd_kernel": {"large": {"bytes_per_launch": 123.0, "source_sha256": bench.source_digest()}}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("situ_glu_bwd_kernel", "large") == 123.0
    assert bench.recorded_traffic("situ_glu_bwd_kernel", "routed_moe") is None
    rec["situ_glu_bwd_kernel"]["large"]["source_sha256"] = "0" * 64
    path.write_text(json.dumps(rec))
    assert bench.recorded_traffic("situ_glu_bwd_kernel", "large") is None
