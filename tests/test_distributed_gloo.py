"""The N > 1 plumbing on CPU: world-size-2 gloo process groups.

Each rank computes its share with the fp64 oracle (the CUDA kernels need a
GPU); the tests check the product's sharding and reduction helpers:

* tensor parallelism: column shards of gate_up / grad_out give local dG, dU
  equal to the matching columns of the unsharded backward, and the
  all-reduced per-rank routing-weight partials equal the full-width gradient;
* data parallelism with a broadcast weight: row shards' partial sums,
  all-reduced, equal the single-process gradient;
* max-over-ranks timing and the shard arithmetic;
* a rank that leaves: the other rank's next collective ends with an error.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ffn_gated_activation_b200 import distributed as D

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(fn, *args):
    port = _free_port()
    mp.spawn(_entry, args=(fn, port, args), nprocs=WORLD, join=True)


def _entry(rank, fn, port, args):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for p in (root, os.path.join(root, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        fn(rank, *args)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _bf16_tensor(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _tp_check(rank, T, I, seed):
    import oracle
    import workloads
    import dataclasses
    wl = dataclasses.replace(workloads.workload(2), tokens=T, inter=I, seed=seed, rw_kind="uniform")
    x = workloads.inputs(wl)
    o = oracle.load()
    full = o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], 4.0, 25.0)
    gu_local = _bits(D.tp_local_gate_up(_bf16_tensor(x["gate_up"]), rank, WORLD))
    go_local = _bits(D.tp_local_columns(_bf16_tensor(x["grad_out"]), rank, WORLD))
    a, b = D.shard_range(I, rank, WORLD, align=8)
    assert gu_local.shape == (T, 2 * (b - a))
    loc = o.bwd(gu_local, x["routing_weights"], go_local, 4.0, 25.0)
    # dG and dU need no exchange: they are the matching columns of the full result
    assert np.array_equal(loc.dg, full.dg[:, a:b]) and np.array_equal(loc.du, full.du[:, a:b])
    # the routing-weight gradient is the sum of the ranks' column partials
    d_rw = torch.tensor(loc.dw, dtype=torch.float64)
    D.allreduce_drw(d_rw)
    np.testing.assert_allclose(d_rw.numpy(), full.dw, rtol=1e-12, atol=1e-12 * full.sw.max())


def _dp_scalar_check(rank, T, I, seed):
    import oracle
    import workloads
    import dataclasses
    wl = dataclasses.replace(workloads.workload(0), tokens=T, inter=I, seed=seed)
    x = workloads.inputs(wl)
    o = oracle.load()
    total, mag = o.dw_scalar(x["gate_up"], x["grad_out"], 4.0, 25.0)
    r0, r1 = D.shard_range(T, rank, WORLD)
    part, _ = o.dw_scalar(x["gate_up"][r0:r1], x["grad_out"][r0:r1], 4.0, 25.0)
    t = torch.tensor([part], dtype=torch.float64)
    D.allreduce_drw(t)
    assert abs(t.item() - total) <= 1e-12 * mag


def _col_weight_check(rank, T, I, seed):
    """Per-column weights: row shards all-reduce their [I] partials; column
    shards own their slice of the gradient outright."""
    import oracle
    import workloads
    import dataclasses
    wl = dataclasses.replace(workloads.workload(0), tokens=T, inter=I, seed=seed)
    x = workloads.inputs(wl)
    o = oracle.load()
    full, mag = o.dw_columns(x["gate_up"], x["grad_out"], 4.0, 25.0)
    r0, r1 = D.shard_range(T, rank, WORLD)
    part, _ = o.dw_columns(x["gate_up"][r0:r1], x["grad_out"][r0:r1], 4.0, 25.0)
    t = torch.tensor(part, dtype=torch.float64)
    D.allreduce_drw(t)
    assert np.all(np.abs(t.numpy() - full) <= 1e-12 * mag)
    # tensor parallel: the rank's columns of gate_up / grad_out give its columns of d_w exactly
    gu_local = _bits(D.tp_local_gate_up(_bf16_tensor(x["gate_up"]), rank, WORLD))
    go_local = _bits(D.tp_local_columns(_bf16_tensor(x["grad_out"]), rank, WORLD))
    a, b = D.shard_range(I, rank, WORLD, align=8)
    loc, _ = o.dw_columns(gu_local, go_local, 4.0, 25.0)
    assert np.array_equal(loc, full[a:b])
    rw_local = torch.ones(b - a)
    assert not D.tp_drw_needs_allreduce((T,), b - a, rw_local)
    assert D.tp_drw_needs_allreduce((T,), b - a, torch.ones(T, 1))


def _tp_nvfp4_check(rank, T, I, seed):
    """Column shards of an NVFP4 Y and d_gate_up (whole 16-element blocks per
    rank): the all-reduced maximum of the shards' maxima is the whole
    tensor's, and each shard's codes and block scales under it are the
    matching columns of the whole tensor's coding."""
    import oracle
    import workloads
    import dataclasses
    wl = dataclasses.replace(workloads.workload(2), tokens=T, inter=I, seed=seed, rw_kind="uniform")
    x = workloads.inputs(wl)
    o = oracle.load()
    rw = x["routing_weights"]
    gu_local = _bits(D.tp_local_gate_up(_bf16_tensor(x["gate_up"]), rank, WORLD, align=16))
    go_local = _bits(D.tp_local_columns(_bf16_tensor(x["grad_out"]), rank, WORLD, align=16))
    a, b = D.shard_range(I, rank, WORLD, align=16)
    assert a % 16 == 0 and b % 16 == 0 and b > a
    y_full = o.fwd(x["gate_up"], rw, 4.0, 25.0)
    full = o.bwd(x["gate_up"], rw, x["grad_out"], 4.0, 25.0)
    d_full = np.concatenate([full.dg, full.du], axis=1)
    y_loc = o.fwd(gu_local, rw, 4.0, 25.0)
    loc = o.bwd(gu_local, rw, go_local, 4.0, 25.0)
    d_loc = np.concatenate([loc.dg, loc.du], axis=1)
    for whole, part, cols in ((y_full, y_loc, [(a, b)]), (d_full, d_loc, [(a, b), (I + a, I + b)])):
        amax = torch.tensor([np.abs(part).max()], dtype=torch.float64)
        D.allreduce_amax(amax)
        assert amax.item() == np.abs(whole).max()
        codes_w, scales_w, s_enc = o.nvfp4_quantize(whole)
        codes_p, scales_p, s_p = o.nvfp4_quantize(part, s_enc=o.nvfp4_tensor_scale(amax.item()))
        assert s_p == s_enc
        want_c = np.concatenate([codes_w[:, c0:c1] for c0, c1 in cols], axis=1)
        want_s = np.concatenate([scales_w[:, c0 // 16:c1 // 16] for c0, c1 in cols], axis=1)
        assert np.array_equal(codes_p, want_c) and np.array_equal(scales_p, want_s)
        # a shard coded with its own maximum instead would differ from the whole tensor's coding
        if amax.item() != np.abs(part).max():
            assert not np.array_equal(o.nvfp4_quantize(part)[1], want_s)


def _max_check(rank):
    assert D.max_over_ranks(1.5 + rank) == 2.5


def test_tensor_parallel_backward_gloo():
    _run(_tp_check, 37, 520, 11)


def test_tensor_parallel_nvfp4_scale_gloo():
    _run(_tp_nvfp4_check, 29, 512, 12)


def test_data_parallel_broadcast_weight_gloo():
    _run(_dp_scalar_check, 61, 64, 12)


def test_column_weight_gradient_gloo():
    _run(_col_weight_check, 45, 136, 13)


def test_tp_drw_reduction_by_weight_shape():
    lead, i_local = (6, 5), 24
    assert D.tp_drw_needs_allreduce(lead, i_local, torch.ones(6, 5, 1))
    assert D.tp_drw_needs_allreduce(lead, i_local, torch.tensor(2.0))
    assert not D.tp_drw_needs_allreduce(lead, i_local, torch.ones(i_local))
    assert not D.tp_drw_needs_allreduce(lead, i_local, torch.ones(6, 5, i_local))


def test_max_over_ranks_gloo():
    _run(_max_check)


@pytest.mark.parametrize("n,world,align", [(10, 3, 1), (520, 2, 8), (7, 4, 1), (4096, 8, 8), (3, 5, 1), (0, 2, 8)])
def test_shard_range_partitions(n, world, align):
    spans = [D.shard_range(n, r, world, align) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a0, b0), (a1, b1) in zip(spans, spans[1:]):
        assert b0 == a1
    for a, b in spans:
        assert a <= b and a % align == 0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= align


def _leave_entry(rank, port, result_path, how):
    """Rank 1 leaves between steps, before its weight-gradient all-reduce
    (`exit`: its process ends; `stall`: it stays alive but never joins);
    rank 0 enters that all-reduce and records how it ended."""
    import datetime
    import json
    import time
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=3))
    if rank == 1:
        if how == "stall":
            time.sleep(10)
        os._exit(0)  # gone, with no collective in flight and no teardown
    t0 = time.monotonic()
    try:
        D.allreduce_drw(torch.ones(4, dtype=torch.float64))
        outcome = "completed"
    except Exception as e:  # gloo reports the lost peer or the timeout
        outcome = f"error: {type(e).__name__}: {str(e)[:200]}"
    with open(result_path, "w") as f:
        json.dump({"outcome": outcome, "seconds": time.monotonic() - t0}, f)
    os._exit(0)  # the group has lost a member: skip its teardown


@pytest.mark.parametrize("how", ["exit", "stall"])
def test_a_rank_that_leaves_ends_the_others_collective_with_an_error(how, tmp_path):
    """Failure detection on the host: with a short process-group timeout (3 s),
    the surviving rank's next collective (the routing-weight gradient's
    all-reduce) raises instead of waiting for the rank that left, whether
    that rank's process ended or it stopped taking part."""
    import json
    result = tmp_path / "rank0.json"
    mp.spawn(_leave_entry, args=(_free_port(), str(result), how), nprocs=WORLD, join=True)
    rec = json.loads(result.read_text())
    assert rec["outcome"].startswith("error"), rec
    assert rec["seconds"] < 9, rec  # before the stalled rank would have gone


def test_max_over_ranks_without_group():
    assert D.max_over_ranks(3.25) == 3.25
