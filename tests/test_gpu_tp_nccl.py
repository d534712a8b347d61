"""The tensor-parallel wrappers on the GPU, inside a real NCCL process group.

The column-parallel plan (spark_model kimi_k3 `tp.rs`, the FC1 column shards)
runs a kernel, an NCCL all-reduce of its result and, for NVFP4, a second
kernel that consumes the reduced value, all on the caller's stream.  A CUDA
run here has one GPU, so the group has one rank: its shard is the whole
tensor, and every result must match the fp64 oracle's whole-tensor results.
What this adds to the gloo tests (which check the sharding and the
reductions with the oracle standing in for the kernels) is the real sequence
kernel -> NCCL all-reduce -> kernel, issued on a side stream.
"""
import dataclasses
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import workloads
from ffn_gated_activation_b200 import distributed as tp

from parity import CANCEL, check_dw, check_nvfp4, check_output, to_device, to_host

pytestmark = pytest.mark.gpu

REL_BF16 = 2.0 ** -10  # the forward's approximate tanh; the backward is far tighter


@pytest.fixture(scope="module")
def nccl_group(cuda_device):
    assert not dist.is_initialized()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    yield dist.group.WORLD
    dist.destroy_process_group()


def tp_inputs(T, I, seed):
    wl = dataclasses.replace(workloads.workload(2), tokens=T, inter=I, seed=5000 + seed, rw_kind="uniform")
    return workloads.inputs(wl)


def test_bwd_tp_on_a_side_stream(nccl_group, cuda_device):
    dev = cuda_device
    T, I = 1000, 1024
    x = tp_inputs(T, I, 1)
    gu_full, go_full = to_device(x["gate_up"], dev), to_device(x["grad_out"], dev)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    gu = tp.tp_local_gate_up(gu_full, 0, 1)
    go = tp.tp_local_columns(go_full, 0, 1)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    d_gu, d_rw = tp.situ_glu_bwd_tp(gu, rw, go, 4.0, 25.0, group=nccl_group, stream=side)
    side.synchronize()
    ref = oracle.load().bwd(x["gate_up"], x["routing_weights"], x["grad_out"], 4.0, 25.0)
    d = to_host(d_gu)
    check_output("dG tp", d[:, :I], ref.dg, ref.cg)
    check_output("dU tp", d[:, I:], ref.du)
    check_dw("d_w tp", to_host(d_rw.reshape(T)), ref.dw, ref.sw)


def test_fwd_nvfp4_tp_on_a_side_stream(nccl_group, cuda_device):
    dev = cuda_device
    T, I = 777, 2048
    x = tp_inputs(T, I, 2)
    gu = tp.tp_local_gate_up(to_device(x["gate_up"], dev), 0, 1, align=16)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    data, scale, amax = tp.situ_glu_fwd_nvfp4_tp(gu, rw, 4.0, 25.0, group=nccl_group, stream=side)
    side.synchronize()
    y = oracle.load().fwd(x["gate_up"], x["routing_weights"], 4.0, 25.0)
    check_nvfp4("Y tp", to_host(data), to_host(scale.view(torch.uint8)), float(amax.item()), y,
                REL_BF16 * np.abs(y) + 1e-30)


def test_bwd_nvfp4_tp_on_a_side_stream(nccl_group, cuda_device):
    dev = cuda_device
    T, I = 513, 2048
    x = tp_inputs(T, I, 3)
    gu = tp.tp_local_gate_up(to_device(x["gate_up"], dev), 0, 1, align=16)
    go = tp.tp_local_columns(to_device(x["grad_out"], dev), 0, 1, align=16)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    data, scale, amax, d_rw = tp.situ_glu_bwd_nvfp4_tp(gu, rw, go, 4.0, 25.0, group=nccl_group, stream=side)
    side.synchronize()
    ref = oracle.load().bwd(x["gate_up"], x["routing_weights"], x["grad_out"], 4.0, 25.0)
    vals = np.concatenate([ref.dg, ref.du], axis=1)
    tol = np.concatenate([REL_BF16 * np.abs(ref.dg) + CANCEL * ref.cg, REL_BF16 * np.abs(ref.du)], axis=1) + 1e-30
    check_nvfp4("d_gate_up tp", to_host(data), to_host(scale.view(torch.uint8)), float(amax.item()), vals, tol)
    check_dw("d_w nvfp4 tp", to_host(d_rw.reshape(T)), ref.dw, ref.sw)
