"""CUDA-graph capture of the library's calls: small calls are launch-bound,
and a graph replays their launches without the host's per-call work.  Each
test warms the calls up eagerly on a side stream (which also sets the kernels'
shared-memory attributes outside the capture), captures them into one
torch.cuda.CUDAGraph, then refills the captured input buffers with new
values and replays.  The replayed outputs must equal, bit for bit, an eager
call on the same inputs, and match the fp64 oracle by the tolerance rule.

Sources: Megatron-LM PR #6673, "Activation" (the formula); NeMo AutoModel
kimi_k3.situ, `_situ_fwd_core` / `_situ_bwd_core` (the routing-weight forms).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
import ffn_gated_activation_b200 as pkg

from parity import check_ar, check_dw, check_output, to_device, to_host

pytestmark = pytest.mark.gpu

T, I = 300, 1024


def _inputs(seed):
    wl = dataclasses.replace(workloads.workload(2), tokens=T, inter=I, seed=5000 + seed, rw_kind="uniform")
    return workloads.inputs(wl)


def _weights(kind, x):
    """Host routing weights of a form and the oracle's mode for them."""
    if kind == "row":
        return np.ascontiguousarray(x["routing_weights"]).reshape(T, 1), oracle.RW_ROW
    if kind == "scalar":
        return np.ascontiguousarray(x["routing_weights"][:1]).reshape(()), oracle.RW_SCALAR
    rng = np.random.default_rng(int(x["routing_weights"].view(np.uint32)[0]))
    if kind == "col":
        return rng.uniform(0.0, 1.0, I).astype(np.float32), oracle.RW_COL
    return rng.uniform(0.0, 1.0, (T, I)).astype(np.float32), oracle.RW_FULL


def _warm(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()


@pytest.mark.parametrize("kind", ["row", "col", "scalar", "full"])
def test_fwd_bwd_graph_replay(kind, cuda_device):
    dev = cuda_device
    x0 = _inputs(0)
    w0, mode = _weights(kind, x0)
    gu = to_device(x0["gate_up"], dev)
    go = to_device(x0["grad_out"], dev)
    rw = torch.from_numpy(np.array(w0)).to(dev)

    def step():
        y = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
        d_gu, d_rw = pkg.situ_glu_bwd(gu, rw, go, 4.0, 25.0)
        return y, d_gu, d_rw

    _warm(step)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        y_s, dgu_s, drw_s = step()
    o = oracle.load()
    for seed in (1, 2):
        x = _inputs(seed)
        w, _ = _weights(kind, x)
        gu.copy_(to_device(x["gate_up"], dev))
        go.copy_(to_device(x["grad_out"], dev))
        rw.copy_(torch.from_numpy(np.array(w)).to(dev))
        g.replay()
        torch.cuda.synchronize()
        got = [to_host(y_s), to_host(dgu_s), to_host(drw_s)]
        ref_eager = [to_host(t) for t in step()]
        torch.cuda.synchronize()
        for a, b in zip(got, ref_eager):
            assert np.array_equal(np.atleast_1d(a).view(np.uint8), np.atleast_1d(b).view(np.uint8)), \
                f"{kind}: replay differs from eager"
        wf = np.array(w, dtype=np.float32)
        ref_y = o.fwd(x["gate_up"], wf.reshape(-1) if kind != "full" else wf, 4.0, 25.0, rw_mode=mode)
        check_output(f"Y {kind} replay {seed}", got[0], ref_y)
        ref = o.bwd(x["gate_up"], wf.reshape(-1) if kind != "full" else wf, x["grad_out"], 4.0, 25.0, rw_mode=mode)
        check_output(f"dG {kind} replay {seed}", got[1][:, :I], ref.dg, ref.cg)
        check_output(f"dU {kind} replay {seed}", got[1][:, I:], ref.du)
        if kind == "row":
            check_dw(f"d_w replay {seed}", got[2].reshape(T), ref.dw, ref.sw)
    del g


def test_mixed_graph_replay(cuda_device):
    """MXFP8 forward and backward, the attention-residual core and the fused
    FC1 in one graph, replayed on new inputs: each output equals an eager call."""
    dev = cuda_device
    x = _inputs(3)
    gu = to_device(x["gate_up"], dev)
    go = to_device(x["grad_out"], dev)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    ar = workloads.attn_res_inputs(T, 4, 512, 3)
    blocks, prefix = to_device(ar["blocks"], dev), to_device(ar["prefix"], dev)
    nw, pw = to_device(ar["norm_weight"], dev), to_device(ar["proj_weight"], dev)
    H, E = 256, 3
    gen = torch.Generator().manual_seed(3)
    xa = (torch.randn(T, H, generator=gen)).to(torch.bfloat16).to(dev)
    w1 = (torch.randn(E, 2 * I, H, generator=gen) * H ** -0.5).to(torch.bfloat16).to(dev)
    offsets = torch.tensor([0, 90, 90, T], dtype=torch.int64, device=dev)

    def step():
        yc, ys = pkg.situ_glu_fwd_mxfp8(gu, rw, 4.0, 25.0, rule="ocp")
        dc, ds, d_rw = pkg.situ_glu_bwd_mxfp8(gu, rw, go, 4.0, 25.0, rule="ocp")
        mix = pkg.apply_attn_res(prefix, blocks, pw, nw, 1e-6)
        fc1 = pkg.situ_glu_fc1_fwd(xa, w1, offsets, rw, 4.0, 25.0)
        return yc, ys, dc, ds, d_rw, mix, fc1

    _warm(step)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = step()
    x2 = _inputs(4)
    ar2 = workloads.attn_res_inputs(T, 4, 512, 4)
    gu.copy_(to_device(x2["gate_up"], dev))
    go.copy_(to_device(x2["grad_out"], dev))
    rw.copy_(to_device(x2["routing_weights"], dev).reshape(T, 1))
    blocks.copy_(to_device(ar2["blocks"], dev))
    prefix.copy_(to_device(ar2["prefix"], dev))
    xa.copy_((torch.randn(T, H, generator=gen)).to(torch.bfloat16).to(dev))
    g.replay()
    torch.cuda.synchronize()
    got = [to_host(t.view(torch.uint8) if t.element_size() == 1 else t) for t in outs]
    eager = [to_host(t.view(torch.uint8) if t.element_size() == 1 else t) for t in step()]
    torch.cuda.synchronize()
    names = ("Y codes", "Y scales", "d_gate_up codes", "d_gate_up scales", "d_w", "attention mix", "FC1 Y")
    for name, a, b in zip(names, got, eager):
        assert np.array_equal(np.atleast_1d(a).view(np.uint8), np.atleast_1d(b).view(np.uint8)), \
            f"{name}: replay differs from eager"
    # the replayed attention mix against the oracle on the new sums (the
    # norm and projection weights are the captured ones)
    ref, mag, _ = oracle.load().attn_res(ar2["blocks"], ar2["prefix"], ar["norm_weight"], ar["proj_weight"], 1e-6)
    check_ar("attention mix replay", got[5], ref, mag)
    del g
