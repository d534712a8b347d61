"""GPU parity at the full workload sizes, in the launch configuration the bench
times (the public tensor API, default launch size, current stream):

  * sampled rows (first, last and seeded random ones) against the fp64 oracle
    element by element;
  * properties that hold at any size, over every row, checked on the device:
    finite outputs, |Y| <= beta * beta_L * |w| (beta * |U| * |w| without a
    linear beta), Y = 0 wherever G = 0 or U = 0, and the routing-weight
    gradient identity d_w[r] * w[r] = sum_i go[r, i] * Y[r, i] (Y is linear
    in w), evaluated from the kernel's own bf16/fp32 Y.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import ffn_gated_activation_b200 as pkg

from parity import check_dw, check_output, to_device, to_host

pytestmark = pytest.mark.gpu

SAMPLE_ROWS = 48


def sample_rows(T: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    rows = {0, 1, T // 2, T - 2, T - 1} | set(rng.integers(0, T, SAMPLE_ROWS).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < T), dtype=np.int64)


def _properties(wl, beta, lb, gu, rw, go, y, d_rw, chunk=4096):
    """Size-independent checks over every row, in row chunks on the device."""
    T, I = wl.tokens, wl.inter
    for r0 in range(0, T, chunk):
        r1 = min(T, r0 + chunk)
        g = gu[r0:r1, :I].double()
        u = gu[r0:r1, I:].double()
        w = rw[r0:r1].double().reshape(-1, 1)
        yy = y[r0:r1].double()
        assert torch.isfinite(yy).all(), "non-finite output"
        bound = (beta * lb if lb is not None else beta * u.abs()) * w.abs()
        assert (yy.abs() <= bound * (1 + 2.0 ** -7)).all(), "|Y| exceeds beta * beta_L * |w|"
        zero = (g == 0) | (u == 0)
        assert (yy[zero] == 0).all(), "Y nonzero where G or U is zero"
        lhs = d_rw[r0:r1].double() * w.reshape(-1)
        prod = go[r0:r1].double() * yy
        rhs, mag = prod.sum(dim=1), prod.abs().sum(dim=1)
        # Y carries one rounding to the storage dtype per element.
        rel = 2.0 ** -8 if y.dtype == torch.bfloat16 else 2.0 ** -16
        assert ((lhs - rhs).abs() <= rel * mag + 1e-4 * rhs.abs() + 1e-30).all(), \
            "d_w * w != sum go * Y"


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_fullsize(index, cuda_device):
    dev = cuda_device
    wl = workloads.workload(index)
    x = workloads.inputs(wl)
    T, I = wl.tokens, wl.inter
    gu = to_device(x["gate_up"], dev)
    go = to_device(x["grad_out"], dev)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    rows = sample_rows(T, seed=index)
    o = oracle.load()
    for beta in wl.betas:
        lb = wl.linear_beta
        y = pkg.situ_glu_fwd(gu, rw, beta, lb)
        d_gu, d_rw = pkg.situ_glu_bwd(gu, rw, go, beta, lb)
        torch.cuda.synchronize()
        _properties(wl, beta, lb, gu, rw.reshape(T), go, y, d_rw.reshape(T))

        idx = torch.from_numpy(rows).to(dev)
        y_s = to_host(y.index_select(0, idx))
        d_s = to_host(d_gu.index_select(0, idx))
        dw_s = to_host(d_rw.reshape(T).index_select(0, idx))
        ref_y = o.fwd(x["gate_up"], x["routing_weights"], beta, lb, rows=rows)
        ref = o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], beta, lb, rows=rows)
        tag = f"{wl.name} beta={beta}"
        check_output(f"Y {tag}", y_s, ref_y)
        check_output(f"dG {tag}", d_s[:, :I], ref.dg, ref.cg)
        check_output(f"dU {tag}", d_s[:, I:], ref.du)
        check_dw(f"d_w {tag}", dw_s, ref.dw, ref.sw)
        del y, d_gu, d_rw
    del gu, go, rw
    torch.cuda.empty_cache()


def test_tiny_workload_every_element(cuda_device):
    """The tiny workload (T = 256, I = 512) compared in full."""
    dev = cuda_device
    wl = workloads.workload(0)
    x = workloads.inputs(wl)
    T, I = wl.tokens, wl.inter
    gu, go = to_device(x["gate_up"], dev), to_device(x["grad_out"], dev)
    rw = to_device(x["routing_weights"], dev).reshape(T, 1)
    y = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
    d_gu, d_rw = pkg.situ_glu_bwd(gu, rw, go, 4.0, 25.0)
    torch.cuda.synchronize()
    o = oracle.load()
    ref_y = o.fwd(x["gate_up"], x["routing_weights"], 4.0, 25.0)
    ref = o.bwd(x["gate_up"], x["routing_weights"], x["grad_out"], 4.0, 25.0)
    check_output("Y tiny", to_host(y), ref_y)
    d = to_host(d_gu)
    check_output("dG tiny", d[:, :I], ref.dg, ref.cg)
    check_output("dU tiny", d[:, I:], ref.du)
    check_dw("d_w tiny", to_host(d_rw.reshape(T)), ref.dw, ref.sw)
