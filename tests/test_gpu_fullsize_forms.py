"""GPU parity at full size for the other output forms, through the public
tensor API in the bench's launch configuration: the routed-MoE workload
(gate_up bf16 [32768, 4096], I = 2048, beta = 4, linear_beta = 25, 1 %
outliers) for every form, and the large workload (gate_up bf16 [131072, 8192])
for the element-wise weights and MXFP8:

  * per-column routing weights [I] and per-element routing weights [T, I]:
    every element of Y and d_gate_up against the fp64 oracle, and every
    element of the weight gradient (the column sums over all rows, or the
    per-element terms);
  * MXFP8 (OCP rule) and NVFP4 Y and d_gate_up with per-row weights: every
    code and every block scale by the interval checkers of parity.py, the
    NVFP4 tensor maxima against the bounds the whole tensor allows, and the
    per-row weight gradient.

The oracle's unchanged per-row code runs on row chunks spread over the host's
threads (the C oracle and numpy release the GIL); each chunk is checked as
soon as it is computed.

Sources: Megatron-LM PR #6673, "Activation" and "Test results" (the formula,
the MXFP8 and NVFP4 recipes); NeMo AutoModel kimi_k3.situ, `_situ_fwd_core` /
`_situ_bwd_core` (the routing weight and its broadcast forms).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import workloads
import ffn_gated_activation_b200 as pkg

from parity import CANCEL, check_dw, check_mx, check_nvfp4, check_output, to_device, to_host

pytestmark = pytest.mark.gpu

THREADS = max(1, min(96, os.cpu_count() or 1))
ROWS = 512            # rows per oracle task
REL_Q = 2.0 ** -10    # the kernels' error bound for bf16 inputs before quantisation (forward MUFU tanh)
BETA, LB = 4.0, 25.0


def _pool(fn, T):
    with ThreadPoolExecutor(max_workers=THREADS) as pool:
        return list(pool.map(fn, range(0, T, ROWS)))


def _inputs(dev, index=2):
    wl = workloads.workload(index)
    x = workloads.inputs(wl)
    return wl, x, to_device(x["gate_up"], dev), to_device(x["grad_out"], dev)


@pytest.mark.parametrize("index", [2, 4], ids=["routed_moe", "large"])
@pytest.mark.parametrize("form", ["per_column", "per_element"])
def test_elementwise_weights_every_element(form, index, cuda_device):
    wl, x, gu, go = _inputs(cuda_device, index)
    T, I = wl.tokens, wl.inter
    beta, lb = wl.betas[0], wl.linear_beta
    assert (beta, lb) == (BETA, LB)
    col = form == "per_column"
    w = workloads.column_weights(wl) if col else workloads.element_weights(wl)
    rw = torch.from_numpy(np.ascontiguousarray(w)).reshape((I,) if col else (T, I)).to(cuda_device)
    y = pkg.situ_glu_fwd(gu, rw, BETA, LB)
    d_gu, d_rw = pkg.situ_glu_bwd(gu, rw, go, BETA, LB)
    torch.cuda.synchronize()
    y_h, dgu_h, drw_h = to_host(y), to_host(d_gu), to_host(d_rw)
    del y, d_gu, d_rw, gu, go, rw
    o = oracle.load()
    gu_h, go_h = x["gate_up"], x["grad_out"]
    mode = oracle.RW_COL if col else oracle.RW_FULL

    def chunk(r0):
        r1 = min(T, r0 + ROWS)
        wr = w if col else w[r0:r1]
        check_output(f"Y rows {r0}..{r1}", y_h[r0:r1], o.fwd(gu_h[r0:r1], wr, BETA, LB, rw_mode=mode))
        ref = o.bwd(gu_h[r0:r1], wr, go_h[r0:r1], BETA, LB, rw_mode=mode)
        check_output(f"dG rows {r0}..{r1}", dgu_h[r0:r1, :I], ref.dg, ref.cg)
        check_output(f"dU rows {r0}..{r1}", dgu_h[r0:r1, I:], ref.du)
        if col:
            return o.dw_columns(gu_h[r0:r1], go_h[r0:r1], BETA, LB)
        check_output(f"d_w rows {r0}..{r1}", drw_h[r0:r1], o.dw_terms(gu_h[r0:r1], go_h[r0:r1], BETA, LB))
        return None

    parts = _pool(chunk, T)
    if col:  # the column sums over every row: the chunks' fp64 sums added in row order
        colsum = np.sum([p[0] for p in parts], axis=0)
        colmag = np.sum([p[1] for p in parts], axis=0)
        check_dw("d_w (per column)", drw_h.reshape(-1), colsum, colmag)


@pytest.mark.parametrize("index", [2, 4], ids=["routed_moe", "large"])
def test_mxfp8_every_code(index, cuda_device):
    wl, x, gu, go = _inputs(cuda_device, index)
    T, I = wl.tokens, wl.inter
    rw = to_device(x["routing_weights"], cuda_device).reshape(T, 1)
    yc, ys = pkg.situ_glu_fwd_mxfp8(gu, rw, BETA, LB, rule="ocp")
    dc, ds, d_rw = pkg.situ_glu_bwd_mxfp8(gu, rw, go, BETA, LB, rule="ocp")
    torch.cuda.synchronize()
    u8 = lambda t: to_host(t.view(torch.uint8))
    yc_h, ys_h, dc_h, ds_h, drw_h = u8(yc), u8(ys), u8(dc), u8(ds), to_host(d_rw.reshape(T))
    del yc, ys, dc, ds, d_rw, gu, go, rw
    o = oracle.load()
    gu_h, go_h = x["gate_up"], x["grad_out"]
    rw_h = np.ascontiguousarray(x["routing_weights"]).reshape(T)

    def chunk(r0):
        r1 = min(T, r0 + ROWS)
        y = o.fwd(gu_h[r0:r1], rw_h[r0:r1], BETA, LB)
        ry = check_mx(f"Y rows {r0}..{r1}", yc_h[r0:r1], ys_h[r0:r1], y, REL_Q * np.abs(y) + 1e-30, oracle.MX_RULE_OCP)
        ref = o.bwd(gu_h[r0:r1], rw_h[r0:r1], go_h[r0:r1], BETA, LB)
        d = np.concatenate([ref.dg, ref.du], axis=1)
        tol = np.concatenate([REL_Q * np.abs(ref.dg) + CANCEL * ref.cg, REL_Q * np.abs(ref.du)], axis=1) + 1e-30
        rd = check_mx(f"d_gate_up rows {r0}..{r1}", dc_h[r0:r1], ds_h[r0:r1], d, tol, oracle.MX_RULE_OCP)
        check_dw(f"d_w rows {r0}..{r1}", drw_h[r0:r1], ref.dw, ref.sw)
        return ry, rd

    parts = _pool(chunk, T)
    for k, name in ((0, "Y"), (1, "d_gate_up")):
        codes = sum(p[k]["codes"] for p in parts)
        exact = sum(p[k]["exact"] for p in parts)
        assert codes == T * I * (1 + k), (name, codes)
        assert exact >= 0.999 * codes, (name, exact, codes)


def test_routed_moe_nvfp4_every_code(cuda_device):
    wl, x, gu, go = _inputs(cuda_device)
    T, I = wl.tokens, wl.inter
    rw = to_device(x["routing_weights"], cuda_device).reshape(T, 1)
    yc, ys, ya = pkg.situ_glu_fwd_nvfp4(gu, rw, BETA, LB)
    dc, ds, da, d_rw = pkg.situ_glu_bwd_nvfp4(gu, rw, go, BETA, LB)
    torch.cuda.synchronize()
    u8 = lambda t: to_host(t.view(torch.uint8))
    yc_h, ys_h, dc_h, ds_h = u8(yc), u8(ys), u8(dc), u8(ds)
    y_amax, d_amax = float(ya.item()), float(da.item())
    drw_h = to_host(d_rw.reshape(T))
    del yc, ys, ya, dc, ds, da, d_rw, gu, go, rw
    o = oracle.load()
    gu_h, go_h = x["gate_up"], x["grad_out"]
    rw_h = np.ascontiguousarray(x["routing_weights"]).reshape(T)

    def bounds(ref, tol):  # the tensor maximum's bounds over this chunk's finite values
        a = np.where(np.isfinite(ref), np.abs(ref), 0.0)
        return float(np.maximum(a - tol, 0.0).max()), float((a + tol).max())

    def chunk(r0):
        r1 = min(T, r0 + ROWS)
        y = o.fwd(gu_h[r0:r1], rw_h[r0:r1], BETA, LB)
        ty = REL_Q * np.abs(y) + 1e-30
        ry = check_nvfp4(f"Y rows {r0}..{r1}", yc_h[r0:r1], ys_h[r0:r1], y_amax, y, ty, full_tensor=False)
        ref = o.bwd(gu_h[r0:r1], rw_h[r0:r1], go_h[r0:r1], BETA, LB)
        d = np.concatenate([ref.dg, ref.du], axis=1)
        td = np.concatenate([REL_Q * np.abs(ref.dg) + CANCEL * ref.cg, REL_Q * np.abs(ref.du)], axis=1) + 1e-30
        rd = check_nvfp4(f"d_gate_up rows {r0}..{r1}", dc_h[r0:r1], ds_h[r0:r1], d_amax, d, td, full_tensor=False)
        check_dw(f"d_w rows {r0}..{r1}", drw_h[r0:r1], ref.dw, ref.sw)
        return ry, rd, bounds(y, ty), bounds(d, td)

    parts = _pool(chunk, T)
    # each tensor maximum within the bounds the whole tensor's oracle values allow
    from parity import NVFP4_SLACK
    for k, amax, name in ((2, y_amax, "Y"), (3, d_amax, "d_gate_up")):
        lo = max(p[k][0] for p in parts)
        hi = max(p[k][1] for p in parts)
        assert lo * (1 - NVFP4_SLACK) <= amax <= hi * (1 + NVFP4_SLACK), (name, lo, amax, hi)
    for k, name in ((0, "Y"), (1, "d_gate_up")):
        codes = sum(p[k]["codes"] for p in parts)
        exact = sum(p[k]["exact"] for p in parts)
        assert codes == T * I * (1 + k), (name, codes)
        assert exact >= 0.999 * codes, (name, exact, codes)
