"""GPU parity of the element-wise routing-weight forms: one weight per column
(w[I], broadcast over rows) and one weight per element (w[T, I]), against the
fp64 oracle on the same seeded inputs (tolerance rule in parity.py).

NeMo AutoModel's kimi_k3.situ `_WeightedSiTUFunction.forward` accepts any
routing_weights that broadcast against the output; the per-column gradient is
the sum over rows of go T_g T_u, the per-element gradient is that term itself.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import Guarded, as_f64, call_bwd, call_fwd, check_dw, check_output, to_device, to_host

pytestmark = pytest.mark.gpu


def ew_inputs(dtype: str, T: int, I: int, seed: int):
    wl = dataclasses.replace(workloads.workload(2), dtype=dtype, tokens=T, inter=I, seed=2000 + seed)
    x = workloads.inputs(wl)
    return (x["gate_up"], x["grad_out"], workloads.column_weights(wl), workloads.element_weights(wl))


def run_ew(dev, dtype, T, I, beta, lb, full, rw_dtype, seed, rw_pad=0, d_rw_pad=0, want_drw=True, gate_values=None):
    gu_h, go_h, wc, wf = ew_inputs(dtype, T, I, seed)
    if gate_values is not None:  # row r's first gate columns: the values rotated by r
        vals = np.array(gate_values, dtype=np.float32)
        vals = workloads.f32_to_bf16_bits(vals) if dtype == "bf16" else vals
        for r in range(T):
            gu_h[r, :len(vals)] = np.roll(vals, r)
    w32 = wf if full else wc
    w_h = workloads.f32_to_bf16_bits(w32) if rw_dtype == "bf16" else w32
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    wdt = torch.bfloat16 if rw_dtype == "bf16" else torch.float32
    gu, go = to_device(gu_h, dev), to_device(go_h, dev)
    mode = abi.SITU_RW_FULL if full else abi.SITU_RW_COL
    if full:
        pitch = I + rw_pad
        wbuf = torch.full((max(T, 1), pitch), float("nan"), dtype=wdt, device=dev)
        wbuf[:T, :I] = to_device(w_h, dev)
        rw, rw_stride = wbuf, pitch
        d_rw = Guarded(T, I, I + d_rw_pad, wdt, dev) if want_drw else None
        d_rw_stride = I + d_rw_pad
    else:
        rw, rw_stride = to_device(w_h, dev), 1
        d_rw = Guarded(1, I, I, wdt, dev) if want_drw else None
        d_rw_stride = 1
    out = Guarded(T, I, I, tdt, dev)
    dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
    abi.check(call_fwd(gu, I, rw, mode, beta, lb, out, rw_stride=rw_stride), "fwd")

    class _Ptr:  # call_bwd takes a tensor-like d_rw with data_ptr()
        def __init__(self, g): self.g = g
        def data_ptr(self): return self.g.ptr()

    abi.check(call_bwd(gu, I, rw, mode, beta, lb, go, dgu, d_rw=_Ptr(d_rw) if d_rw else None,
                       rw_stride=rw_stride, d_rw_stride=d_rw_stride), "bwd")
    torch.cuda.synchronize()
    out.check()
    dgu.check()
    if d_rw is not None:
        d_rw.check()

    o = oracle.load()
    omode = oracle.RW_FULL if full else oracle.RW_COL
    ref_y = o.fwd(gu_h, w_h, beta, lb, rw_mode=omode)
    ref = o.bwd(gu_h, w_h, go_h, beta, lb, rw_mode=omode)
    check_output("Y", to_host(out.view), ref_y)
    d = to_host(dgu.view)
    check_output("dG", d[:, :I], ref.dg, cancel_scale=ref.cg)
    check_output("dU", d[:, I:], ref.du)
    if d_rw is None:
        return d
    got = to_host(d_rw.view)
    if full:
        check_output("d_w (per element)", got, o.dw_terms(gu_h, go_h, beta, lb))
    else:
        colsum, colmag = o.dw_columns(gu_h, go_h, beta, lb)
        check_dw("d_w (per column)", got.reshape(-1), colsum, colmag)
    return d, got


# 16-row chunks: T = 1, 3 (one ragged chunk), 130, 257 (several, ragged tail).
# I = 8200 (bf16) and 4096 (fp32) exceed two vectors per thread: the looped form.
SHAPES = [("bf16", 1, 8), ("bf16", 3, 24), ("bf16", 257, 520), ("bf16", 130, 2048), ("bf16", 70, 3072),
          ("bf16", 37, 8200), ("f32", 1, 4), ("f32", 33, 260), ("f32", 65, 4096)]
COMBOS = [(4.0, 25.0, "f32"), (1.0, None, "bf16"), (2.0, 1.5, "f32"), (16.0, None, "bf16")]


@pytest.mark.parametrize("full", [False, True], ids=["per_column", "per_element"])
@pytest.mark.parametrize("dtype,T,I", SHAPES, ids=[f"{d}-{t}x{i}" for d, t, i in SHAPES])
@pytest.mark.parametrize("beta,lb,rw_dtype", COMBOS, ids=[f"b{b}-lb{l}-w{w}" for b, l, w in COMBOS])
def test_elementwise_parity(dtype, T, I, beta, lb, rw_dtype, full, cuda_device):
    run_ew(cuda_device, dtype, T, I, beta, lb, full, rw_dtype, seed=T * 5 + I)


# Gate values around and beyond the bf16 backward's clamp at -27.75 (where the
# per-column form's signed gate arithmetic stops following g) and the usual
# special values.
GATE_SPECIALS = [0.0, -0.0, np.inf, -np.inf, 3e38, -3e38, -1e-30, 1e-39, -1.21875, 60.0, -27.5, -27.75, -28.0,
                 -30.0, -40.0, -60.0, -88.0, -100.0, 1e-3, -1e-3]


@pytest.mark.parametrize("full", [False, True], ids=["per_column", "per_element"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_elementwise_special_gate_values(dtype, full, cuda_device):
    run_ew(cuda_device, dtype, 40, 64, 4.0, 25.0, full, "f32", seed=11, gate_values=GATE_SPECIALS)


@pytest.mark.parametrize("dtype,rw_dtype", [("bf16", "f32"), ("bf16", "bf16"), ("f32", "f32")])
def test_per_element_strided_weights(dtype, rw_dtype, cuda_device):
    """Row pitches of w and d_w above I (16-byte multiples); guard bytes catch
    any write into the padding."""
    pad = 8 if rw_dtype == "bf16" else 4
    run_ew(cuda_device, dtype, 67, 264, 4.0, 25.0, True, rw_dtype, seed=3, rw_pad=pad, d_rw_pad=2 * pad)


@pytest.mark.parametrize("full", [False, True])
def test_elementwise_gradient_not_wanted(full, cuda_device):
    """Without a weight gradient dG and dU are bitwise the same."""
    a, _ = run_ew(cuda_device, "bf16", 129, 520, 4.0, 25.0, full, "f32", seed=9)
    b = run_ew(cuda_device, "bf16", 129, 520, 4.0, 25.0, full, "f32", seed=9, want_drw=False)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("I", [1024, 8200])
def test_per_column_gradient_grid_invariant(I, cuda_device):
    """The [I] gradient adds fixed 16-row chunks in chunk order: the result does
    not depend on how many CTAs run (registers or shared memory alike)."""
    results = []
    for ctas in (0, 1, 3, 37):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            results.append(run_ew(cuda_device, "bf16", 300, I, 4.0, 25.0, False, "f32", seed=4)[1])
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for r in results[1:]:
        assert np.array_equal(r.view(np.uint8), results[0].view(np.uint8))


def test_per_column_zero_tokens(cuda_device):
    dev = cuda_device
    gu = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    w = torch.ones(32, device=dev)
    d_w = torch.full((32,), 7.0, device=dev)
    y = pkg.situ_glu_fwd(gu, w)
    assert y.shape == (0, 32)
    pkg.situ_glu_bwd(gu, w, torch.empty(0, 32, dtype=torch.bfloat16, device=dev), d_rw=d_w)
    torch.cuda.synchronize()
    assert torch.all(d_w == 0.0)


@pytest.mark.parametrize("form", ["per_column", "per_element"])
def test_elementwise_autograd(form, cuda_device):
    """weighted_situ with [I] and [B, S, I] weights through torch.autograd."""
    dev = cuda_device
    B, S, I = 2, 45, 264
    T = B * S
    gu_h, go_h, wc, wf = ew_inputs("bf16", T, I, seed=31)
    gu = to_device(gu_h, dev).reshape(B, S, 2 * I).requires_grad_(True)
    go = to_device(go_h, dev).reshape(B, S, I)
    if form == "per_column":
        w = to_device(wc, dev).requires_grad_(True)
        w_h, omode = wc, oracle.RW_COL
    else:
        w = to_device(wf, dev).reshape(B, S, I).requires_grad_(True)
        w_h, omode = wf, oracle.RW_FULL
    y = pkg.weighted_situ(gu, w, 4.0, 25.0)
    assert y.shape == (B, S, I)
    y.backward(go)
    assert w.grad.shape == w.shape
    o = oracle.load()
    check_output("Y", to_host(y.reshape(T, I)), o.fwd(gu_h, w_h, 4.0, 25.0, rw_mode=omode))
    ref = o.bwd(gu_h, w_h, go_h, 4.0, 25.0, rw_mode=omode)
    g = to_host(gu.grad.reshape(T, 2 * I))
    check_output("dG", g[:, :I], ref.dg, ref.cg)
    check_output("dU", g[:, I:], ref.du)
    if form == "per_column":
        colsum, colmag = o.dw_columns(gu_h, go_h, 4.0, 25.0)
        check_dw("d_w", to_host(w.grad), colsum, colmag)
    else:
        check_output("d_w", to_host(w.grad.reshape(T, I)), o.dw_terms(gu_h, go_h, 4.0, 25.0))
