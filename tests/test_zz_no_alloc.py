"""The allocation-free backward (situ_glu_bwd_no_alloc), through the C ABI.

Callers that cannot allocate device memory where they run the backward (an
engine that plans all of HBM up front, a C caller without a CUDA allocator)
use this entry point: it takes the scratch of the broadcast-weight mode from a
fixed array inside the library.  Its results must match situ_glu_bwd given a
caller-owned workspace, on two calls in a row (the second call reuses the
array the first one left behind).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from ffn_gated_activation_b200 import abi

import parity
from parity import Guarded, call_bwd, to_device, to_host
from test_gpu_parity import case_inputs

pytestmark = pytest.mark.gpu

NO_ALLOC_MAX_TOKENS = 262144


def no_alloc_bwd(gu, inter, rw, rw_mode, beta, lb, go, dgu, d_rw):
    return abi.situ_glu_bwd_no_alloc(gu.data_ptr(), parity.dtype_code(gu), gu.shape[0], inter, gu.stride(0),
                                     rw.data_ptr(), parity.dtype_code(rw), rw_mode, 1, float(beta),
                                     int(lb is not None), float(lb or 0.0), go.data_ptr(), go.stride(0),
                                     dgu.ptr(), dgu.pitch, d_rw.data_ptr() if d_rw is not None else None, 1, 0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_matches_workspace_entry_point_twice(dtype, cuda_device):
    dev = cuda_device
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    for call, (T, I, seed) in enumerate([(777, 520 if dtype == "bf16" else 260, 1), (3001, 2048, 2)]):
        gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=900 + seed)
        gu, go = to_device(gu_h, dev), to_device(go_h, dev)
        w = to_device(rw32[:1].copy(), dev)  # one weight broadcast to every row: the mode that needs scratch
        ref_dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
        ref_dw = torch.empty(1, dtype=torch.float32, device=dev)
        abi.check(call_bwd(gu, I, w, abi.SITU_RW_SCALAR, 4.0, 25.0, go, ref_dgu, d_rw=ref_dw), "situ_glu_bwd")
        out_dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
        out_dw = torch.full((1,), float("nan"), dtype=torch.float32, device=dev)
        abi.check(no_alloc_bwd(gu, I, w, abi.SITU_RW_SCALAR, 4.0, 25.0, go, out_dgu, out_dw),
                  "situ_glu_bwd_no_alloc")
        torch.cuda.synchronize()
        out_dgu.check()
        a, b = to_host(out_dgu.view), to_host(ref_dgu.view)
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), f"call {call}: d_gate_up differs"
        da, db = float(out_dw.item()), float(ref_dw.item())
        assert abs(da - db) <= parity.DW_REL * abs(db), f"call {call}: d_w {da} vs {db}"
        assert da == db  # same kernels, same fixed reduction order


def test_per_column_weights_use_the_fixed_scratch(cuda_device):
    """[I] weights keep one partial per column per 16-row chunk in the scratch."""
    dev = cuda_device
    T, I = 300, 520
    gu_h, _, go_h = case_inputs("bf16", T, I, seed=960)
    gu, go = to_device(gu_h, dev), to_device(go_h, dev)
    w = torch.linspace(0.1, 1.0, I, device=dev)
    ref_dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    ref_dw = torch.empty(I, dtype=torch.float32, device=dev)
    abi.check(call_bwd(gu, I, w, abi.SITU_RW_COL, 4.0, 25.0, go, ref_dgu, d_rw=ref_dw), "situ_glu_bwd")
    for _ in range(2):
        out_dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
        out_dw = torch.full((I,), float("nan"), device=dev)
        abi.check(no_alloc_bwd(gu, I, w, abi.SITU_RW_COL, 4.0, 25.0, go, out_dgu, out_dw), "situ_glu_bwd_no_alloc")
        torch.cuda.synchronize()
        out_dgu.check()
        assert torch.equal(out_dgu.view.view(torch.int16), ref_dgu.view.view(torch.int16))
        assert torch.equal(out_dw, ref_dw)


def test_row_mode_needs_no_scratch(cuda_device):
    dev = cuda_device
    T, I = 129, 264
    gu_h, rw32, go_h = case_inputs("bf16", T, I, seed=950)
    gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
    ref_dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    ref_dw = torch.empty(T, dtype=torch.float32, device=dev)
    abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, ref_dgu, d_rw=ref_dw), "situ_glu_bwd")
    out_dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    out_dw = torch.empty(T, dtype=torch.float32, device=dev)
    abi.check(no_alloc_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, out_dgu, out_dw), "situ_glu_bwd_no_alloc")
    torch.cuda.synchronize()
    assert torch.equal(out_dgu.view.view(torch.int16), ref_dgu.view.view(torch.int16))
    assert torch.equal(out_dw, ref_dw)


def test_rejects_rows_beyond_the_fixed_scratch(cuda_device):
    dev = cuda_device
    T, I = NO_ALLOC_MAX_TOKENS + 1, 8
    gu = torch.zeros(T, 2 * I, dtype=torch.bfloat16, device=dev)
    go = torch.zeros(T, I, dtype=torch.bfloat16, device=dev)
    w = torch.ones(1, dtype=torch.float32, device=dev)
    dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    d_w = torch.full((1,), 5.0, device=dev)
    st = no_alloc_bwd(gu, I, w, abi.SITU_RW_SCALAR, 4.0, 25.0, go, dgu, d_w)
    assert st == abi.SITU_ERR_UNSUPPORTED
    assert "fixed scratch" in abi.situ_glu_last_error()
    torch.cuda.synchronize()
    assert d_w.item() == 5.0  # nothing was launched


def test_rejects_per_column_partials_beyond_the_fixed_scratch(cuda_device):
    dev = cuda_device
    T, I = 16 * 65, 4096  # 65 chunks x 4096 columns x 4 bytes > 1 MiB
    gu = torch.zeros(T, 2 * I, dtype=torch.bfloat16, device=dev)
    go = torch.zeros(T, I, dtype=torch.bfloat16, device=dev)
    w = torch.ones(I, dtype=torch.float32, device=dev)
    dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    d_w = torch.full((I,), 5.0, device=dev)
    st = no_alloc_bwd(gu, I, w, abi.SITU_RW_COL, 4.0, 25.0, go, dgu, d_w)
    assert st == abi.SITU_ERR_UNSUPPORTED
    assert "fixed scratch" in abi.situ_glu_last_error()
    torch.cuda.synchronize()
    assert torch.all(d_w == 5.0)
