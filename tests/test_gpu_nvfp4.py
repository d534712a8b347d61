"""GPU parity of the NVFP4 outputs (situ_glu_fwd_nvfp4, situ_glu_bwd_nvfp4)
against the fp64 oracle's values quantised by the oracle's NVFP4 block
scaling (E2M1 codes, an E4M3 scale per 16 elements of a row, the per-tensor
scale 2688 / A).

The kernel quantises its fp32 results, which differ from the oracle's exact
values by at most `tol` (2^-10 relative for bf16 inputs -- the forward's
approximate tanh -- 1e-5 for fp32 inputs, plus 2^-18 C_G for dG, the bound of
the native-output tests).  Quantisation is monotone, so
parity.check_nvfp4 bounds the kernel's tensor maximum A, each block scale and
each code between the oracle's results at the two ends of that interval, and
asks at least 90 % of the codes to equal the oracle's exactly.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import CANCEL, Guarded, check_dw, check_nvfp4, to_device, to_host, unpack_e2m1

pytestmark = pytest.mark.gpu

REL = {"bf16": 2.0 ** -10, "f32": 1e-5}
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def nv_inputs(dtype: str, T: int, I: int, seed: int):
    wl = dataclasses.replace(workloads.workload(2), dtype=dtype, tokens=T, inter=I, seed=4000 + seed,
                             rw_kind="uniform")
    x = workloads.inputs(wl)
    return x["gate_up"], x["routing_weights"], x["grad_out"]


def rw_case(kind, rw32):
    if kind == "row_f32":
        return rw32, abi.SITU_RW_ROW
    if kind == "row_bf16":
        return workloads.f32_to_bf16_bits(rw32), abi.SITU_RW_ROW
    if kind == "scalar":
        return rw32[:1].copy(), abi.SITU_RW_SCALAR
    return None, abi.SITU_RW_NONE


def oracle_y(gu_h, rw_h, T, beta, lb):
    o = oracle.load()
    if rw_h is None:
        return o.fwd(gu_h, np.ones(T, dtype=np.float32), beta, lb)
    mode = oracle.RW_SCALAR if rw_h.size == 1 and T != 1 else oracle.RW_ROW
    return o.fwd(gu_h, rw_h, beta, lb, rw_mode=mode)


def run_nv(dev, dtype, T, I, beta, lb, kind, seed, pad=0, gu_h=None, given=None, data_pitch=None):
    g_h, rw32, _ = nv_inputs(dtype, T, I, seed)
    gu_h = g_h if gu_h is None else gu_h
    rw_h, mode = rw_case(kind, rw32)
    gu = to_device(gu_h, dev)
    rw = to_device(rw_h, dev) if rw_h is not None else None
    rw_ptr = rw.data_ptr() if rw is not None else None
    rw_dt = (abi.SITU_DTYPE_BF16 if rw.dtype == torch.bfloat16 else abi.SITU_DTYPE_F32) if rw is not None else 1
    dt = abi.SITU_DTYPE_BF16 if dtype == "bf16" else abi.SITU_DTYPE_F32
    data = Guarded(T, I // 2, data_pitch or I // 2 + 16 * pad, torch.uint8, dev)
    scale = Guarded(T, I // 16, I // 16 + pad, torch.uint8, dev)
    amax = torch.full((1,), float("nan") if given is None else given, dtype=torch.float32, device=dev)
    abi.check(abi.situ_glu_fwd_nvfp4(gu.data_ptr(), dt, T, I, gu.stride(0), rw_ptr, rw_dt, mode, 1, beta,
                                     int(lb is not None), float(lb or 0.0), data.ptr(), data.pitch, scale.ptr(),
                                     scale.pitch, amax.data_ptr(), int(given is not None), 0), "fwd_nvfp4")
    torch.cuda.synchronize()
    data.check()
    scale.check()
    a = float(amax.item())
    if given is not None:
        assert a == np.float32(given), "a given tensor maximum was overwritten"
    y = oracle_y(gu_h, rw_h, T, beta, lb)
    tol = REL[dtype] * np.abs(np.nan_to_num(y)) + 1e-30
    rep = check_nvfp4("Y", to_host(data.view), to_host(scale.view), a, y, tol, full_tensor=given is None)
    return rep, (to_host(data.view), to_host(scale.view), a)


# Rows of 16 (one block) up to 8192 (the looped form: more than two vectors a thread).
SHAPES = [("bf16", 1, 16), ("bf16", 3, 48), ("bf16", 257, 512), ("bf16", 64, 2048), ("bf16", 40, 3072),
          ("bf16", 5, 8192), ("f32", 1, 16), ("f32", 33, 272), ("f32", 17, 4096)]
COMBOS = [(4.0, 25.0, "row_f32"), (1.0, None, "row_bf16"), (2.0, 1.5, "scalar"), (16.0, None, "none")]


@pytest.mark.parametrize("dtype,T,I", SHAPES, ids=[f"{d}-{t}x{i}" for d, t, i in SHAPES])
@pytest.mark.parametrize("beta,lb,kind", COMBOS, ids=[f"b{b}-lb{l}-{k}" for b, l, k in COMBOS])
def test_nvfp4_parity(dtype, T, I, beta, lb, kind, cuda_device):
    run_nv(cuda_device, dtype, T, I, beta, lb, kind, seed=T * 5 + I)


def test_nvfp4_padded_pitches(cuda_device):
    """Row pitches above the row (data +16 bytes, scales +1; and an 8-byte data
    row, I = 16, with a 12-byte pitch): guard bytes catch any write into the
    padding."""
    run_nv(cuda_device, "bf16", 67, 256, 4.0, 25.0, "row_f32", seed=5, pad=1)
    run_nv(cuda_device, "f32", 9, 16, 4.0, 25.0, "row_f32", seed=5, data_pitch=12)


def test_nvfp4_given_amax(cuda_device):
    """A caller's tensor maximum (twice the call's own) is used as given and
    not overwritten."""
    _, (_, _, a) = run_nv(cuda_device, "bf16", 70, 512, 4.0, 25.0, "row_f32", seed=6)
    run_nv(cuda_device, "bf16", 70, 512, 4.0, 25.0, "row_f32", seed=6, given=2.0 * a)


def test_nvfp4_special_blocks(cuda_device):
    """NaN and infinite elements mark their own blocks (scale code 0x7F) and
    stay out of the tensor maximum; an all-zero row has zero scales and codes;
    tiny rows get small or zero block scales."""
    T, I = 6, 128
    g_h, _, _ = nv_inputs("bf16", T, I, seed=78)
    gu = workloads.bf16_bits_to_f32(g_h).copy()
    gu[0, 5] = np.nan
    gu[1, I + 40] = np.inf
    gu[2, :] = 0.0
    gu[3, :I] = 1e30
    gu[4, :] *= np.float32(1e-30)
    gu[5, :I] = -np.inf
    bits = workloads.f32_to_bf16_bits(gu.astype(np.float32))
    _, (d, s, a) = run_nv(cuda_device, "bf16", T, I, 4.0, None, "none", seed=78, gu_h=bits)
    assert s[0, 0] == 0x7F and s[1, 2] == 0x7F and np.isfinite(a)
    assert np.all(s[2] == 0) and not np.any(unpack_e2m1(d[2:3]) & 7)


def test_nvfp4_all_zero_tensor(cuda_device):
    """A = 0: S_enc = 1, every scale and code zero, A written as 0."""
    T, I = 9, 64
    bits = np.zeros((T, 2 * I), dtype=np.uint16)
    _, (d, s, a) = run_nv(cuda_device, "bf16", T, I, 4.0, 25.0, "none", seed=1, gu_h=bits)
    assert a == 0.0 and not np.any(s) and not np.any(unpack_e2m1(d) & 7)


def test_nvfp4_grid_invariant(cuda_device):
    """Codes, scales and the tensor maximum do not depend on the launch size."""
    outs = []
    for ctas in (0, 1, 7):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_nv(cuda_device, "bf16", 150, 1024, 4.0, 25.0, "row_f32", seed=8)[1])
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        assert np.array_equal(other[0], outs[0][0]) and np.array_equal(other[1], outs[0][1])
        assert other[2] == outs[0][2]


def decode(data: torch.Tensor, scale: torch.Tensor, amax: float) -> np.ndarray:
    codes = unpack_e2m1(data.cpu().numpy())
    q = np.where(codes & 8, -1.0, 1.0) * E2M1[codes & 7]
    sb = scale.to(torch.float64).cpu().numpy()
    s_enc = oracle.load().nvfp4_tensor_scale(amax)
    return q * np.repeat(sb, 16, axis=-1) / s_enc, np.repeat(sb, 16, axis=-1) / s_enc


def test_nvfp4_tensor_api(cuda_device):
    """The tensor-level function: shapes, dtypes, leading dimensions, the same
    bytes as the C-ABI call, and decoding (torch's E4M3 for the block scales)
    within NVFP4's error: a quarter of the block's step (max(1, |q|) / 4 of
    s_b / S_enc) plus the kernel's own 2^-10 relative error."""
    dev = cuda_device
    B, S, I = 2, 33, 256
    T = B * S
    g_h, rw32, _ = nv_inputs("bf16", T, I, seed=9)
    gu = to_device(g_h, dev).reshape(B, S, 2 * I)
    rw = to_device(rw32, dev).reshape(B, S, 1)
    d, s, a = pkg.situ_glu_fwd_nvfp4(gu, rw, 4.0, 25.0)
    assert d.dtype == torch.uint8 and d.shape == (B, S, I // 2)
    assert s.dtype == torch.float8_e4m3fn and s.shape == (B, S, I // 16)
    assert a.dtype == torch.float32 and a.shape == (1,)
    _, (dc, sc, ac) = run_nv(dev, "bf16", T, I, 4.0, 25.0, "row_f32", seed=9)
    assert np.array_equal(d.reshape(T, -1).cpu().numpy(), dc)
    assert np.array_equal(s.view(torch.uint8).reshape(T, -1).cpu().numpy(), sc)
    assert float(a.item()) == ac
    y, unit = decode(d, s, float(a.item()))
    ref = oracle.load().fwd(g_h, rw32, 4.0, 25.0).reshape(B, S, I)
    assert np.all(np.abs(y - ref) <= 0.25 * np.maximum(unit, np.abs(ref)) * (1 + 2.0 ** -6) + 2.0 ** -10 * np.abs(ref))
    # a second call with the returned maximum as given gives the same bytes
    d2, s2, _ = pkg.situ_glu_fwd_nvfp4(gu, rw, 4.0, 25.0, amax=a.clone())
    assert torch.equal(d2, d) and torch.equal(s2.view(torch.uint8), s.view(torch.uint8))


def test_nvfp4_zero_tokens(cuda_device):
    gu = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda_device)
    d, s, a = pkg.situ_glu_fwd_nvfp4(gu, None, 4.0, 25.0)
    torch.cuda.synchronize()
    assert d.shape == (0, 16) and s.shape == (0, 2) and float(a.item()) == 0.0


def test_nvfp4_routed_moe_size_sampled_rows(cuda_device):
    """32768 token rows, I = 2048, per-row weights: 48 sampled rows against the
    oracle; the tensor maximum against the kernel's own bf16 forward over every
    row (within one bf16 rounding) and at least the sampled rows' maximum."""
    wl = workloads.workload(2)
    x = workloads.inputs(wl)
    T, I, beta = wl.tokens, wl.inter, wl.betas[0]
    gu = to_device(x["gate_up"], cuda_device)
    rw = to_device(x["routing_weights"], cuda_device).reshape(T, 1)
    d, s, a = pkg.situ_glu_fwd_nvfp4(gu, rw, beta, wl.linear_beta)
    y16 = pkg.situ_glu_fwd(gu, rw, beta, wl.linear_beta)
    torch.cuda.synchronize()
    a = float(a.item())
    m16 = float(y16.float().abs().max().item())
    assert abs(a - m16) <= 2.0 ** -8 * m16, (a, m16)
    rng = np.random.default_rng(31)
    rows = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 46)]))
    o = oracle.load()
    y = o.fwd(x["gate_up"][rows], x["routing_weights"][rows], beta, wl.linear_beta)
    check_nvfp4("Y (sampled rows)", d[rows.tolist()].cpu().numpy(), s.view(torch.uint8)[rows.tolist()].cpu().numpy(),
                a, y, 2.0 ** -10 * np.abs(y) + 1e-30, full_tensor=False)


# ---- backward ---------------------------------------------------------------------------

def run_nv_bwd(dev, dtype, T, I, beta, lb, kind, seed, pad=0, gu_h=None, given=None):
    g_h, rw32, go_h = nv_inputs(dtype, T, I, seed)
    gu_h = g_h if gu_h is None else gu_h
    rw_h, mode = rw_case(kind, rw32)
    gu, go = to_device(gu_h, dev), to_device(go_h, dev)
    rw = to_device(rw_h, dev) if rw_h is not None else None
    rw_ptr = rw.data_ptr() if rw is not None else None
    rw_dt = (abi.SITU_DTYPE_BF16 if rw.dtype == torch.bfloat16 else abi.SITU_DTYPE_F32) if rw is not None else 1
    dt = abi.SITU_DTYPE_BF16 if dtype == "bf16" else abi.SITU_DTYPE_F32
    data = Guarded(T, I, I + 16 * pad, torch.uint8, dev)
    scale = Guarded(T, I // 8, I // 8 + pad, torch.uint8, dev)
    amax = torch.full((1,), float("nan") if given is None else given, dtype=torch.float32, device=dev)
    want = rw is not None
    d_rw = torch.full((rw.numel(),), float("nan"), dtype=rw.dtype, device=dev) if want else None
    ws_bytes = abi.situ_glu_bwd_workspace_bytes(T, I, mode, int(want))
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    abi.check(abi.situ_glu_bwd_nvfp4(gu.data_ptr(), dt, T, I, gu.stride(0), rw_ptr, rw_dt, mode, 1, beta,
                                     int(lb is not None), float(lb or 0.0), go.data_ptr(), go.stride(0),
                                     data.ptr(), data.pitch, scale.ptr(), scale.pitch, amax.data_ptr(),
                                     int(given is not None), d_rw.data_ptr() if want else None, 1,
                                     ws.data_ptr() if ws_bytes else None, ws_bytes, 0), "bwd_nvfp4")
    torch.cuda.synchronize()
    data.check()
    scale.check()
    a = float(amax.item())
    if given is not None:
        assert a == np.float32(given), "a given tensor maximum was overwritten"
    o = oracle.load()
    if rw_h is None:
        orw, omode = np.ones(T, dtype=np.float32), oracle.RW_ROW
    else:
        orw, omode = rw_h, (oracle.RW_SCALAR if rw_h.size == 1 and T != 1 else oracle.RW_ROW)
    ref = o.bwd(gu_h, orw, go_h, beta, lb, rw_mode=omode)
    d = np.concatenate([ref.dg, ref.du], axis=1)
    rel = REL[dtype]
    tol = np.concatenate([rel * np.abs(np.nan_to_num(ref.dg)) + CANCEL * np.nan_to_num(ref.cg),
                          rel * np.abs(np.nan_to_num(ref.du))], axis=1) + 1e-30
    rep = check_nvfp4("d_gate_up", to_host(data.view), to_host(scale.view), a, d, tol, full_tensor=given is None)
    if want:
        got = to_host(d_rw)
        if mode == abi.SITU_RW_SCALAR:
            total, mag = o.dw_scalar(gu_h, go_h, beta, lb)
            check_dw("d_w (scalar)", got, np.array([total]), np.array([mag]))
        else:
            check_dw("d_w", got, ref.dw, ref.sw)
    return rep, (to_host(data.view), to_host(scale.view), a)


@pytest.mark.parametrize("dtype,T,I", SHAPES, ids=[f"{d}-{t}x{i}" for d, t, i in SHAPES])
@pytest.mark.parametrize("beta,lb,kind", COMBOS, ids=[f"b{b}-lb{l}-{k}" for b, l, k in COMBOS])
def test_nvfp4_bwd_parity(dtype, T, I, beta, lb, kind, cuda_device):
    run_nv_bwd(cuda_device, dtype, T, I, beta, lb, kind, seed=T * 7 + I)


def test_nvfp4_bwd_padded_and_given(cuda_device):
    """Padded pitches (guard bytes catch writes into the padding), and a given
    tensor maximum (twice the call's own), used and not overwritten."""
    _, (_, _, a) = run_nv_bwd(cuda_device, "bf16", 67, 256, 4.0, 25.0, "row_f32", seed=5, pad=1)
    run_nv_bwd(cuda_device, "bf16", 67, 256, 4.0, 25.0, "row_f32", seed=5, pad=1, given=2.0 * a)


def test_nvfp4_bwd_special_blocks(cuda_device):
    """A NaN gate value marks dG's and dU's blocks (0x7F) and stays out of the
    tensor maximum; a zero row has zero codes."""
    T, I = 6, 128
    g_h, _, _ = nv_inputs("bf16", T, I, seed=79)
    gu = workloads.bf16_bits_to_f32(g_h).copy()
    gu[0, 5] = np.nan
    gu[2, :] = 0.0
    bits = workloads.f32_to_bf16_bits(gu.astype(np.float32))
    _, (d, s, a) = run_nv_bwd(cuda_device, "bf16", T, I, 4.0, None, "none", seed=79, gu_h=bits)
    assert s[0, 0] == 0x7F and s[0, I // 16] == 0x7F and np.isfinite(a)
    assert not np.any(unpack_e2m1(d[2:3]) & 7)


def test_nvfp4_bwd_gates_beyond_the_signed_clamp(cuda_device):
    """Gate values below the bf16 backward's clamp at -27.75 (tiny T_g) in
    whole rows, a band, a single element, and just above it."""
    from test_gpu_mxfp8 import gates_beyond_clamp
    T, I = 8, 256
    g_h, _, _ = nv_inputs("bf16", T, I, seed=83)
    run_nv_bwd(cuda_device, "bf16", T, I, 4.0, 25.0, "row_f32", seed=83, gu_h=gates_beyond_clamp(g_h, I, 83))


def test_nvfp4_bwd_grid_invariant(cuda_device):
    outs = []
    for ctas in (0, 1, 7):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_nv_bwd(cuda_device, "bf16", 150, 1024, 4.0, 25.0, "row_f32", seed=8)[1])
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        assert np.array_equal(other[0], outs[0][0]) and np.array_equal(other[1], outs[0][1])
        assert other[2] == outs[0][2]


def test_nvfp4_bwd_tensor_api(cuda_device):
    """The tensor-level function: shapes, dtypes, the same bytes as the C-ABI
    call, the weight gradient, and decoding within NVFP4's error."""
    dev = cuda_device
    B, S, I = 2, 33, 256
    T = B * S
    g_h, rw32, go_h = nv_inputs("bf16", T, I, seed=10)
    gu = to_device(g_h, dev).reshape(B, S, 2 * I)
    rw = to_device(rw32, dev).reshape(B, S, 1)
    go = to_device(go_h, dev).reshape(B, S, I)
    d, s, a, d_rw = pkg.situ_glu_bwd_nvfp4(gu, rw, go, 4.0, 25.0)
    assert d.dtype == torch.uint8 and d.shape == (B, S, I)
    assert s.dtype == torch.float8_e4m3fn and s.shape == (B, S, 2 * I // 16)
    assert a.shape == (1,) and d_rw.shape == rw.shape
    _, (dc, sc, ac) = run_nv_bwd(dev, "bf16", T, I, 4.0, 25.0, "row_f32", seed=10)
    assert np.array_equal(d.reshape(T, -1).cpu().numpy(), dc)
    assert np.array_equal(s.view(torch.uint8).reshape(T, -1).cpu().numpy(), sc)
    assert float(a.item()) == ac
    y, unit = decode(d, s, float(a.item()))
    ref = oracle.load().bwd(g_h, rw32, go_h, 4.0, 25.0)
    r = np.concatenate([ref.dg, ref.du], axis=1).reshape(B, S, 2 * I)
    cg = np.concatenate([ref.cg, np.zeros_like(ref.du)], axis=1).reshape(B, S, 2 * I)
    assert np.all(np.abs(y - r) <= 0.25 * np.maximum(unit, np.abs(r)) * (1 + 2.0 ** -6) + 2.0 ** -10 * np.abs(r)
                  + CANCEL * cg)


def test_nvfp4_bwd_zero_tokens(cuda_device):
    gu = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda_device)
    go = torch.empty(0, 32, dtype=torch.bfloat16, device=cuda_device)
    d, s, a, _ = pkg.situ_glu_bwd_nvfp4(gu, None, go, 4.0, 25.0)
    torch.cuda.synchronize()
    assert d.shape == (0, 32) and s.shape == (0, 4) and float(a.item()) == 0.0


def test_nvfp4_bwd_routed_moe_size_sampled_rows(cuda_device):
    """32768 token rows, I = 2048, per-row weights: 48 sampled rows against the
    oracle; the tensor maximum against the kernel's own bf16 backward over
    every row (within one bf16 rounding)."""
    wl = workloads.workload(2)
    x = workloads.inputs(wl)
    T, I, beta = wl.tokens, wl.inter, wl.betas[0]
    gu = to_device(x["gate_up"], cuda_device)
    go = to_device(x["grad_out"], cuda_device)
    rw = to_device(x["routing_weights"], cuda_device).reshape(T, 1)
    d, s, a, d_rw = pkg.situ_glu_bwd_nvfp4(gu, rw, go, beta, wl.linear_beta)
    d16, _ = pkg.situ_glu_bwd(gu, rw, go, beta, wl.linear_beta)
    torch.cuda.synchronize()
    a = float(a.item())
    m16 = float(d16.float().abs().max().item())
    assert abs(a - m16) <= 2.0 ** -8 * m16, (a, m16)
    rng = np.random.default_rng(32)
    rows = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 46)]))
    ref = oracle.load().bwd(x["gate_up"], x["routing_weights"], x["grad_out"], beta, wl.linear_beta, rows=rows)
    dd = np.concatenate([ref.dg, ref.du], axis=1)
    tol = np.concatenate([2.0 ** -10 * np.abs(ref.dg) + CANCEL * ref.cg, 2.0 ** -10 * np.abs(ref.du)], axis=1) + 1e-30
    check_nvfp4("d_gate_up (sampled rows)", d[rows.tolist()].cpu().numpy(),
                s.view(torch.uint8)[rows.tolist()].cpu().numpy(), a, dd, tol, full_tensor=False)
    check_dw("d_w (sampled rows)", d_rw.reshape(-1)[rows.tolist()].cpu().numpy(), ref.dw, ref.sw)


def test_nvfp4_amax_only(cuda_device):
    """amax_given = 2 computes the tensor maximum alone (no codes, scales or
    weight gradient: their pointers are NULL) and agrees with the maximum the
    full calls compute; the sharded two-step coding (the maximum, then codes
    under a given maximum) gives the same bytes as one call."""
    dev = cuda_device
    T, I = 90, 512
    g_h, rw32, go_h = nv_inputs("bf16", T, I, seed=12)
    gu, go = to_device(g_h, dev), to_device(go_h, dev)
    rw = to_device(rw32, dev).reshape(T, 1)
    d, s, a = pkg.situ_glu_fwd_nvfp4(gu, rw, 4.0, 25.0)
    _, _, a_only = pkg.situ_glu_fwd_nvfp4(gu, rw, 4.0, 25.0, amax_only=True)
    d2, s2, _ = pkg.situ_glu_fwd_nvfp4(gu, rw, 4.0, 25.0, amax=a_only)
    bd, bs, ba, bdrw = pkg.situ_glu_bwd_nvfp4(gu, rw, go, 4.0, 25.0)
    _, _, ba_only, none = pkg.situ_glu_bwd_nvfp4(gu, rw, go, 4.0, 25.0, amax_only=True)
    bd2, bs2, _, bdrw2 = pkg.situ_glu_bwd_nvfp4(gu, rw, go, 4.0, 25.0, amax=ba_only)
    torch.cuda.synchronize()
    assert none is None
    assert float(a_only.item()) == float(a.item()) and float(ba_only.item()) == float(ba.item())
    assert torch.equal(d2, d) and torch.equal(s2.view(torch.uint8), s.view(torch.uint8))
    assert torch.equal(bd2, bd) and torch.equal(bs2.view(torch.uint8), bs.view(torch.uint8))
    assert torch.equal(bdrw2, bdrw)
