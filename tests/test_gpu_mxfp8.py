"""GPU parity of the MXFP8 outputs (situ_glu_fwd_mxfp8 / situ_glu_bwd_mxfp8)
against the fp64 oracle's values quantised by the oracle's MX block scaling
(OCP MX v1.0: E4M3 codes, one E8M0 scale per 32 elements of a row).

The kernel quantises its fp32 results; the oracle's exact values differ from
those by at most the kernel's error bound `tol` (2^-10 relative for bf16
inputs -- the forward's approximate tanh -- 1e-5 relative for fp32 inputs,
plus 2^-18 C_G for dG, the bound of the native-output tests).  Quantisation is
a monotone step function, so:

  * each block's shared exponent must lie between the oracle's exponents for
    the smallest and the largest block maximum within tol;
  * given the kernel's scale X, each code must lie between the oracle's codes
    for (ref - tol) / X and (ref + tol) / X; and at least 90 % of the codes
    must equal the oracle's code for ref / X exactly (the interval only
    absorbs values next to a rounding boundary).
A block whose oracle values hold a NaN or an infinity must carry the NaN
scale 255.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import Guarded, CANCEL, check_dw, check_mx, to_device, to_host

pytestmark = pytest.mark.gpu

REL = {"bf16": 2.0 ** -10, "f32": 1e-5}
RULES = {"ocp": oracle.MX_RULE_OCP, "ceil": oracle.MX_RULE_CEIL}


def mx_inputs(dtype: str, T: int, I: int, seed: int):
    wl = dataclasses.replace(workloads.workload(2), dtype=dtype, tokens=T, inter=I, seed=3000 + seed,
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


def oracle_rw(rw_h, T):
    if rw_h is None:
        return np.ones(T, dtype=np.float32), oracle.RW_ROW
    return rw_h, (oracle.RW_SCALAR if rw_h.size == 1 and T != 1 else oracle.RW_ROW)


def run_mx(dev, dtype, T, I, beta, lb, kind, rule, seed, pad=0, gu_h=None):
    g_h, rw32, go_h = mx_inputs(dtype, T, I, seed)
    gu_h = g_h if gu_h is None else gu_h
    rw_h, mode = rw_case(kind, rw32)
    gu, go = to_device(gu_h, dev), to_device(go_h, dev)
    rw = to_device(rw_h, dev) if rw_h is not None else None
    rw_ptr = rw.data_ptr() if rw is not None else None
    rw_dt = (abi.SITU_DTYPE_BF16 if rw.dtype == torch.bfloat16 else abi.SITU_DTYPE_F32) if rw is not None else 1
    dt = abi.SITU_DTYPE_BF16 if dtype == "bf16" else abi.SITU_DTYPE_F32
    has = int(lb is not None)
    ycodes = Guarded(T, I, I + 16 * pad, torch.uint8, dev)
    yscale = Guarded(T, I // 32, I // 32 + pad, torch.uint8, dev)
    abi.check(abi.situ_glu_fwd_mxfp8(gu.data_ptr(), dt, T, I, gu.stride(0), rw_ptr, rw_dt, mode, 1, beta, has,
                                     float(lb or 0.0), ycodes.ptr(), ycodes.pitch, yscale.ptr(), yscale.pitch,
                                     RULES[rule], 0), "fwd_mxfp8")
    dcodes = Guarded(T, 2 * I, 2 * I + 16 * pad, torch.uint8, dev)
    dscale = Guarded(T, 2 * I // 32, 2 * I // 32 + pad, torch.uint8, dev)
    want = rw is not None
    d_rw = torch.full((rw.numel(),), float("nan"), dtype=rw.dtype, device=dev) if want else None
    ws_bytes = abi.situ_glu_bwd_workspace_bytes(T, I, mode, int(want))
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    abi.check(abi.situ_glu_bwd_mxfp8(gu.data_ptr(), dt, T, I, gu.stride(0), rw_ptr, rw_dt, mode, 1, beta, has,
                                     float(lb or 0.0), go.data_ptr(), go.stride(0), dcodes.ptr(), dcodes.pitch,
                                     dscale.ptr(), dscale.pitch, RULES[rule],
                                     d_rw.data_ptr() if want else None, 1, ws.data_ptr() if ws_bytes else None,
                                     ws_bytes, 0), "bwd_mxfp8")
    torch.cuda.synchronize()
    for g in (ycodes, yscale, dcodes, dscale):
        g.check()

    o = oracle.load()
    orw, omode = oracle_rw(rw_h, T)
    rel = REL[dtype]
    y = o.fwd(gu_h, orw, beta, lb, rw_mode=omode)
    rep = {"y": check_mx("Y", to_host(ycodes.view), to_host(yscale.view), y, rel * np.abs(y) + 1e-30,
                         RULES[rule])}
    ref = o.bwd(gu_h, orw, go_h, beta, lb, rw_mode=omode)
    d = np.concatenate([ref.dg, ref.du], axis=1)
    tol = np.concatenate([rel * np.abs(ref.dg) + CANCEL * ref.cg, rel * np.abs(ref.du)], axis=1) + 1e-30
    rep["dgu"] = check_mx("d_gate_up", to_host(dcodes.view), to_host(dscale.view), d, tol, RULES[rule])
    if want:
        got = to_host(d_rw)
        if mode == abi.SITU_RW_SCALAR:
            total, mag = o.dw_scalar(gu_h, go_h, beta, lb)
            check_dw("d_w (scalar)", got, np.array([total]), np.array([mag]))
        else:
            check_dw("d_w", got, ref.dw, ref.sw)
    return rep, (to_host(ycodes.view), to_host(yscale.view), to_host(dcodes.view), to_host(dscale.view))


# I = 8192 (bf16) and 4096 (fp32) exceed two vectors per thread: the looped form.
SHAPES = [("bf16", 1, 32), ("bf16", 3, 96), ("bf16", 257, 512), ("bf16", 64, 2048), ("bf16", 40, 3072),
          ("bf16", 5, 8192), ("f32", 1, 32), ("f32", 33, 256), ("f32", 17, 4096)]
COMBOS = [(4.0, 25.0, "row_f32", "ocp"), (4.0, 25.0, "row_f32", "ceil"), (1.0, None, "row_bf16", "ocp"),
          (2.0, 1.5, "scalar", "ceil"), (16.0, None, "none", "ocp")]


@pytest.mark.parametrize("dtype,T,I", SHAPES, ids=[f"{d}-{t}x{i}" for d, t, i in SHAPES])
@pytest.mark.parametrize("beta,lb,kind,rule", COMBOS, ids=[f"b{b}-lb{l}-{k}-{r}" for b, l, k, r in COMBOS])
def test_mxfp8_parity(dtype, T, I, beta, lb, kind, rule, cuda_device):
    run_mx(cuda_device, dtype, T, I, beta, lb, kind, rule, seed=T * 3 + I)


def test_mxfp8_padded_pitches(cuda_device):
    """Row pitches above the row (code pitch +16 bytes, scale pitch +1): guard
    bytes catch any write into the padding."""
    run_mx(cuda_device, "bf16", 67, 256, 4.0, 25.0, "row_f32", "ocp", seed=5, pad=1)


@pytest.mark.parametrize("rule", ["ocp", "ceil"])
def test_mxfp8_special_blocks(rule, cuda_device):
    """NaN and infinite inputs give NaN blocks (scale 255) and leave the other
    blocks of the row alone; an all-zero row has scale byte 0; huge gate
    values saturate T_g; tiny rows use small scales."""
    T, I = 6, 128
    g_h, _, _ = mx_inputs("bf16", T, I, seed=77)
    gu = workloads.bf16_bits_to_f32(g_h).copy()
    gu[0, 5] = np.nan                 # Y[0, 5] NaN: block 0 of row 0
    gu[1, I + 40] = np.inf            # U = inf without a linear beta: Y[1, 40] infinite
    gu[2, :] = 0.0                    # Y = 0 everywhere
    gu[3, :I] = 1e30                  # T_g saturates at beta
    gu[4, :] *= np.float32(1e-30)     # tiny values
    gu[5, :I] = -np.inf               # T_g(-inf) = 0
    bits = workloads.f32_to_bf16_bits(gu.astype(np.float32))
    rep, (yc, ys, dc, ds) = run_mx(cuda_device, "bf16", T, I, 4.0, None, "none", rule, seed=77, gu_h=bits)
    assert ys[0, 0] == 255 and ys[1, 1] == 255
    assert np.all(ys[2] == 0) and not np.any(yc[2] & 0x7F)


def gates_beyond_clamp(g_bits, I, seed):
    """Gate values below -27.75, where the bf16 backward's signed form would need
    its clamp: row 0 all of them (T_g down to 1e-26: blocks that keep their own
    small scales), row 1 a band of them in the middle, row 2 one among ordinary
    values (its warp takes the |g| form, the others the signed form), row 3
    values just above the clamp."""
    gu = workloads.bf16_bits_to_f32(g_bits).copy()
    rng = np.random.default_rng(seed)
    gu[0, :I] = -rng.uniform(28.0, 60.0, I)
    gu[1, I // 4:3 * I // 4] = -rng.uniform(27.8, 40.0, I // 2)
    gu[2, 17] = -40.0
    gu[3, :I] = -rng.uniform(26.0, 27.7, I)
    return workloads.f32_to_bf16_bits(gu.astype(np.float32))


@pytest.mark.parametrize("rule", ["ocp", "ceil"])
def test_mxfp8_gates_beyond_the_signed_clamp(rule, cuda_device):
    T, I = 8, 256
    g_h, _, _ = mx_inputs("bf16", T, I, seed=81)
    run_mx(cuda_device, "bf16", T, I, 4.0, 25.0, "row_f32", rule, seed=81, gu_h=gates_beyond_clamp(g_h, I, 81))


def test_mxfp8_grid_invariant(cuda_device):
    """Codes and scales do not depend on the launch size."""
    outs = []
    for ctas in (0, 1, 7):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_mx(cuda_device, "bf16", 150, 1024, 4.0, 25.0, "row_f32", "ocp", seed=8)[1])
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert np.array_equal(a, b)


def test_mxfp8_tensor_api(cuda_device):
    """The tensor-level functions: shapes, dtypes, leading dimensions, and the
    same bytes as the C-ABI call."""
    dev = cuda_device
    B, S, I = 2, 33, 256
    T = B * S
    g_h, rw32, go_h = mx_inputs("bf16", T, I, seed=9)
    gu = to_device(g_h, dev).reshape(B, S, 2 * I)
    rw = to_device(rw32, dev).reshape(B, S, 1)
    go = to_device(go_h, dev).reshape(B, S, I)
    yd, ys = pkg.situ_glu_fwd_mxfp8(gu, rw, 4.0, 25.0, rule="ceil")
    assert yd.dtype == torch.float8_e4m3fn and yd.shape == (B, S, I)
    assert ys.dtype == torch.uint8 and ys.shape == (B, S, I // 32)
    dd, ds, d_rw = pkg.situ_glu_bwd_mxfp8(gu, rw, go, 4.0, 25.0, rule="ceil")
    assert dd.shape == (B, S, 2 * I) and ds.shape == (B, S, 2 * I // 32) and d_rw.shape == rw.shape
    _, (yc, ysc, dc, dsc) = run_mx(dev, "bf16", T, I, 4.0, 25.0, "row_f32", "ceil", seed=9)
    assert np.array_equal(yd.view(torch.uint8).reshape(T, I).cpu().numpy(), yc)
    assert np.array_equal(ys.reshape(T, -1).cpu().numpy(), ysc)
    assert np.array_equal(dd.view(torch.uint8).reshape(T, 2 * I).cpu().numpy(), dc)
    assert np.array_equal(ds.reshape(T, -1).cpu().numpy(), dsc)
    # decoding the codes with torch's own float8 type recovers Y within the MX error
    # (half an E4M3 step: 2^-4 relative for normals, 2^-10 X below 2^-6 X; plus
    # the kernel's own 2^-10 relative error)
    X = torch.exp2(ys.to(torch.float64) - 127).repeat_interleave(32, dim=-1).cpu().numpy()
    y = yd.to(torch.float64).cpu().numpy() * X
    ref = oracle.load().fwd(g_h, rw32, 4.0, 25.0).reshape(B, S, I)
    assert np.all(np.abs(y - ref) <= (2.0 ** -4 + 2.0 ** -9) * np.abs(ref) + 2.0 ** -10 * X)


def test_mxfp8_zero_tokens(cuda_device):
    gu = torch.empty(0, 64, dtype=torch.bfloat16, device=cuda_device)
    yd, ys = pkg.situ_glu_fwd_mxfp8(gu, None, 4.0, 25.0)
    assert yd.shape == (0, 32) and ys.shape == (0, 1)
