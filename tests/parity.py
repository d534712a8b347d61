"""Shared helpers of the GPU parity tests: device upload/download of the seeded
inputs, guarded output buffers, direct calls through the C ABI, and the
tolerance rule.

Tolerance rule (derived from the arithmetic; the oracle value ``ref`` is the
unrounded fp64 result):
  * bf16 outputs (Y, dG, dU): |y - ref| <= 2^-8 |ref| + 1e-6, or y is one of the
    two bf16 values that bracket ref (a faithful rounding: an fp32 chain whose
    error is far below a bf16 ulp can still round a value that sits next to a
    rounding midpoint to the other neighbour).
  * fp32 outputs (Y, dU): |y - ref| <= 1e-5 |ref| + 1e-30.
  * dG, both dtypes: the bound above plus 2^-18 * C_G, where C_G is the
    uncancelled magnitude |go w T_u| (|sech^2 sigmoid| + |beta tanh sigmoid
    (1 - sigmoid)|).  The two terms of T_g' cancel at a beta-dependent
    G* < 0 (G* = -1.21876 for beta = 4); there the fp32 rounding of each term,
    not the result, sets the error.
  * d_w: |d - ref| <= 1e-4 |ref| + 2^-18 * S, S = sum_i |go T_g T_u| (the
    rounding of a long fp32 sum scales with the sum of magnitudes).
"""
from __future__ import annotations

import json
import os
import threading

import numpy as np
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi

BF16_REL = 2.0 ** -8
BF16_ABS = 1e-6
F32_REL = 1e-5
F32_ABS = 1e-30
CANCEL = 2.0 ** -18
DW_REL = 1e-4

SENTINEL = 0xA5
GUARD_BYTES = 4096

# Where a run records what its checks found (one JSON object per line): the
# path in SITU_PARITY_REPORT, if set.  Nothing is written otherwise.
_REPORT_LOCK = threading.Lock()


def report(record: dict) -> None:
    path = os.environ.get("SITU_PARITY_REPORT")
    if not path:
        return
    with _REPORT_LOCK, open(path, "a") as f:
        f.write(json.dumps(record) + "\n")


# ---- device transfer -----------------------------------------------------------

def to_device(a: np.ndarray, device) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    """Exact copy back: bf16 as uint16 bit patterns, fp32 as float32."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def as_f64(a: np.ndarray) -> np.ndarray:
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def dtype_code(t: torch.Tensor) -> int:
    return abi.SITU_DTYPE_BF16 if t.dtype == torch.bfloat16 else abi.SITU_DTYPE_F32


# ---- guarded buffers ---------------------------------------------------------------

class Guarded:
    """An output buffer [rows, pitch] with GUARD_BYTES of sentinel bytes on each
    side; ``view`` is the [rows, width] window the kernel may write.  check()
    asserts that no byte outside the window changed (guards and row gaps)."""

    def __init__(self, rows: int, width: int, pitch: int, dtype, device):
        self.es = torch.empty((), dtype=dtype).element_size()
        g = GUARD_BYTES // self.es
        self.g, self.rows, self.width, self.pitch = g, rows, width, pitch
        self.buf = torch.empty(2 * g + max(rows * pitch, 1), dtype=dtype, device=device)
        self.buf.view(torch.uint8).fill_(SENTINEL)
        self.mat = self.buf[g:g + rows * pitch].view(rows, pitch) if rows else self.buf[g:g]
        self.view = self.mat[:, :width] if rows else self.mat

    def ptr(self) -> int:
        return self.buf[self.g:].data_ptr()

    def check(self):
        b = self.buf.view(torch.uint8)
        gb = self.g * self.es
        assert torch.all(b[:gb] == SENTINEL), "write before the output buffer"
        assert torch.all(b[gb + self.rows * self.pitch * self.es:] == SENTINEL), "write past the output buffer"
        if self.rows and self.pitch > self.width:
            gap = self.mat[:, self.width:].contiguous().view(torch.uint8)
            assert torch.all(gap == SENTINEL), "write into the row padding"


# ---- direct C-ABI calls ---------------------------------------------------------------

def call_fwd(gu: torch.Tensor, inter: int, rw, rw_mode: int, beta: float, lb, out: Guarded,
             rw_stride: int = 1, stream: int = 0) -> int:
    tokens = gu.shape[0]
    rw_ptr = rw.data_ptr() if rw is not None else None
    rw_dt = dtype_code(rw) if rw is not None else abi.SITU_DTYPE_F32
    return abi.situ_glu_fwd(gu.data_ptr(), dtype_code(gu), tokens, inter, gu.stride(0),
                            rw_ptr, rw_dt, rw_mode, rw_stride, float(beta), int(lb is not None),
                            float(lb or 0.0), out.ptr(), out.pitch, stream)


def call_bwd(gu: torch.Tensor, inter: int, rw, rw_mode: int, beta: float, lb, go: torch.Tensor,
             dgu: Guarded, d_rw=None, rw_stride: int = 1, d_rw_stride: int = 1, workspace=None,
             stream: int = 0) -> int:
    tokens = gu.shape[0]
    rw_ptr = rw.data_ptr() if rw is not None else None
    rw_dt = dtype_code(rw) if rw is not None else abi.SITU_DTYPE_F32
    ws_bytes = abi.situ_glu_bwd_workspace_bytes(tokens, inter, rw_mode, int(d_rw is not None))
    ws_ptr = None
    if ws_bytes:
        if workspace is None:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=gu.device)
        ws_ptr = workspace.data_ptr()
    return abi.situ_glu_bwd(gu.data_ptr(), dtype_code(gu), tokens, inter, gu.stride(0),
                            rw_ptr, rw_dt, rw_mode, rw_stride, float(beta), int(lb is not None),
                            float(lb or 0.0), go.data_ptr(), go.stride(0),
                            dgu.ptr(), dgu.pitch,
                            d_rw.data_ptr() if d_rw is not None else None, d_rw_stride,
                            ws_ptr, ws_bytes, stream)


# ---- tolerance ------------------------------------------------------------------------

def _bf16_key(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _bf16_from_key(k: np.ndarray) -> np.ndarray:
    return np.where(k >= 0, k, 0x8000 | (-k)).astype(np.uint16)


def bf16_faithful(bits: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """True where the bf16 value ``bits`` is one of the two bf16 neighbours of ref."""
    y = as_f64(bits)
    k = _bf16_key(bits)
    up, down = ref > y, ref < y
    toward = as_f64(_bf16_from_key(np.where(up, k + 1, np.where(down, k - 1, k))))
    return (y == ref) | (up & (toward >= ref)) | (down & (toward <= ref))


def by_row_chunks(fn, rows: np.ndarray, chunk: int = 16):
    """``fn(rows_chunk)`` -- an oracle call returning an array, or a tuple of
    arrays, with one leading entry per row -- evaluated on chunks of ``rows``
    over the host's threads (the C oracle releases the GIL) and joined in row
    order."""
    from concurrent.futures import ThreadPoolExecutor
    parts = [rows[i:i + chunk] for i in range(0, rows.size, chunk)] or [rows]
    with ThreadPoolExecutor(max_workers=max(1, min(96, os.cpu_count() or 1))) as pool:
        outs = list(pool.map(fn, parts))
    if isinstance(outs[0], tuple):
        return tuple(np.concatenate([o[k] for o in outs], axis=0) for k in range(len(outs[0])))
    return np.concatenate(outs, axis=0)


def check_ar(name, got, ref, mag):
    """The attention-residual core's output against the oracle: bf16 by the
    2^-8 relative rule (or a faithful neighbour), fp32 within 1e-5, each plus
    2^-18 of the oracle's accumulation magnitude."""
    y = as_f64(got)
    err = np.abs(y - ref)
    if got.dtype == np.uint16:
        ok = (err <= 2.0 ** -8 * np.abs(ref) + 1e-6 + 2.0 ** -18 * mag) | bf16_faithful(got, ref)
    else:
        ok = err <= 1e-5 * np.abs(ref) + 2.0 ** -18 * mag + 1e-30
    bad = np.flatnonzero(~ok)
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} of {ok.size} out of tolerance; first at flat {i}: got "
                             f"{y.flat[i]!r}, oracle {ref.flat[i]!r}, scale {mag.flat[i]!r}")


def check_output(name: str, got: np.ndarray, ref: np.ndarray, cancel_scale: np.ndarray | None = None):
    """Assert the tolerance rule elementwise.  Returns counts: ``n``;
    ``faithful_only``, the bf16 elements that pass only as a neighbour of ref;
    ``cancel_only``, the elements that pass only through the 2^-18 C_G term;
    ``extra_clause``, their sum; ``cancel_ratio_max``, the largest |ref| / C_G
    among the cancel-only elements (small: they sit where T_g' cancels); and
    ``max_rel``, the largest relative error over finite elements."""
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    y = as_f64(got)
    err = np.abs(y - ref)
    extra = CANCEL * cancel_scale if cancel_scale is not None else 0.0
    with np.errstate(invalid="ignore"):
        if got.dtype == np.uint16:
            base = BF16_REL * np.abs(ref) + BF16_ABS
            strict = err <= base
            faithful = bf16_faithful(got, ref)
        else:
            base = F32_REL * np.abs(ref) + F32_ABS
            strict = err <= base
            faithful = np.zeros_like(strict)
        cancel = err <= base + extra
        # equal values (equal infinities included) and NaN against NaN agree
        same = (y == ref) | (np.isnan(y) & np.isnan(ref))
    strict |= same
    ok = strict | faithful | cancel
    bad = np.flatnonzero(~ok)
    if bad.size:
        i = bad[0]
        cs = cancel_scale.reshape(-1)[i] if cancel_scale is not None else 0.0
        raise AssertionError(f"{name}: {bad.size} of {ok.size} elements out of tolerance; first at flat "
                             f"index {i}: got {y.reshape(-1)[i]!r}, oracle {ref.reshape(-1)[i]!r}, "
                             f"cancel scale {cs!r}")
    fin = np.isfinite(ref) & np.isfinite(y)
    rel = err[fin] / np.maximum(np.abs(ref[fin]), 1e-300)
    faithful_only = ~strict & faithful
    cancel_only = ~strict & ~faithful
    ratio = 0.0
    if cancel_scale is not None and cancel_only.any():
        cs = np.broadcast_to(cancel_scale, ref.shape)[cancel_only]
        ratio = float(np.max(np.abs(ref[cancel_only]) / np.maximum(cs, 1e-300)))
    return {"n": int(ok.size), "faithful_only": int(faithful_only.sum()), "cancel_only": int(cancel_only.sum()),
            "extra_clause": int((~strict).sum()), "cancel_ratio_max": ratio,
            "max_rel": float(np.max(rel, initial=0.0))}


def check_dw(name: str, got: np.ndarray, ref: np.ndarray, mag: np.ndarray):
    y = as_f64(got).reshape(-1)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1)
    mag = np.asarray(mag, dtype=np.float64).reshape(-1)
    tol = DW_REL * np.abs(ref) + CANCEL * mag
    if got.dtype == np.uint16:  # a bf16 weight gradient is also rounded once
        tol = tol + BF16_REL * np.abs(ref)
    bad = np.flatnonzero(~((np.abs(y - ref) <= tol) | (y == ref) | (np.isnan(y) & np.isnan(ref))))
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} of {y.size} rows out of tolerance; first row {i}: "
                             f"got {y[i]!r}, oracle {ref[i]!r}, sum |terms| {mag[i]!r}")
    strict = (np.abs(y - ref) <= DW_REL * np.abs(ref)) | (y == ref)
    loose = ~strict
    ratio = float(np.max(np.abs(ref[loose]) / np.maximum(mag[loose], 1e-300))) if loose.any() else 0.0
    return {"n": int(y.size), "extra_clause": int(loose.sum()), "cancel_ratio_max": ratio}


# ---- MXFP8 outputs ----------------------------------------------------------------------

def _exact_floor(name: str, exact: int, total: int, straddle: int, min_exact: float) -> None:
    """Codes that must equal the oracle's.  Every code already lies between the
    oracle's codes for ref -+ tol, so only the ``straddle`` codes whose interval
    holds a rounding boundary can differ at all.  The kernel's fp32 error is at
    most tol and mostly far below it, so at least ``min_exact`` of all codes
    must equal the oracle's, and at most half of the straddling ones may
    differ."""
    report({"check": name, "codes": total, "exact": exact, "straddle": straddle})
    miss = total - exact
    assert total == 0 or exact >= min_exact * total, \
        f"{name}: only {exact} of {total} codes equal the oracle's ({straddle} straddle a boundary)"
    assert miss <= straddle // 2 + 1, f"{name}: {miss} codes differ from the oracle's, of {straddle} that may"


def e4m3_key(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes in value order (sign-magnitude; both zeros equal)."""
    c = codes.astype(np.int32)
    m = c & 0x7F
    return np.where(c & 0x80, -m, m)


def check_mx(name: str, codes: np.ndarray, scales: np.ndarray, ref: np.ndarray, tol: np.ndarray, rule: int,
             min_exact: float = 0.999):
    """MXFP8 codes [R, C] and scale bytes [R, C / 32] against the oracle's
    exact values ``ref`` when the kernel's fp32 values may differ from ref by
    up to ``tol`` (elementwise).  Quantisation is monotone, so each block's
    shared exponent must lie between the oracle's exponents for the smallest
    and largest block maximum within tol, and, given the kernel's scale X, each
    code between the oracle's codes for (ref - tol) / X and (ref + tol) / X;
    at least ``min_exact`` of the codes must equal the oracle's code for
    ref / X.  Blocks holding NaN or infinity must carry scale byte 255."""
    o = oracle.load()
    R, C = ref.shape
    nb = C // 32
    assert codes.shape == (R, C) and scales.shape == (R, nb), (codes.shape, scales.shape, ref.shape)
    refb, tolb = ref.reshape(R, nb, 32), tol.reshape(R, nb, 32)
    special = ~np.isfinite(refb).all(axis=2)
    absb = np.where(np.isfinite(refb), np.abs(refb), 0.0)
    amax_lo = np.maximum(absb - tolb, 0.0).max(axis=2)
    amax_hi = (absb + tolb).max(axis=2)
    got_e = scales.astype(np.int64) - 127
    sp = np.flatnonzero(special & (scales != 255))
    assert sp.size == 0, f"{name}: block {np.unravel_index(sp[0], special.shape)} holds NaN/inf, scale {scales.flat[sp[0]]}"

    def oracle_exp(amax):
        # the oracle's shared exponent of every block maximum at once: a block
        # holding just that maximum, through the oracle's own quantiser
        m = np.zeros((R, C))
        m[:, ::32] = np.where(special, 0.0, amax)
        return o.mxfp8_quantize(m, rule)[1].astype(np.int64) - 127

    e_lo, e_hi = oracle_exp(amax_lo), oracle_exp(amax_hi)
    bad = np.flatnonzero(~special & ~((e_lo <= got_e) & (got_e <= e_hi)))
    if bad.size:
        r, b = np.unravel_index(bad[0], special.shape)
        raise AssertionError(f"{name}: {bad.size} block exponents out of range; first block ({r}, {b}) exponent "
                             f"{got_e[r, b]} outside [{e_lo[r, b]}, {e_hi[r, b]}] "
                             f"(amax {amax_lo[r, b]}..{amax_hi[r, b]})")
    Xe = np.repeat(np.exp2(np.where(scales == 255, 0, got_e).astype(np.float64)), 32, axis=1)
    fin = np.repeat(~special, 32, axis=1) & np.isfinite(ref)
    with np.errstate(invalid="ignore"):
        lo = e4m3_key(o.e4m3_encode((ref - tol) / Xe))
        hi = e4m3_key(o.e4m3_encode((ref + tol) / Xe))
        mid = e4m3_key(o.e4m3_encode(ref / Xe))
    g = e4m3_key(codes)
    bad = np.flatnonzero(fin & ~((lo <= g) & (g <= hi)))
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} codes out of range; first at flat {i}: code {codes.flat[i]:#x}, "
                             f"oracle value {ref.flat[i]!r} / X {Xe.flat[i]!r}, allowed keys "
                             f"[{lo.flat[i]}, {hi.flat[i]}]")
    exact, total = int(np.sum(fin & (g == mid))), int(np.sum(fin))
    straddle = int(np.sum(fin & (lo != hi)))
    _exact_floor(name, exact, total, straddle, min_exact)
    return {"codes": total, "exact": exact, "straddle": straddle}


# ---- NVFP4 outputs ----------------------------------------------------------------------

def e2m1_key(codes: np.ndarray) -> np.ndarray:
    """E2M1 codes (one per byte) in value order (sign-magnitude; both zeros equal)."""
    c = codes.astype(np.int32)
    m = c & 0x7
    return np.where(c & 0x8, -m, m)


def unpack_e2m1(packed: np.ndarray) -> np.ndarray:
    """[R, C / 2] bytes -> [R, C] codes, element 2k from the low nibble of byte k."""
    p = packed.astype(np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


# The kernel forms S_enc, the block-scale argument and the element ratio in
# fp32 (a few roundings of 2^-24 each): they may sit this far (relative) from
# the oracle's fp64 values.
NVFP4_SLACK = 2.0 ** -20


def check_nvfp4(name: str, packed: np.ndarray, scales: np.ndarray, amax: float, ref: np.ndarray, tol: np.ndarray,
                min_exact: float = 0.999, full_tensor: bool = True):
    """NVFP4 codes (packed [R, C / 2]), E4M3 block scales [R, C / 16] and the
    tensor maximum ``amax`` the kernel used, against the oracle's exact values
    ``ref`` [R, C] when the kernel's fp32 values may differ from ref by up to
    ``tol``.  ``amax`` must lie within the bounds the oracle's values allow
    (max |ref| -+ tol, when ``ref`` holds the whole tensor, else at least the
    lower bound); with S = 2688 / amax, each block scale must lie between the
    oracle's E4M3 codes for the smallest and the largest block maximum within
    tol, times S / 6; given the kernel's block scale s, each code between the
    oracle's E2M1 codes for (ref -+ tol) S / s; and at least ``min_exact`` of
    the codes equal the oracle's code of ref S / s (oracle.nvfp4_quantize with
    the same S, on the rows it covers).  Blocks holding NaN or infinity must
    carry scale code 0x7F; a block whose scale decodes to 0 must hold only zero
    codes."""
    o = oracle.load()
    R, C = ref.shape
    nb = C // 16
    codes = unpack_e2m1(packed)
    assert codes.shape == (R, C) and scales.shape == (R, nb), (codes.shape, scales.shape, ref.shape)
    fin_all = np.isfinite(ref)
    absr = np.where(fin_all, np.abs(ref), 0.0)
    a_lo = float(np.maximum(absr - tol, 0.0).max()) if ref.size else 0.0
    a_hi = float((absr + tol).max()) if ref.size else 0.0
    assert amax >= a_lo * (1 - NVFP4_SLACK), f"{name}: amax {amax!r} below the oracle's lower bound {a_lo!r}"
    if full_tensor:
        assert amax <= a_hi * (1 + NVFP4_SLACK), f"{name}: amax {amax!r} above the oracle's upper bound {a_hi!r}"
    s = o.nvfp4_tensor_scale(amax)
    refb, tolb = ref.reshape(R, nb, 16), tol.reshape(R, nb, 16)
    special = ~np.isfinite(refb).all(axis=2)
    absb = np.where(np.isfinite(refb), np.abs(refb), 0.0)
    bmax_lo = np.maximum(absb - tolb, 0.0).max(axis=2) * s / 6.0 * (1 - NVFP4_SLACK)
    bmax_hi = (absb + tolb).max(axis=2) * s / 6.0 * (1 + NVFP4_SLACK)
    k_lo, k_hi = e4m3_key(o.e4m3_encode(bmax_lo)), e4m3_key(o.e4m3_encode(bmax_hi))
    k = e4m3_key(scales)
    sp = np.flatnonzero(special & (scales != 0x7F))
    assert sp.size == 0, f"{name}: block {np.unravel_index(sp[0], special.shape)} holds NaN/inf, scale {scales.flat[sp[0]]:#x}"
    bad = np.flatnonzero(~special & ~((k_lo <= k) & (k <= k_hi)))
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} block scales out of range; first block {np.unravel_index(i, k.shape)}: "
                             f"code {scales.flat[i]:#x}, allowed keys [{k_lo.flat[i]}, {k_hi.flat[i]}]")
    sb = np.where(special, 0.0, o.e4m3_decode(np.where(special, 0, scales)))
    sbe = np.repeat(sb, 16, axis=1)
    use = np.repeat(~special, 16, axis=1) & fin_all
    zero_blk = use & (sbe == 0.0)
    zb = np.flatnonzero(zero_blk & (e2m1_key(codes) != 0))
    assert zb.size == 0, f"{name}: a block with scale 0 holds a nonzero code at flat {zb[0]}"
    live = use & (sbe > 0.0)
    ratio = np.where(live, s / np.where(sbe > 0.0, sbe, 1.0), 0.0)
    with np.errstate(invalid="ignore"):
        x_lo, x_hi = (ref - tol) * ratio, (ref + tol) * ratio
        lo = e2m1_key(o.e2m1_encode(np.where(live, x_lo - np.abs(x_lo) * NVFP4_SLACK, 0.0)))
        hi = e2m1_key(o.e2m1_encode(np.where(live, x_hi + np.abs(x_hi) * NVFP4_SLACK, 0.0)))
    oc, osc, _ = o.nvfp4_quantize(np.where(fin_all, ref, np.nan), s_enc=s)
    g = e2m1_key(codes)
    bad = np.flatnonzero(live & ~((lo <= g) & (g <= hi)))
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} codes out of range; first at flat {i}: code {codes.flat[i]:#x}, "
                             f"oracle value {ref.flat[i]!r} x {ratio.flat[i]!r}, allowed keys "
                             f"[{lo.flat[i]}, {hi.flat[i]}]")
    same_scale = np.repeat(osc == scales, 16, axis=1)
    exact = int(np.sum(live & same_scale & (g == e2m1_key(oc))))
    total = int(np.sum(live))
    # a code may differ from the oracle's where its interval holds a rounding
    # boundary, or where the block scale itself may differ
    k_straddle = np.repeat(k_lo != k_hi, 16, axis=1)
    straddle = int(np.sum(live & ((lo != hi) | k_straddle | ~same_scale)))
    _exact_floor(name, exact, total, straddle, min_exact)
    return {"codes": total, "exact": exact, "straddle": straddle,
            "scales_equal": float(np.mean(osc == scales)) if osc.size else 1.0}
