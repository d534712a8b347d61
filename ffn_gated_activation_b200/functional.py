"""Tensor-level binding: marshals torch tensors into the C ABI of libsitu_glu.so.

PyTorch supplies device memory and the current stream; every step of the
computation runs in the library's kernels.  The autograd function follows the
contract of NeMo AutoModel's kimi_k3.situ `_WeightedSiTUFunction`: the forward
saves only the low-precision inputs (gate_up and routing_weights in their own
dtypes), the backward recomputes the fp32 chain and returns
(d_gate_up, d_routing_weights or None, None, None).
"""
from __future__ import annotations

import math

import torch

from . import abi

# Kimi-K3 defaults (Megatron-LM PR #6673, "Activation": beta1 = 4, beta2 = 25;
# the Kimi-K3 config.json: activation_situ_beta 4.0, activation_situ_linear_beta 25.0).
DEFAULT_BETA = 4.0
DEFAULT_LINEAR_BETA = 25.0

_DTYPES = {torch.bfloat16: abi.SITU_DTYPE_BF16, torch.float32: abi.SITU_DTYPE_F32}


def _dtype_code(t: torch.Tensor, what: str) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"{what} must be bfloat16 or float32, got {t.dtype}") from None


def _check_beta(beta, linear_beta):
    # Megatron-LM PR #6673 "Design": SiTU-GLU betas must be finite and positive.
    if not (isinstance(beta, (int, float)) and math.isfinite(beta) and beta > 0):
        raise ValueError(f"beta must be a finite positive number, got {beta!r}")
    if linear_beta is not None and not (isinstance(linear_beta, (int, float))
                                        and math.isfinite(linear_beta) and linear_beta > 0):
        raise ValueError(f"linear_beta must be None or a finite positive number, got {linear_beta!r}")


def _rows(gate_up: torch.Tensor):
    """gate_up [..., 2I] -> (2-D view [T, 2I], leading shape, I)."""
    if gate_up.device.type != "cuda":
        raise ValueError("gate_up must be a CUDA tensor")
    if gate_up.dim() < 1 or gate_up.shape[-1] % 2:
        raise ValueError(f"gate_up's last dimension must be 2 * intermediate, got {tuple(gate_up.shape)}")
    inter = gate_up.shape[-1] // 2
    lead = tuple(gate_up.shape[:-1])
    g2 = gate_up if gate_up.dim() == 2 else gate_up.reshape(-1, 2 * inter)  # 2-D: no view to build
    if g2.stride(1) != 1 or (g2.shape[0] > 1 and g2.stride(0) < 2 * inter):
        g2 = g2.contiguous()
    return g2, lead, inter


def _given(t: torch.Tensor, shape: tuple, device, what: str, dtype=None) -> torch.Tensor:
    """A caller's output buffer, checked before the library writes to it (the
    library sees a pointer and a row pitch only, so a smaller or strided
    buffer would be written past): exactly ``shape``, ``dtype`` (None: any
    one-byte dtype, for code and scale bytes), on ``device``, elements of a
    row adjacent and rows apart by at least a row.  Returns the 2-D view
    [rows, shape[-1]] the library is given."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what} shape {tuple(t.shape)} != {tuple(shape)}")
    if (t.element_size() != 1) if dtype is None else (t.dtype != dtype):
        raise TypeError(f"{what} must be {dtype if dtype is not None else 'a one-byte dtype'}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{what} must be on {device}, got {t.device}")
    cols = shape[-1]
    try:
        t2 = t if t.dim() == 2 else t.view(-1, cols)  # a view or nothing: never a copy
    except RuntimeError:
        raise ValueError(f"{what} must be viewable as [rows, {cols}]") from None
    if t2.numel() and (t2.stride(1) != 1 or (t2.shape[0] > 1 and t2.stride(0) < cols)):
        raise ValueError(f"{what} must hold each row's elements adjacent, rows not overlapping")
    return t2


def _given_drw(d_rw: torch.Tensor, routing_weights: torch.Tensor, device) -> torch.Tensor:
    """A caller's routing-weight gradient buffer: the weights' shape and dtype."""
    if tuple(d_rw.shape) != tuple(routing_weights.shape) or d_rw.dtype != routing_weights.dtype:
        raise ValueError(f"d_rw must have routing_weights' shape {tuple(routing_weights.shape)} and dtype "
                         f"{routing_weights.dtype}, got {tuple(d_rw.shape)} {d_rw.dtype}")
    if d_rw.device != device:
        raise ValueError(f"d_rw must be on {device}, got {d_rw.device}")
    return d_rw


def routing_mode(gate_up_lead: tuple, inter: int, routing_weights):
    """Classify routing_weights against the output [*lead, inter] the way
    broadcasting aligns them (NeMo `_situ_rw_is_row_aligned` and
    `_WeightedSiTUFunction.forward`, parameter routing_weights).  Returns
    (mode, view, stride): the C-ABI mode, the tensor the library reads, and
    its element stride (rows for row-aligned and full weights).

    None -> unweighted; one element -> broadcast scalar; [*lead, 1] ->
    row-aligned; inter elements along the last axis ([I], [1, I], ...) -> one
    weight per column; [*lead, I] -> one weight per element."""
    if routing_weights is None:
        return abi.SITU_RW_NONE, None, 1
    rw = routing_weights
    if rw.numel() == 1:
        return abi.SITU_RW_SCALAR, rw.reshape(1), 1
    if rw.dim() == 2 and len(gate_up_lead) == 1 and rw.shape[0] == gate_up_lead[0] and rw.shape[1] == 1:
        return abi.SITU_RW_ROW, rw, rw.stride(0)  # [T, 1]: row r at rw.stride(0) * r, as in its flat view
    if rw.dim() == len(gate_up_lead) + 1 and tuple(rw.shape[:-1]) == gate_up_lead and rw.shape[-1] == 1:
        flat = rw.reshape(-1)
        return abi.SITU_RW_ROW, flat, flat.stride(0) if flat.numel() > 1 else 1
    if rw.dim() >= 1 and rw.shape[-1] == inter and rw.numel() == inter:
        return abi.SITU_RW_COL, rw.reshape(inter).contiguous(), 1
    if tuple(rw.shape) == tuple(gate_up_lead) + (inter,):
        w2 = rw.reshape(-1, inter)
        if w2.stride(1) != 1 or (w2.shape[0] > 1 and w2.stride(0) < inter):
            w2 = w2.contiguous()
        return abi.SITU_RW_FULL, w2, w2.stride(0) if w2.shape[0] > 1 else inter
    raise NotImplementedError(
        f"routing_weights of shape {tuple(rw.shape)} do not broadcast to the output {gate_up_lead + (inter,)} "
        "as one of: [..., 1] (per row), one value, [I] (per column), [..., I] (per element)")


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def situ_glu_fwd(gate_up: torch.Tensor, routing_weights, beta: float = DEFAULT_BETA,
                 linear_beta: float | None = DEFAULT_LINEAR_BETA, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Y = T_g(G) * T_u(U) * w for gate_up [..., 2I]; returns [..., I] in gate_up's dtype."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    if rw is not None:
        if rw.device != g2.device:
            raise ValueError("routing_weights must be on gate_up's device")
        rw_dtype = _dtype_code(rw, "routing_weights")
    else:
        rw_dtype = abi.SITU_DTYPE_F32
    if out is None:
        out = torch.empty(lead + (inter,), dtype=gate_up.dtype, device=gate_up.device)
        o2 = out if out.dim() == 2 else out.view(-1, inter)
    else:
        o2 = _given(out, lead + (inter,), gate_up.device, "out", gate_up.dtype)
    tokens = g2.shape[0]
    st = abi.situ_glu_fwd(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                          rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                          float(beta), int(linear_beta is not None),
                          float(linear_beta) if linear_beta is not None else 0.0,
                          o2.data_ptr(), o2.stride(0) if tokens > 1 else inter, _stream_handle(stream))
    abi.check(st, "situ_glu_fwd")
    return out


def situ_glu_bwd(gate_up: torch.Tensor, routing_weights, grad_out: torch.Tensor,
                 beta: float = DEFAULT_BETA, linear_beta: float | None = DEFAULT_LINEAR_BETA,
                 want_drw: bool = True, d_gate_up: torch.Tensor | None = None,
                 d_rw: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 stream=None):
    """Analytic backward.  Returns (d_gate_up [..., 2I], d_routing_weights shaped
    like routing_weights, or None when not wanted / unweighted)."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    if grad_out.dtype != gate_up.dtype:
        raise TypeError("grad_out must have gate_up's dtype")
    if tuple(grad_out.shape) != lead + (inter,):
        raise ValueError(f"grad_out shape {tuple(grad_out.shape)} != {lead + (inter,)}")
    go2 = grad_out if grad_out.dim() == 2 else grad_out.reshape(-1, inter)
    if go2.stride(1) != 1 or (go2.shape[0] > 1 and go2.stride(0) < inter):
        go2 = go2.contiguous()
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    want = bool(want_drw) and rw is not None
    if d_gate_up is None:
        d_gate_up = torch.empty(lead + (2 * inter,), dtype=gate_up.dtype, device=gate_up.device)
        dg2 = d_gate_up if d_gate_up.dim() == 2 else d_gate_up.view(-1, 2 * inter)
    else:
        dg2 = _given(d_gate_up, lead + (2 * inter,), gate_up.device, "d_gate_up", gate_up.dtype)
    d_rw_flat, d_rw_stride = None, 1
    if want:
        if d_rw is None:
            d_rw = torch.empty(routing_weights.shape, dtype=routing_weights.dtype, device=gate_up.device)
        else:
            _given_drw(d_rw, routing_weights, gate_up.device)
        if mode == abi.SITU_RW_FULL:
            d_rw_flat = d_rw.view(-1, inter)
            d_rw_stride = d_rw_flat.stride(0) if d_rw_flat.shape[0] > 1 else inter
        elif d_rw.dim() == 2 and d_rw.shape[1] == 1 and d_rw.shape[0] > 1:
            d_rw_flat, d_rw_stride = d_rw, d_rw.stride(0)  # [T, 1]: as its flat view
        else:
            d_rw_flat = d_rw.view(-1)
            d_rw_stride = d_rw_flat.stride(0) if d_rw_flat.numel() > 1 else 1
    tokens = g2.shape[0]
    # Only a broadcast or per-column weight's gradient takes scratch.
    ws_bytes = (abi.situ_glu_bwd_workspace_bytes(tokens, inter, mode, int(want))
                if want and mode in (abi.SITU_RW_SCALAR, abi.SITU_RW_COL) else 0)
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=gate_up.device)
    st = abi.situ_glu_bwd(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                          rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                          float(beta), int(linear_beta is not None),
                          float(linear_beta) if linear_beta is not None else 0.0,
                          go2.data_ptr(), go2.stride(0) if tokens > 1 else inter,
                          dg2.data_ptr(), dg2.stride(0) if tokens > 1 else 2 * inter,
                          d_rw_flat.data_ptr() if d_rw_flat is not None else None, d_rw_stride,
                          workspace.data_ptr() if ws_bytes else None, ws_bytes,
                          _stream_handle(stream))
    abi.check(st, "situ_glu_bwd")
    return d_gate_up, (d_rw if want else None)


_MX_RULES = {"ocp": abi.SITU_MX_RULE_OCP, "ceil": abi.SITU_MX_RULE_CEIL}


def _mx_rule(rule) -> int:
    if isinstance(rule, str):
        try:
            return _MX_RULES[rule]
        except KeyError:
            raise ValueError(f"rule must be one of {sorted(_MX_RULES)}, got {rule!r}") from None
    return int(rule)


def _mx_buffers(lead: tuple, cols: int, device, data=None, scale=None):
    """E4M3 codes [..., cols] (torch.float8_e4m3fn) and E8M0 scale bytes
    [..., cols / 32] (torch.uint8), allocated when not given; returns the two
    tensors and their 2-D byte views."""
    if data is None:
        data = torch.empty(lead + (cols,), dtype=torch.float8_e4m3fn, device=device)
        d2 = data.view(-1, cols)
    else:
        d2 = _given(data, lead + (cols,), device, "MXFP8 data")
    if scale is None:
        scale = torch.empty(lead + (cols // 32,), dtype=torch.uint8, device=device)
        s2 = scale.view(-1, cols // 32)
    else:
        s2 = _given(scale, lead + (cols // 32,), device, "MXFP8 scale")
    return data, scale, d2, s2


def situ_glu_fwd_mxfp8(gate_up: torch.Tensor, routing_weights, beta: float = DEFAULT_BETA,
                       linear_beta: float | None = DEFAULT_LINEAR_BETA, rule="ocp", data=None, scale=None,
                       stream=None):
    """Forward with an MXFP8 Y (OCP MX v1.0: E4M3 codes, one E8M0 scale per 32
    elements of a row).  Returns (codes [..., I] as torch.float8_e4m3fn,
    scale bytes [..., I / 32] as torch.uint8).  rule: "ocp" (shared exponent
    floor(log2 amax) - 8, elements clamped to +-448) or "ceil" (smallest
    exponent with no clamping).  I must be a multiple of 32; routing weights
    per row, broadcast, or None."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    data, scale, d2, s2 = _mx_buffers(lead, inter, gate_up.device, data, scale)
    tokens = g2.shape[0]
    st = abi.situ_glu_fwd_mxfp8(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                                rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                                float(beta), int(linear_beta is not None),
                                float(linear_beta) if linear_beta is not None else 0.0,
                                d2.data_ptr(), d2.stride(0) if tokens > 1 else inter,
                                s2.data_ptr(), s2.stride(0) if tokens > 1 else inter // 32,
                                _mx_rule(rule), _stream_handle(stream))
    abi.check(st, "situ_glu_fwd_mxfp8")
    return data, scale


def situ_glu_bwd_mxfp8(gate_up: torch.Tensor, routing_weights, grad_out: torch.Tensor,
                       beta: float = DEFAULT_BETA, linear_beta: float | None = DEFAULT_LINEAR_BETA,
                       rule="ocp", want_drw: bool = True, data=None, scale=None, d_rw=None, workspace=None,
                       stream=None):
    """Backward with an MXFP8 d_gate_up: returns (codes [..., 2I] as
    torch.float8_e4m3fn with dG then dU, scale bytes [..., 2I / 32],
    d_routing_weights or None).  Same rules and restrictions as
    situ_glu_fwd_mxfp8; the weight gradient is as in situ_glu_bwd."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    if grad_out.dtype != gate_up.dtype:
        raise TypeError("grad_out must have gate_up's dtype")
    if tuple(grad_out.shape) != lead + (inter,):
        raise ValueError(f"grad_out shape {tuple(grad_out.shape)} != {lead + (inter,)}")
    go2 = grad_out if grad_out.dim() == 2 else grad_out.reshape(-1, inter)
    if go2.stride(1) != 1 or (go2.shape[0] > 1 and go2.stride(0) < inter):
        go2 = go2.contiguous()
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    want = bool(want_drw) and rw is not None
    data, scale, d2, s2 = _mx_buffers(lead, 2 * inter, gate_up.device, data, scale)
    d_rw_flat, d_rw_stride = None, 1
    if want:
        if d_rw is None:
            d_rw = torch.empty(routing_weights.shape, dtype=routing_weights.dtype, device=gate_up.device)
        else:
            _given_drw(d_rw, routing_weights, gate_up.device)
        d_rw_flat = d_rw.view(-1)
        d_rw_stride = d_rw_flat.stride(0) if d_rw_flat.numel() > 1 else 1
    tokens = g2.shape[0]
    ws_bytes = abi.situ_glu_bwd_workspace_bytes(tokens, inter, mode, int(want))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=gate_up.device)
    st = abi.situ_glu_bwd_mxfp8(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                                rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                                float(beta), int(linear_beta is not None),
                                float(linear_beta) if linear_beta is not None else 0.0,
                                go2.data_ptr(), go2.stride(0) if tokens > 1 else inter,
                                d2.data_ptr(), d2.stride(0) if tokens > 1 else 2 * inter,
                                s2.data_ptr(), s2.stride(0) if tokens > 1 else 2 * inter // 32,
                                _mx_rule(rule), d_rw_flat.data_ptr() if d_rw_flat is not None else None,
                                d_rw_stride, workspace.data_ptr() if ws_bytes else None, ws_bytes,
                                _stream_handle(stream))
    abi.check(st, "situ_glu_bwd_mxfp8")
    return data, scale, (d_rw if want else None)


def situ_glu_fc1_fwd(x: torch.Tensor, w1: torch.Tensor, offsets: torch.Tensor, routing_weights=None,
                     beta: float = DEFAULT_BETA, linear_beta: float | None = DEFAULT_LINEAR_BETA,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """FC1 grouped GEMM with the SiTU-GLU epilogue (Megatron-LM PR #6673
    "Design": the fused grouped GEMM + SiTU-GLU).

    x: bf16 [T, H] token rows grouped by expert; w1: bf16 [E, 2I, H] (or
    [E * 2I, H]) -- per expert I gate rows then I up rows; offsets: int64
    [E + 1] on x's device, rows of expert e = [offsets[e], offsets[e+1]);
    routing_weights: [T, 1] / [T] per row, one value, or None.  Returns bf16
    Y [T, I]; rows outside every expert are left as they are in ``out``
    (uninitialised when out is None)."""
    _check_beta(beta, linear_beta)
    if x.dtype != torch.bfloat16 or w1.dtype != torch.bfloat16:
        raise TypeError("x and w1 must be bfloat16")
    if x.device.type != "cuda" or w1.device != x.device or offsets.device != x.device:
        raise ValueError("x, w1 and offsets must be on the same CUDA device")
    if offsets.dtype != torch.int64 or offsets.dim() != 1:
        raise TypeError("offsets must be a 1-D int64 tensor")
    experts = offsets.numel() - 1
    if x.dim() != 2:
        raise ValueError("x must be [tokens, hidden]")
    tokens, hidden = x.shape
    w2 = w1.reshape(-1, w1.shape[-1])
    if w2.shape[1] != hidden or w2.shape[0] % (2 * experts):
        raise ValueError(f"w1 {tuple(w1.shape)} does not match {experts} experts of hidden size {hidden}")
    inter = w2.shape[0] // (2 * experts)
    if x.stride(1) != 1:
        x = x.contiguous()
    if w2.stride(1) != 1:
        w2 = w2.contiguous()
    mode, rw, rw_stride = routing_mode((tokens,), inter, routing_weights)
    if mode in (abi.SITU_RW_COL, abi.SITU_RW_FULL):
        raise NotImplementedError("situ_glu_fc1_fwd takes per-row, broadcast or no routing weights")
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    if out is None:
        out = torch.empty(tokens, inter, dtype=torch.bfloat16, device=x.device)
    else:
        _given(out, (tokens, inter), x.device, "out", torch.bfloat16)
    st = abi.situ_glu_fc1_fwd(x.data_ptr(), tokens, hidden, x.stride(0) if tokens > 1 else hidden,
                              w2.data_ptr(), experts, inter, w2.stride(0), offsets.data_ptr(),
                              rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                              float(beta), int(linear_beta is not None),
                              float(linear_beta) if linear_beta is not None else 0.0,
                              out.data_ptr(), out.stride(0) if tokens > 1 else inter, _stream_handle(stream))
    abi.check(st, "situ_glu_fc1_fwd")
    return out


def situ_glu_fc2_dgrad_bwd(dout: torch.Tensor, w2t: torch.Tensor, offsets: torch.Tensor, gate_up: torch.Tensor,
                           routing_weights=None, beta: float = DEFAULT_BETA,
                           linear_beta: float | None = DEFAULT_LINEAR_BETA, want_drw: bool = True,
                           d_gate_up=None, d_rw=None, workspace=None, stream=None):
    """FC2 data gradient fused with the SiTU-GLU backward.  dout: bf16 [T, H];
    w2t: bf16 [E, I, H] (or [E * I, H]) -- FC2's weight transposed per expert;
    offsets: int64 [E + 1] on dout's device; gate_up: the saved bf16 [T, 2I];
    routing_weights: per-row [T, 1] / [T] or None.  Returns (d_gate_up [T, 2I],
    d_routing_weights shaped like routing_weights, or None)."""
    _check_beta(beta, linear_beta)
    for t, name in ((dout, "dout"), (w2t, "w2t"), (gate_up, "gate_up")):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    if dout.dim() != 2 or gate_up.dim() != 2:
        raise ValueError("dout and gate_up must be 2-D")
    tokens, hidden = dout.shape
    inter = gate_up.shape[1] // 2
    experts = offsets.numel() - 1
    w2 = w2t.reshape(-1, w2t.shape[-1])
    if w2.shape != (experts * inter, hidden):
        raise ValueError(f"w2t {tuple(w2t.shape)} does not match {experts} experts x {inter} x {hidden}")
    dout = dout if dout.stride(1) == 1 else dout.contiguous()
    w2 = w2 if w2.stride(1) == 1 else w2.contiguous()
    gate_up = gate_up if gate_up.stride(1) == 1 else gate_up.contiguous()
    mode, rw, rw_stride = routing_mode((tokens,), inter, routing_weights)
    if mode not in (abi.SITU_RW_ROW, abi.SITU_RW_NONE):
        raise NotImplementedError("situ_glu_fc2_dgrad_bwd takes per-row or no routing weights")
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    want = bool(want_drw) and rw is not None
    if d_gate_up is None:
        d_gate_up = torch.empty(tokens, 2 * inter, dtype=torch.bfloat16, device=dout.device)
    else:
        _given(d_gate_up, (tokens, 2 * inter), dout.device, "d_gate_up", torch.bfloat16)
    d_rw_flat = None
    if want:
        if d_rw is None:
            d_rw = torch.empty(routing_weights.shape, dtype=routing_weights.dtype, device=dout.device)
        else:
            _given_drw(d_rw, routing_weights, dout.device)
        d_rw_flat = d_rw.view(-1)
    ws = abi.situ_glu_fc2_dgrad_workspace_bytes(tokens, inter, int(want))
    if ws and (workspace is None or workspace.numel() * workspace.element_size() < ws):
        workspace = torch.empty(ws, dtype=torch.uint8, device=dout.device)
    st = abi.situ_glu_fc2_dgrad_bwd(dout.data_ptr(), tokens, hidden, dout.stride(0) if tokens > 1 else hidden,
                                    w2.data_ptr(), experts, inter, w2.stride(0), offsets.data_ptr(),
                                    gate_up.data_ptr(), gate_up.stride(0) if tokens > 1 else 2 * inter,
                                    rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                                    float(beta), int(linear_beta is not None),
                                    float(linear_beta) if linear_beta is not None else 0.0,
                                    d_gate_up.data_ptr(), d_gate_up.stride(0) if tokens > 1 else 2 * inter,
                                    d_rw_flat.data_ptr() if d_rw_flat is not None else None,
                                    d_rw_flat.stride(0) if d_rw_flat is not None and d_rw_flat.numel() > 1 else 1,
                                    workspace.data_ptr() if ws else None, ws, _stream_handle(stream))
    abi.check(st, "situ_glu_fc2_dgrad_bwd")
    return d_gate_up, (d_rw if want else None)


_DTYPE_OF = {torch.bfloat16: abi.SITU_DTYPE_BF16, torch.float32: abi.SITU_DTYPE_F32}


def _attn_res_launch(blocks, prefix, norm_weight, proj_weight, variance_epsilon, out_dtype, out):
    src = blocks if blocks is not None else prefix
    if src.device.type != "cuda":
        raise ValueError("the sources must be CUDA tensors")
    dtype = _dtype_code(src, "values")
    if blocks is not None and prefix is not None and blocks.dtype != prefix.dtype:
        raise TypeError("block_residual and prefix_sum must share a dtype")
    tokens, hidden = src.shape[0], src.shape[-1]
    nw = norm_weight.reshape(-1)
    pw = proj_weight.reshape(-1)
    if nw.numel() != hidden or pw.numel() != hidden:
        raise ValueError(f"norm_weight and proj_weight must hold {hidden} values")
    nw, pw = nw.contiguous(), pw.contiguous()
    out_dtype = src.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty(tokens, hidden, dtype=out_dtype, device=src.device)
    else:
        _given(out, (tokens, hidden), src.device, "out", out.dtype)
    nb = 0
    if blocks is not None:
        if blocks.stride(-1) != 1:
            blocks = blocks.contiguous()
        nb = blocks.shape[1]
    if prefix is not None and prefix.stride(-1) != 1:
        prefix = prefix.contiguous()
    st = abi.situ_attn_res_fwd(blocks.data_ptr() if blocks is not None else None, nb,
                               blocks.stride(0) if blocks is not None else hidden,
                               blocks.stride(1) if blocks is not None else hidden,
                               prefix.data_ptr() if prefix is not None else None,
                               prefix.stride(0) if prefix is not None else hidden, dtype, tokens, hidden,
                               nw.data_ptr(), _dtype_code(nw, "norm_weight"), pw.data_ptr(),
                               _dtype_code(pw, "proj_weight"), float(variance_epsilon), out.data_ptr(),
                               _dtype_code(out, "out"), out.stride(0) if tokens > 1 else hidden,
                               _stream_handle(None))
    abi.check(st, "situ_attn_res_fwd")
    return out


def attn_res_core(values: torch.Tensor, norm_weight: torch.Tensor, proj_weight: torch.Tensor,
                  variance_epsilon: float, out_dtype: torch.dtype | None = None, out=None) -> torch.Tensor:
    """NeMo `_attn_res_core`: fp32 attention-residual mixing of values
    [tokens, sources, hidden] (block residuals with the current prefix sum
    appended) -> [tokens, hidden] in out_dtype (default: values' dtype)."""
    if values.dim() != 3:
        raise ValueError("values must be [tokens, sources, hidden]")
    return _attn_res_launch(values, None, norm_weight, proj_weight, variance_epsilon, out_dtype, out)


def apply_attn_res(prefix_sum: torch.Tensor, block_residual: torch.Tensor, proj_weight: torch.Tensor,
                   norm_weight: torch.Tensor, variance_epsilon: float, out_dtype: torch.dtype | None = None,
                   out=None) -> torch.Tensor:
    """NeMo `_apply_attn_res`: mix prefix_sum [tokens, hidden] with the stored
    block_residual [tokens, blocks, hidden] without stacking them (the prefix
    sum is the last source)."""
    if prefix_sum.dim() != 2 or block_residual.dim() != 3:
        raise ValueError("prefix_sum must be [tokens, hidden] and block_residual [tokens, blocks, hidden]")
    return _attn_res_launch(block_residual, prefix_sum, norm_weight, proj_weight, variance_epsilon, out_dtype, out)


def situ_glu_fwd_nvfp4(gate_up: torch.Tensor, routing_weights, beta: float = DEFAULT_BETA,
                       linear_beta: float | None = DEFAULT_LINEAR_BETA, amax: torch.Tensor | None = None,
                       data=None, scale=None, amax_out: torch.Tensor | None = None, amax_only: bool = False,
                       stream=None):
    """Forward with an NVFP4 Y: returns (packed E2M1 codes [..., I / 2] uint8,
    E4M3 block scales [..., I / 16] as torch.float8_e4m3fn, amax: a 1-element
    fp32 tensor holding the tensor maximum A).  Pass ``amax`` (1 element, on
    gate_up's device) to use a known A instead of computing it; otherwise A is
    computed into ``amax_out`` (allocated when None).  ``amax_only``: compute
    A alone and return (None, None, amax).  Decode code q of block b as
    q * scale_b * A / 2688."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    if amax_only and amax is not None:
        raise ValueError("amax_only computes the tensor maximum: do not pass one")
    if not amax_only:
        if data is None:
            data = torch.empty(lead + (inter // 2,), dtype=torch.uint8, device=gate_up.device)
        else:
            _given(data, lead + (inter // 2,), gate_up.device, "NVFP4 data")
        if scale is None:
            scale = torch.empty(lead + (inter // 16,), dtype=torch.float8_e4m3fn, device=gate_up.device)
        else:
            _given(scale, lead + (inter // 16,), gate_up.device, "NVFP4 scale")
    given = amax is not None
    if amax is None:
        amax = amax_out if amax_out is not None else torch.empty(1, dtype=torch.float32, device=gate_up.device)
    if amax.dtype != torch.float32 or amax.numel() != 1 or amax.device != gate_up.device:
        raise ValueError("amax must be one float32 element on gate_up's device")
    tokens = g2.shape[0]
    if amax_only:
        d_ptr, d_pitch, s_ptr, s_pitch = None, inter // 2, None, inter // 16
    else:
        d2 = data.view(-1, inter // 2)
        s2 = scale.view(-1, inter // 16)
        d_ptr, d_pitch = d2.data_ptr(), d2.stride(0) if tokens > 1 else inter // 2
        s_ptr, s_pitch = s2.data_ptr(), s2.stride(0) if tokens > 1 else inter // 16
    st = abi.situ_glu_fwd_nvfp4(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                                rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                                float(beta), int(linear_beta is not None),
                                float(linear_beta) if linear_beta is not None else 0.0,
                                d_ptr, d_pitch, s_ptr, s_pitch, amax.data_ptr(), 2 if amax_only else int(given),
                                _stream_handle(stream))
    abi.check(st, "situ_glu_fwd_nvfp4")
    return (None, None, amax) if amax_only else (data, scale, amax)


def situ_glu_bwd_nvfp4(gate_up: torch.Tensor, routing_weights, grad_out: torch.Tensor,
                       beta: float = DEFAULT_BETA, linear_beta: float | None = DEFAULT_LINEAR_BETA,
                       want_drw: bool = True, amax: torch.Tensor | None = None, data=None, scale=None,
                       amax_out: torch.Tensor | None = None, d_rw=None, workspace=None, amax_only: bool = False,
                       stream=None):
    """Backward with an NVFP4 d_gate_up: returns (packed E2M1 codes [..., I]
    uint8 with dG's I / 2 bytes then dU's, E4M3 block scales [..., 2I / 16] as
    torch.float8_e4m3fn, amax: a 1-element fp32 tensor holding d_gate_up's
    tensor maximum A, d_routing_weights or None).  ``amax`` gives A instead
    of computing it; otherwise it is computed into ``amax_out``.
    ``amax_only``: compute A alone (no codes, no weight gradient) and return
    (None, None, amax, None).  The weight gradient is as in situ_glu_bwd."""
    _check_beta(beta, linear_beta)
    g2, lead, inter = _rows(gate_up)
    dtype = _dtype_code(g2, "gate_up")
    if grad_out.dtype != gate_up.dtype:
        raise TypeError("grad_out must have gate_up's dtype")
    if tuple(grad_out.shape) != lead + (inter,):
        raise ValueError(f"grad_out shape {tuple(grad_out.shape)} != {lead + (inter,)}")
    go2 = grad_out if grad_out.dim() == 2 else grad_out.reshape(-1, inter)
    if go2.stride(1) != 1 or (go2.shape[0] > 1 and go2.stride(0) < inter):
        go2 = go2.contiguous()
    mode, rw, rw_stride = routing_mode(lead, inter, routing_weights)
    rw_dtype = _dtype_code(rw, "routing_weights") if rw is not None else abi.SITU_DTYPE_F32
    want = bool(want_drw) and rw is not None and not amax_only
    if amax_only and amax is not None:
        raise ValueError("amax_only computes the tensor maximum: do not pass one")
    if not amax_only:
        if data is None:
            data = torch.empty(lead + (inter,), dtype=torch.uint8, device=gate_up.device)
        else:
            _given(data, lead + (inter,), gate_up.device, "NVFP4 data")
        if scale is None:
            scale = torch.empty(lead + (2 * inter // 16,), dtype=torch.float8_e4m3fn, device=gate_up.device)
        else:
            _given(scale, lead + (2 * inter // 16,), gate_up.device, "NVFP4 scale")
    given = amax is not None
    if amax is None:
        amax = amax_out if amax_out is not None else torch.empty(1, dtype=torch.float32, device=gate_up.device)
    if amax.dtype != torch.float32 or amax.numel() != 1 or amax.device != gate_up.device:
        raise ValueError("amax must be one float32 element on gate_up's device")
    tokens = g2.shape[0]
    if amax_only:
        d_ptr, d_pitch, s_ptr, s_pitch = None, inter, None, 2 * inter // 16
    else:
        d2 = data.view(-1, inter)
        s2 = scale.view(-1, 2 * inter // 16)
        d_ptr, d_pitch = d2.data_ptr(), d2.stride(0) if tokens > 1 else inter
        s_ptr, s_pitch = s2.data_ptr(), s2.stride(0) if tokens > 1 else 2 * inter // 16
    d_rw_flat, d_rw_stride = None, 1
    if want:
        if d_rw is None:
            d_rw = torch.empty(routing_weights.shape, dtype=routing_weights.dtype, device=gate_up.device)
        else:
            _given_drw(d_rw, routing_weights, gate_up.device)
        d_rw_flat = d_rw.view(-1)
        d_rw_stride = d_rw_flat.stride(0) if d_rw_flat.numel() > 1 else 1
    ws_bytes = abi.situ_glu_bwd_workspace_bytes(tokens, inter, mode, int(want))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=gate_up.device)
    st = abi.situ_glu_bwd_nvfp4(g2.data_ptr(), dtype, tokens, inter, g2.stride(0) if tokens > 1 else 2 * inter,
                                rw.data_ptr() if rw is not None else None, rw_dtype, mode, rw_stride,
                                float(beta), int(linear_beta is not None),
                                float(linear_beta) if linear_beta is not None else 0.0,
                                go2.data_ptr(), go2.stride(0) if tokens > 1 else inter,
                                d_ptr, d_pitch, s_ptr, s_pitch, amax.data_ptr(), 2 if amax_only else int(given),
                                d_rw_flat.data_ptr() if d_rw_flat is not None else None, d_rw_stride,
                                workspace.data_ptr() if ws_bytes else None, ws_bytes, _stream_handle(stream))
    abi.check(st, "situ_glu_bwd_nvfp4")
    if amax_only:
        return None, None, amax, None
    return data, scale, amax, (d_rw if want else None)


class WeightedSiTUFunction(torch.autograd.Function):
    """Routing-weighted SiTU-GLU with the analytic fused backward.

    Saves only gate_up and routing_weights (NeMo `_WeightedSiTUFunction`:
    "saves only the low-precision inputs"); backward returns
    (d_gate_up, d_routing_weights, None, None)."""

    @staticmethod
    def forward(ctx, gate_up, routing_weights, beta, linear_beta):
        out = situ_glu_fwd(gate_up, routing_weights, beta, linear_beta)
        if routing_weights is None:
            ctx.save_for_backward(gate_up)
        else:
            ctx.save_for_backward(gate_up, routing_weights)
        ctx.has_rw = routing_weights is not None
        ctx.beta = beta
        ctx.linear_beta = linear_beta
        return out

    @staticmethod
    def backward(ctx, grad_out):
        saved = ctx.saved_tensors
        gate_up = saved[0]
        rw = saved[1] if ctx.has_rw else None
        want_drw = ctx.has_rw and ctx.needs_input_grad[1]
        d_gate_up, d_rw = situ_glu_bwd(gate_up, rw, grad_out, ctx.beta, ctx.linear_beta,
                                       want_drw=want_drw)
        return d_gate_up, d_rw, None, None


def weighted_situ(gate_up: torch.Tensor, routing_weights, beta: float = DEFAULT_BETA,
                  linear_beta: float | None = DEFAULT_LINEAR_BETA) -> torch.Tensor:
    """Apply SiTU-GLU and routing weights to gate_up [..., 2 * intermediate]
    (NeMo `_weighted_situ`): gate in the first half, up in the second.
    routing_weights: [..., 1] row-aligned, one broadcast value, [I] per
    column, [..., I] per element, or None."""
    return WeightedSiTUFunction.apply(gate_up, routing_weights, beta, linear_beta)


def situlu(gate_up: torch.Tensor, beta: float = DEFAULT_BETA,
           linear_beta: float | None = DEFAULT_LINEAR_BETA) -> torch.Tensor:
    """Unweighted SiTU-GLU (Megatron-LM PR #6673 "Design": the `situlu`
    pointwise reference / TE SiTUGLU op), on the same kernels."""
    return WeightedSiTUFunction.apply(gate_up, None, beta, linear_beta)
