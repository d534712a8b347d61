"""Randomised argument checks of the C ABI on the CPU (hypothesis).

Each call starts from a valid argument set of an entry point and replaces a
random subset of its fields with values drawn from pools of edge cases
(NULL and misaligned addresses, zero, negative and huge sizes and strides,
bad enums, non-finite betas).  Properties:

* every call returns one of the documented status codes (no crash);
* a call whose extents overflow int64 (a huge token count, stride or
  intermediate size) or that lacks a required pointer is rejected on the host
  -- never SITU_OK, never a CUDA-side error (on this GPU-less machine a call
  that passes validation reaches CUDA and returns SITU_ERR_CUDA).

The addresses are fake, so the module is skipped where a GPU is present: a
valid draw would launch a kernel on them.
"""
import pytest
import torch
from hypothesis import HealthCheck, given, settings, strategies as st

from ffn_gated_activation_b200 import abi

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device addresses: CPU-only test")

GU, RW, OUT, GO, DGU, DRW, WS, AMX, SC, XP, W1, OFF, W2, NW, PW, BL, PR = (0x1000_0000 * k for k in range(1, 18))
CODES = {abi.SITU_OK, abi.SITU_ERR_INVALID_ARG, abi.SITU_ERR_UNSUPPORTED, abi.SITU_ERR_MISALIGNED,
         abi.SITU_ERR_CUDA}
HUGE = [2 ** 40, 2 ** 62, 2 ** 63 - 1]
SIZES = st.sampled_from([0, 1, 2, 3, 8, 16, 17, 32, 64, 100, 256, -1, -7] + HUGE)
PTRS = st.sampled_from([None, 0x8, 0x2, 0x1000_0001, 0x1000_0008, 0x7000_0000, 0x8000_0000])
ENUMS = st.sampled_from([-1, 0, 1, 2, 3, 4, 5, 9])
BETAS = st.sampled_from([4.0, 1.0, 0.0, -2.0, float("nan"), float("inf"), 1e-30, 1e30])

BASE = {
    "fwd": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1, rw_mode=0,
                rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, out=OUT, out_row_stride=64, stream=None),
    "bwd": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1, rw_mode=0,
                rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO, grad_out_row_stride=64,
                d_gate_up=DGU, d_gate_up_row_stride=128, d_rw=DRW, d_rw_stride=1, workspace=None,
                workspace_bytes=0, stream=None),
    "fwd_mxfp8": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1,
                      rw_mode=0, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, y_data=OUT,
                      y_data_row_stride=64, y_scale=SC, y_scale_row_stride=2, rule=0, stream=None),
    "fwd_nvfp4": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1,
                      rw_mode=0, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, y_data=OUT,
                      y_data_row_stride=32, y_scale=SC, y_scale_row_stride=4, amax=AMX, amax_given=1, stream=None),
    "bwd_nvfp4": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1,
                      rw_mode=0, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO,
                      grad_out_row_stride=64, d_gate_up_data=DGU, d_gate_up_data_row_stride=64,
                      d_gate_up_scale=SC, d_gate_up_scale_row_stride=8, amax=AMX, amax_given=1, d_rw=DRW,
                      d_rw_stride=1, workspace=None, workspace_bytes=0, stream=None),
    "bwd_mxfp8": dict(gate_up=GU, dtype=0, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=1,
                      rw_mode=0, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO,
                      grad_out_row_stride=64, d_gate_up_data=DGU, d_gate_up_data_row_stride=128, d_gate_up_scale=SC,
                      d_gate_up_scale_row_stride=4, rule=0, d_rw=DRW, d_rw_stride=1, workspace=None,
                      workspace_bytes=0, stream=None),
    "fc1": dict(x=XP, tokens=256, hidden=128, x_row_stride=128, w1=W1, experts=2, inter=128, w1_row_stride=128,
                offsets=OFF, rw=RW, rw_dtype=1, rw_mode=0, rw_stride=1, beta=4.0, has_linear_beta=1,
                linear_beta=25.0, y=OUT, y_row_stride=128, stream=None),
    "fc2": dict(dout=GO, tokens=256, hidden=128, dout_row_stride=128, w2t=W2, experts=2, inter=256,
                w2t_row_stride=128, offsets=OFF, gate_up=GU, gate_up_row_stride=512, rw=RW, rw_dtype=1, rw_mode=0,
                rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, d_gate_up=DGU, d_gate_up_row_stride=512,
                d_rw=DRW, d_rw_stride=1, workspace=WS, workspace_bytes=1 << 20, stream=None),
    "attn_res": dict(blocks=BL, nblocks=8, block_row_stride=8 * 256, block_stride=256, prefix=PR,
                     prefix_row_stride=256, dtype=0, tokens=64, hidden=256, norm_weight=NW, norm_dtype=1,
                     proj_weight=PW, proj_dtype=1, variance_epsilon=1e-6, out=OUT, out_dtype=0, out_row_stride=256,
                     stream=None),
}
CALL = {"fwd": abi.situ_glu_fwd, "bwd": abi.situ_glu_bwd, "fwd_mxfp8": abi.situ_glu_fwd_mxfp8,
        "fwd_nvfp4": abi.situ_glu_fwd_nvfp4, "bwd_nvfp4": abi.situ_glu_bwd_nvfp4,
        "bwd_mxfp8": abi.situ_glu_bwd_mxfp8, "fc1": abi.situ_glu_fc1_fwd, "fc2": abi.situ_glu_fc2_dgrad_bwd,
        "attn_res": abi.situ_attn_res_fwd}
REQUIRED = {"fwd": ["gate_up", "out"], "bwd": ["gate_up", "grad_out", "d_gate_up"],
            "fwd_mxfp8": ["gate_up", "y_data", "y_scale"], "fwd_nvfp4": ["gate_up", "y_data", "y_scale", "amax"],
            "bwd_nvfp4": ["gate_up", "grad_out", "d_gate_up_data", "d_gate_up_scale", "amax"],
            "bwd_mxfp8": ["gate_up", "grad_out", "d_gate_up_data", "d_gate_up_scale"],
            "fc1": ["x", "w1", "offsets", "y"], "fc2": ["dout", "w2t", "offsets", "gate_up", "d_gate_up"],
            "attn_res": ["norm_weight", "proj_weight", "out"]}
# entry points whose byte extents the overflow property below models
EXTENTS_MODELLED = {"fwd", "bwd", "fwd_mxfp8", "fwd_nvfp4", "bwd_nvfp4", "bwd_mxfp8", "fc1", "fc2", "attn_res"}


def field_strategy(name):
    if name in ("gate_up", "rw", "out", "grad_out", "d_gate_up", "d_rw", "workspace", "y_data", "y_scale", "amax",
                "d_gate_up_data", "d_gate_up_scale", "x", "w1", "offsets", "y", "dout", "w2t", "blocks", "prefix",
                "norm_weight", "proj_weight"):
        return PTRS
    if name in ("dtype", "rw_dtype", "rw_mode", "rule", "amax_given", "has_linear_beta", "norm_dtype",
                "proj_dtype", "out_dtype"):
        return ENUMS
    if name in ("beta", "linear_beta", "variance_epsilon"):
        return BETAS
    if name == "stream":
        return st.just(None)
    return SIZES


def extent_overflows(entry, a, amax_only):
    """Whether the byte extent (rows - 1) * pitch + row of a tensor the call
    uses exceeds int64 -- exact integer arithmetic."""
    limit = 2 ** 63 - 1
    T = a["tokens"]
    if entry == "attn_res":  # sources [T, B, H] at (row, source) strides, prefix and out [T, H]
        H, B = a["hidden"], a["nblocks"]
        es = 2 if a["dtype"] == 0 else 4
        oes = 2 if a["out_dtype"] == 0 else 4
        ext = []
        if a["blocks"] is not None and B > 0 and a["block_row_stride"] >= 0 and a["block_stride"] >= 0:
            ext.append(((T - 1) * a["block_row_stride"] + (B - 1) * a["block_stride"] + H) * es)
        if a["prefix"] is not None and a["prefix_row_stride"] >= H:
            ext.append(((T - 1) * a["prefix_row_stride"] + H) * es)
        if a["out_row_stride"] >= H:
            ext.append(((T - 1) * a["out_row_stride"] + H) * oes)
        return H > 0 and any(e > limit for e in ext)
    I = a["inter"]
    es = 2 if a.get("dtype", 0) == 0 else 4
    rw_es = 2 if a["rw_dtype"] == 0 else 4
    if entry in ("fc1", "fc2"):  # bf16 only; weights [E * 2I or E * I, H]
        H, E = a["hidden"], a["experts"]
        if entry == "fc1":
            spans = [(a["x_row_stride"], H, 2), (a["y_row_stride"], I, 2)]
            w_rows, w_pitch = E * 2 * I, a["w1_row_stride"]
        else:
            spans = [(a["dout_row_stride"], H, 2), (a["gate_up_row_stride"], 2 * I, 2),
                     (a["d_gate_up_row_stride"], 2 * I, 2)]
            w_rows, w_pitch = E * I, a["w2t_row_stride"]
        if w_pitch >= H >= 0 and E > 0 and ((w_rows - 1) * w_pitch + H) * 2 > limit:
            return True
        if a["rw_mode"] == abi.SITU_RW_ROW and a["rw"] is not None:
            spans.append((a["rw_stride"], 1, rw_es))
            if entry == "fc2" and a.get("d_rw") is not None:
                spans.append((a["d_rw_stride"], 1, rw_es))
        return any(w * e > limit or ((T - 1) * p + w) * e > limit for p, w, e in spans if p >= w >= 0)
    spans = [(a["gate_up_row_stride"], 2 * I, es)]
    if entry == "fwd":
        spans.append((a["out_row_stride"], I, es))
    if entry in ("bwd", "bwd_nvfp4", "bwd_mxfp8"):
        spans.append((a["grad_out_row_stride"], I, es))
    if entry == "bwd":
        spans.append((a["d_gate_up_row_stride"], 2 * I, es))
    if entry == "fwd_mxfp8":
        spans += [(a["y_data_row_stride"], I, 1), (a["y_scale_row_stride"], I // 32, 1)]
    if entry == "bwd_mxfp8":
        spans += [(a["d_gate_up_data_row_stride"], 2 * I, 1), (a["d_gate_up_scale_row_stride"], 2 * I // 32, 1)]
    if entry == "fwd_nvfp4" and not amax_only:
        spans += [(a["y_data_row_stride"], I // 2, 1), (a["y_scale_row_stride"], I // 16, 1)]
    if entry == "bwd_nvfp4" and not amax_only:
        spans += [(a["d_gate_up_data_row_stride"], I, 1), (a["d_gate_up_scale_row_stride"], 2 * I // 16, 1)]
    if a["rw_mode"] == abi.SITU_RW_ROW and a["rw"] is not None:  # a broadcast or absent weight has no stride
        spans.append((a["rw_stride"], 1, rw_es))
        if a.get("d_rw") is not None:
            spans.append((a["d_rw_stride"], 1, rw_es))
    return any(w * e > limit or ((T - 1) * p + w) * e > limit for p, w, e in spans if p >= w >= 0)


@st.composite
def calls(draw):
    entry = draw(st.sampled_from(sorted(BASE)))
    args = dict(BASE[entry])
    names = draw(st.lists(st.sampled_from(sorted(k for k in args if k != "stream")), min_size=1, max_size=3,
                          unique=True))
    for n in names:
        args[n] = draw(field_strategy(n))
    return entry, args


@settings(max_examples=2000, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(call=calls())
def test_random_arguments_are_validated_on_the_host(call, native_lib_path):
    entry, args = call
    status = CALL[entry](**args)
    assert status in CODES, (entry, args, status)
    tokens = args["tokens"]
    if tokens <= 0 or args.get("dtype", 0) not in (0, 1) or args.get("rw_dtype", 1) not in (0, 1):
        return
    amax_only = args.get("amax_given") == 2  # NVFP4: the tensor maximum alone, no codes written
    if entry in EXTENTS_MODELLED and extent_overflows(entry, args, amax_only):
        assert status not in (abi.SITU_OK, abi.SITU_ERR_CUDA), (entry, args, abi.situ_glu_last_error())
    required = [k for k in REQUIRED[entry]
                if not (amax_only and k in ("y_data", "y_scale", "d_gate_up_data", "d_gate_up_scale"))]
    if any(args[k] is None for k in required):
        assert status not in (abi.SITU_OK, abi.SITU_ERR_CUDA), (entry, args, abi.situ_glu_last_error())
