"""The C-ABI boundary on the CPU: the library loads, exports every entry point
include/situ_glu.h declares, and rejects bad arguments on the host before
any CUDA call (no GPU is touched by these tests)."""
import json
import os
import re
import subprocess

import pytest

from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]

BF16, F32 = abi.SITU_DTYPE_BF16, abi.SITU_DTYPE_F32
ROW, SCALAR, NONE = abi.SITU_RW_ROW, abi.SITU_RW_SCALAR, abi.SITU_RW_NONE
OK, INVALID, UNSUP, MISAL = abi.SITU_OK, abi.SITU_ERR_INVALID_ARG, abi.SITU_ERR_UNSUPPORTED, abi.SITU_ERR_MISALIGNED

# Fake, well-separated, 256-byte-aligned device addresses: validation never
# dereferences them.
GU, RW, OUT, GO, DGU, DRW, WS = (0x1000_0000 * k for k in range(1, 8))


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(situ_(?:glu|attn_res)_\w+)\s*\(", text, flags=re.M))
    return names


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"situ_glu_fwd", "situ_glu_bwd", "situ_glu_bwd_workspace_bytes", "situ_glu_status_string",
            "situ_glu_last_error", "situ_glu_abi_version", "situ_glu_set_max_ctas",
            "situ_glu_set_load_path", "situ_glu_device_status"} <= names


def test_library_exports_every_declared_symbol(native_lib_path):
    out = subprocess.run(["nm", "-D", "--defined-only", native_lib_path], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = declared_functions() - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    lib = abi.lib()
    for name in declared_functions():
        getattr(lib, name)  # resolvable through ctypes


def test_binding_covers_the_header_exactly():
    assert set(abi.SIGNATURES) == declared_functions()
    for name in abi.SIGNATURES:
        assert hasattr(abi, name), f"binding lacks a Python function named {name}"


def test_version_and_status_strings(native_lib_path):
    assert abi.situ_glu_abi_version() == abi.ABI_VERSION == 8
    assert abi.situ_glu_status_string(OK) == "SITU_OK"
    assert abi.situ_glu_status_string(MISAL) == "SITU_ERR_MISALIGNED"
    assert abi.situ_glu_status_string(99) == "SITU_ERR_UNKNOWN"


def test_workspace_query(native_lib_path):
    COL, FULL = abi.SITU_RW_COL, abi.SITU_RW_FULL
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, ROW, 1) == 0
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, FULL, 1) == 0
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, SCALAR, 0) == 0
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, SCALAR, 1) == 4096
    assert abi.situ_glu_bwd_workspace_bytes(64, 64, SCALAR, 1) == 256
    assert abi.situ_glu_bwd_workspace_bytes(0, 64, SCALAR, 1) == 0
    assert abi.situ_glu_bwd_workspace_bytes(-5, 64, SCALAR, 1) == 0
    # per-column weights: one partial per column per chunk of 16 rows
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, COL, 1) == 63 * 64 * 4
    assert abi.situ_glu_bwd_workspace_bytes(65, 520, COL, 1) == (5 * 520 * 4 + 255) // 256 * 256
    assert abi.situ_glu_bwd_workspace_bytes(1000, 64, COL, 0) == 0
    assert abi.situ_glu_bwd_workspace_bytes(1000, 0, COL, 1) == 0


def test_load_path_knob(native_lib_path):
    prev = abi.situ_glu_set_load_path(1)
    assert abi.situ_glu_set_load_path(prev) == 1
    assert abi.situ_glu_set_load_path(2) == -1
    assert abi.situ_glu_set_load_path(-1) == -1


def test_max_ctas_knob(native_lib_path):
    prev = abi.situ_glu_set_max_ctas(7)
    assert abi.situ_glu_set_max_ctas(prev) == 7
    assert abi.situ_glu_set_max_ctas(-1) == -1


@pytest.mark.parametrize("limit_ns", [0, -1, 10_000_000_001])
def test_wait_probe_rejects_the_limit_before_any_launch(limit_ns, native_lib_path):
    assert abi.situ_glu_wait_probe(limit_ns) == INVALID
    assert "limit_ns" in abi.situ_glu_last_error()


def fwd(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, out=OUT,
             out_row_stride=64, stream=None)
    a.update(kw)
    return abi.situ_glu_fwd(**a)


def bwd(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO,
             grad_out_row_stride=64, d_gate_up=DGU, d_gate_up_row_stride=128, d_rw=DRW, d_rw_stride=1,
             workspace=None, workspace_bytes=0, stream=None)
    a.update(kw)
    return abi.situ_glu_bwd(**a)


FWD_CASES = [
    ("bad dtype", dict(dtype=7), INVALID),
    ("bad rw_mode", dict(rw_mode=9), INVALID),
    ("full weights: stride short", dict(rw_mode=4, rw_stride=63), INVALID),
    ("full weights misaligned", dict(rw_mode=4, rw_stride=64, rw=RW + 4), MISAL),
    ("full weights pitch misaligned", dict(rw_mode=4, rw_stride=65), MISAL),
    ("full bf16 weights, fp32 gate_up: pitch not 8-byte", dict(dtype=1, rw_dtype=0, rw_mode=4, rw_stride=66), MISAL),
    ("column weights misaligned", dict(rw_mode=3, rw=RW + 8), MISAL),
    ("column weights: inter too large", dict(rw_mode=3, inter=1 << 15, gate_up_row_stride=1 << 16,
                                              out_row_stride=1 << 15), UNSUP),
    ("bad rw_dtype", dict(rw_dtype=3), INVALID),
    ("negative tokens", dict(tokens=-1), INVALID),
    ("zero inter", dict(inter=0), INVALID),
    ("huge inter", dict(inter=1 << 29, gate_up_row_stride=1 << 30, out_row_stride=1 << 29), UNSUP),
    ("beta zero", dict(beta=0.0), INVALID),
    ("beta negative", dict(beta=-4.0), INVALID),
    ("beta inf", dict(beta=float("inf")), INVALID),
    ("beta nan", dict(beta=float("nan")), INVALID),
    ("has_linear_beta not 0/1", dict(has_linear_beta=2), INVALID),
    ("linear beta zero", dict(linear_beta=0.0), INVALID),
    ("linear beta nan", dict(linear_beta=float("nan")), INVALID),
    ("gate_up stride short", dict(gate_up_row_stride=127), INVALID),
    ("out stride short", dict(out_row_stride=63), INVALID),
    ("rw NULL in row mode", dict(rw=None), INVALID),
    ("rw given when unweighted", dict(rw_mode=NONE), INVALID),
    ("negative rw stride", dict(rw_stride=-1), INVALID),
    ("inter not a 16-byte multiple", dict(inter=12, gate_up_row_stride=24, out_row_stride=12), MISAL),
    ("gate_up NULL", dict(gate_up=None), INVALID),
    ("out NULL", dict(out=None), INVALID),
    ("gate_up misaligned", dict(gate_up=GU + 8), MISAL),
    ("out misaligned", dict(out=OUT + 2), MISAL),
    ("gate_up pitch misaligned", dict(gate_up_row_stride=132), MISAL),
    ("rw misaligned", dict(rw=RW + 2), MISAL),
    ("out overlaps gate_up", dict(out=GU + 256), INVALID),
    ("out overlaps rw", dict(out=RW - 16 * 64 * 2 + 16), INVALID),
    ("extent overflow", dict(tokens=1 << 40, gate_up_row_stride=1 << 40), INVALID),
]


@pytest.mark.parametrize("name,kw,status", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fwd_rejects(name, kw, status, native_lib_path):
    assert fwd(**kw) == status
    assert abi.situ_glu_last_error() != ""


BWD_CASES = [
    ("grad_out stride short", dict(grad_out_row_stride=63), INVALID),
    ("d_gate_up stride short", dict(d_gate_up_row_stride=100), INVALID),
    ("d_rw when unweighted", dict(rw=None, rw_mode=NONE), INVALID),
    ("d_rw stride zero", dict(d_rw_stride=0), INVALID),
    ("scalar without workspace", dict(rw_mode=SCALAR), INVALID),
    ("column weights without workspace", dict(rw_mode=3), INVALID),
    ("full weights: d_rw stride short", dict(rw_mode=4, rw_stride=64, d_rw_stride=63), INVALID),
    ("full weights: d_rw overlaps rw", dict(rw_mode=4, rw_stride=64, d_rw_stride=64, d_rw=RW + 256), INVALID),
    ("scalar workspace short", dict(rw_mode=SCALAR, workspace=WS, workspace_bytes=32), INVALID),
    ("scalar workspace misaligned", dict(rw_mode=SCALAR, workspace=WS + 4, workspace_bytes=256), MISAL),
    ("grad_out NULL", dict(grad_out=None), INVALID),
    ("d_gate_up NULL", dict(d_gate_up=None), INVALID),
    ("grad_out misaligned", dict(grad_out=GO + 4), MISAL),
    ("d_rw misaligned", dict(d_rw=DRW + 1), MISAL),
    ("d_gate_up overlaps grad_out", dict(d_gate_up=GO), INVALID),
    ("d_gate_up overlaps gate_up", dict(d_gate_up=GU + 2048), INVALID),
    ("d_rw overlaps d_gate_up", dict(d_rw=DGU + 64), INVALID),
    ("d_rw overlaps rw", dict(d_rw=RW), INVALID),
    ("workspace overlaps grad_out", dict(rw_mode=SCALAR, workspace=GO, workspace_bytes=256), INVALID),
    ("beta negative", dict(beta=-1.0), INVALID),
]


@pytest.mark.parametrize("name,kw,status", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_bwd_rejects(name, kw, status, native_lib_path):
    assert bwd(**kw) == status
    assert abi.situ_glu_last_error() != ""


def test_zero_tokens_launch_nothing(native_lib_path):
    assert fwd(tokens=0, gate_up=None, out=None, rw=None) == OK
    assert bwd(tokens=0, gate_up=None, grad_out=None, d_gate_up=None, d_rw=None) == OK
    assert abi.situ_glu_last_error() == ""


def test_binding_routing_modes():
    import torch
    from ffn_gated_activation_b200.functional import routing_mode
    lead, inter = (4, 6), 16
    COL, FULL = abi.SITU_RW_COL, abi.SITU_RW_FULL
    assert routing_mode(lead, inter, None)[0] == NONE
    assert routing_mode(lead, inter, torch.tensor(0.5))[0] == SCALAR
    assert routing_mode(lead, inter, torch.ones(1, 1, 1))[0] == SCALAR
    m, flat, stride = routing_mode(lead, inter, torch.ones(4, 6, 1))
    assert m == ROW and flat.shape == (24,) and stride == 1
    # a column slice of top-k weights: rows 8 elements apart
    m, flat, stride = routing_mode(lead, inter, torch.ones(4, 6, 8)[..., 2:3])
    assert m == ROW and stride == 8
    assert routing_mode(lead, inter, torch.ones(16))[0] == COL
    assert routing_mode(lead, inter, torch.ones(1, 1, 16))[0] == COL
    m, w2, stride = routing_mode(lead, inter, torch.ones(4, 6, 16))
    assert m == FULL and w2.shape == (24, 16) and stride == 16
    for bad in (torch.ones(4, 6), torch.ones(4, 6, 8), torch.ones(6, 16)):
        with pytest.raises(NotImplementedError):  # none of these broadcast as a per-row / column / element weight
            routing_mode(lead, inter, bad)


def test_binding_validates_betas():
    from ffn_gated_activation_b200.functional import _check_beta
    _check_beta(4.0, 25.0)
    _check_beta(4.0, None)
    for bad in ((0.0, 25.0), (float("inf"), None), (4.0, -1.0), (4.0, float("nan"))):
        with pytest.raises(ValueError):
            _check_beta(*bad)


def test_defaults_match_the_pages():
    golden = json.load(open(os.path.join(ROOT, "tests", "golden", "situ_defaults.json")))
    assert pkg.DEFAULT_BETA == golden["beta"]["value"]
    assert pkg.DEFAULT_LINEAR_BETA == golden["linear_beta"]["value"]
    assert golden["moe_intermediate_size"]["value"] == 3072


# ---- MXFP8 entry points: argument checks run before any CUDA call --------------

MXD = 0x80000000   # fake 16-byte aligned device addresses for the outputs, clear of the inputs
MXS = 0x88000000


def fwd_mx(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, y_data=MXD,
             y_data_row_stride=64, y_scale=MXS, y_scale_row_stride=2, rule=abi.SITU_MX_RULE_OCP, stream=None)
    a.update(kw)
    return abi.situ_glu_fwd_mxfp8(**a)


def bwd_mx(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO,
             grad_out_row_stride=64, d_gate_up_data=MXD, d_gate_up_data_row_stride=128, d_gate_up_scale=MXS,
             d_gate_up_scale_row_stride=4, rule=abi.SITU_MX_RULE_OCP, d_rw=DRW, d_rw_stride=1, workspace=None,
             workspace_bytes=0, stream=None)
    a.update(kw)
    return abi.situ_glu_bwd_mxfp8(**a)


MX_CASES = [
    ("inter not a multiple of 32", dict(inter=40, gate_up_row_stride=80), INVALID),
    ("bad rule", dict(rule=5), INVALID),
    ("per-column weights", dict(rw_mode=3), UNSUP),
    ("per-element weights", dict(rw_mode=4, rw_stride=64), UNSUP),
    ("scale pitch short", dict(scale_short=True), INVALID),
    ("data pitch short", dict(data_short=True), INVALID),
    ("data pitch not 16-byte", dict(data_pitch_odd=True), MISAL),
    ("data misaligned", dict(data_off=8), MISAL),
    ("data NULL", dict(data_null=True), INVALID),
    ("data overlaps gate_up", dict(data_at_gu=True), INVALID),
    ("scale overlaps data", dict(scale_at_data=True), INVALID),
    ("bad beta", dict(beta=-1.0), INVALID),
]


def _mx_kw(kw, cols, prefix):
    kw = dict(kw)
    d, dp, sc, sp = (f"{prefix}data", f"{prefix}data_row_stride", f"{prefix}scale", f"{prefix}scale_row_stride")
    if kw.pop("scale_short", False):
        kw[sp] = cols // 32 - 1
    if kw.pop("data_short", False):
        kw[dp] = cols - 16
    if kw.pop("data_pitch_odd", False):
        kw[dp] = cols + 8
    off = kw.pop("data_off", 0)
    if off:
        kw[d] = MXD + off
    if kw.pop("data_null", False):
        kw[d] = None
    if kw.pop("data_at_gu", False):
        kw[d] = GU
    if kw.pop("scale_at_data", False):
        kw[sc] = MXD + 32
    return kw


@pytest.mark.parametrize("name,kw,want", MX_CASES, ids=[c[0] for c in MX_CASES])
def test_fwd_mxfp8_argument_errors(name, kw, want, native_lib_path):
    inter = kw.get("inter", 64)
    assert fwd_mx(**_mx_kw(kw, inter, "y_")) == want, abi.situ_glu_last_error()


@pytest.mark.parametrize("name,kw,want", MX_CASES, ids=[c[0] for c in MX_CASES])
def test_bwd_mxfp8_argument_errors(name, kw, want, native_lib_path):
    inter = kw.get("inter", 64)
    assert bwd_mx(**_mx_kw(kw, 2 * inter, "d_gate_up_")) == want, abi.situ_glu_last_error()


def test_mxfp8_zero_tokens_is_a_no_op(native_lib_path):
    assert fwd_mx(tokens=0, y_data=None, y_scale=None) == OK
    assert bwd_mx(tokens=0, d_gate_up_data=None, d_gate_up_scale=None, d_rw=None) == OK


# ---- NVFP4 forward: argument checks run before any CUDA call ---------------------

AMX = 0x8C000000


def fwd_nv(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, y_data=MXD,
             y_data_row_stride=32, y_scale=MXS, y_scale_row_stride=4, amax=AMX, amax_given=1, stream=None)
    a.update(kw)
    return abi.situ_glu_fwd_nvfp4(**a)


NV_CASES = [
    ("inter not a multiple of 16", dict(inter=40, gate_up_row_stride=80, y_data_row_stride=32,
                                        y_scale_row_stride=4), INVALID),
    ("per-column weights", dict(rw_mode=3), UNSUP),
    ("per-element weights", dict(rw_mode=4, rw_stride=64), UNSUP),
    ("scale pitch short", dict(y_scale_row_stride=3), INVALID),
    ("data pitch short", dict(y_data_row_stride=16), INVALID),
    ("data pitch not 4-byte", dict(y_data_row_stride=34), MISAL),
    ("data misaligned", dict(y_data=MXD + 2), MISAL),
    ("data NULL", dict(y_data=None), INVALID),
    ("scale NULL", dict(y_scale=None), INVALID),
    ("amax NULL", dict(amax=None), INVALID),
    ("amax misaligned", dict(amax=AMX + 2), MISAL),
    ("amax_given not 0, 1 or 2", dict(amax_given=3), INVALID),
    ("data overlaps gate_up", dict(y_data=GU), INVALID),
    ("amax inside the scales", dict(amax=MXS + 8), INVALID),
    ("scale overlaps data", dict(y_scale=MXD + 32), INVALID),
    ("bad beta", dict(beta=-1.0), INVALID),
    ("bad dtype", dict(dtype=7), INVALID),
]


@pytest.mark.parametrize("name,kw,want", NV_CASES, ids=[c[0] for c in NV_CASES])
def test_fwd_nvfp4_argument_errors(name, kw, want, native_lib_path):
    assert fwd_nv(**kw) == want, abi.situ_glu_last_error()


def test_nvfp4_zero_tokens_with_given_amax_is_a_no_op(native_lib_path):
    assert fwd_nv(tokens=0, y_data=None, y_scale=None) == OK
    assert bwd_nv(tokens=0, d_gate_up_data=None, d_gate_up_scale=None, d_rw=None) == OK


def bwd_nv(**kw):
    a = dict(gate_up=GU, dtype=BF16, tokens=16, inter=64, gate_up_row_stride=128, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, grad_out=GO,
             grad_out_row_stride=64, d_gate_up_data=MXD, d_gate_up_data_row_stride=64, d_gate_up_scale=MXS,
             d_gate_up_scale_row_stride=8, amax=AMX, amax_given=1, d_rw=DRW, d_rw_stride=1, workspace=None,
             workspace_bytes=0, stream=None)
    a.update(kw)
    return abi.situ_glu_bwd_nvfp4(**a)


NV_BWD_CASES = [
    ("inter not a multiple of 16", dict(inter=40, gate_up_row_stride=80, grad_out_row_stride=40), INVALID),
    ("per-column weights", dict(rw_mode=3), UNSUP),
    ("per-element weights", dict(rw_mode=4, rw_stride=64), UNSUP),
    ("scale pitch short", dict(d_gate_up_scale_row_stride=7), INVALID),
    ("data pitch short", dict(d_gate_up_data_row_stride=60), INVALID),
    ("data pitch not 4-byte", dict(d_gate_up_data_row_stride=66), MISAL),
    ("data misaligned", dict(d_gate_up_data=MXD + 2), MISAL),
    ("data NULL", dict(d_gate_up_data=None), INVALID),
    ("scale NULL", dict(d_gate_up_scale=None), INVALID),
    ("amax NULL", dict(amax=None), INVALID),
    ("amax misaligned", dict(amax=AMX + 2), MISAL),
    ("amax_given not 0, 1 or 2", dict(amax_given=3), INVALID),
    ("amax only with d_rw", dict(amax_given=2), INVALID),
    ("data overlaps grad_out", dict(d_gate_up_data=GO), INVALID),
    ("scales overlap gate_up", dict(d_gate_up_scale=GU + 64), INVALID),
    ("amax inside the data", dict(amax=MXD + 16), INVALID),
    ("d_rw overlaps amax", dict(d_rw=AMX), INVALID),
    ("grad_out pitch short", dict(grad_out_row_stride=32), INVALID),
    ("bad linear beta", dict(linear_beta=0.0), INVALID),
]


@pytest.mark.parametrize("name,kw,want", NV_BWD_CASES, ids=[c[0] for c in NV_BWD_CASES])
def test_bwd_nvfp4_argument_errors(name, kw, want, native_lib_path):
    assert bwd_nv(**kw) == want, abi.situ_glu_last_error()


# ---- FC1 grouped GEMM + SiTU-GLU: argument checks run before any CUDA call -------

XP, W1P, OFFP, YP = 0x20000000, 0x28000000, 0x30000000, 0x38000000


def fc1(**kw):
    a = dict(x=XP, tokens=256, hidden=128, x_row_stride=128, w1=W1P, experts=2, inter=128, w1_row_stride=128,
             offsets=OFFP, rw=RW, rw_dtype=F32, rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1,
             linear_beta=25.0, y=YP, y_row_stride=128, stream=None)
    a.update(kw)
    return abi.situ_glu_fc1_fwd(**a)


FC1_CASES = [
    ("hidden not a multiple of 64", dict(hidden=96, x_row_stride=96, w1_row_stride=96), UNSUP),
    ("inter not a multiple of 128", dict(inter=64, y_row_stride=64), UNSUP),
    ("no experts", dict(experts=0), UNSUP),
    ("too many experts", dict(experts=1025), UNSUP),
    ("per-column weights", dict(rw_mode=3), UNSUP),
    ("bad rw_mode", dict(rw_mode=9), INVALID),
    ("negative tokens", dict(tokens=-1), INVALID),
    ("x stride short", dict(x_row_stride=64), INVALID),
    ("w1 stride short", dict(w1_row_stride=64), INVALID),
    ("y stride short", dict(y_row_stride=64), INVALID),
    ("x NULL", dict(x=None), INVALID),
    ("offsets NULL", dict(offsets=None), INVALID),
    ("x misaligned", dict(x=XP + 8), MISAL),
    ("y pitch not 16-byte", dict(y_row_stride=132), MISAL),
    ("offsets misaligned", dict(offsets=OFFP + 4), MISAL),
    ("y overlaps x", dict(y=XP + 256), INVALID),
    ("y overlaps offsets", dict(y=OFFP - 64), INVALID),
    ("beta nan", dict(beta=float("nan")), INVALID),
    ("linear beta zero", dict(linear_beta=0.0), INVALID),
    ("rw with SITU_RW_NONE", dict(rw_mode=2), INVALID),
]


@pytest.mark.parametrize("name,kw,want", FC1_CASES, ids=[c[0] for c in FC1_CASES])
def test_fc1_argument_errors(name, kw, want, native_lib_path):
    assert fc1(**kw) == want, abi.situ_glu_last_error()


def test_fc1_zero_tokens_is_a_no_op(native_lib_path):
    assert fc1(tokens=0, x=None, offsets=None, y=None) == OK


# ---- attention-residual core: argument checks run before any CUDA call -------------

ARB, ARP, ARNW, ARPW, ARO = 0x40000000, 0x48000000, 0x50000000, 0x58000000, 0x60000000


def attn_res(**kw):
    a = dict(blocks=ARB, nblocks=8, block_row_stride=8 * 256, block_stride=256, prefix=ARP, prefix_row_stride=256,
             dtype=BF16, tokens=64, hidden=256, norm_weight=ARNW, norm_dtype=F32, proj_weight=ARPW, proj_dtype=F32,
             variance_epsilon=1e-6, out=ARO, out_dtype=BF16, out_row_stride=256, stream=None)
    a.update(kw)
    return abi.situ_attn_res_fwd(**a)


AR_CASES = [
    ("too many sources", dict(nblocks=16), UNSUP),
    ("no sources", dict(nblocks=0, prefix=None), UNSUP),
    ("negative blocks", dict(nblocks=-1), INVALID),
    ("hidden too large", dict(hidden=40000, block_stride=40000, block_row_stride=320000, prefix_row_stride=40000,
                              out_row_stride=40000), UNSUP),
    ("hidden not a 16-byte multiple", dict(hidden=100, block_stride=100, block_row_stride=800, prefix_row_stride=100,
                                           out_row_stride=100), MISAL),
    ("epsilon negative", dict(variance_epsilon=-1.0), INVALID),
    ("epsilon nan", dict(variance_epsilon=float("nan")), INVALID),
    ("source stride short", dict(block_stride=128), INVALID),
    ("out stride short", dict(out_row_stride=128), INVALID),
    ("bad dtype", dict(out_dtype=5), INVALID),
    ("blocks NULL", dict(blocks=None), INVALID),
    ("blocks misaligned", dict(blocks=ARB + 8), MISAL),
    ("source pitch not 16-byte", dict(block_stride=260, block_row_stride=8 * 260), MISAL),
    ("out overlaps blocks", dict(out=ARB + 512), INVALID),
    ("out overlaps the prefix", dict(out=ARP + 64), INVALID),
    # 8 sources 2^62 elements apart: nblocks * block_stride wraps in int64 (found by the randomised test)
    ("source extent overflows int64", dict(block_stride=2 ** 62), INVALID),
    ("row extent overflows int64", dict(block_row_stride=2 ** 62), INVALID),
]


@pytest.mark.parametrize("name,kw,want", AR_CASES, ids=[c[0] for c in AR_CASES])
def test_attn_res_argument_errors(name, kw, want, native_lib_path):
    assert attn_res(**kw) == want, abi.situ_glu_last_error()


def test_attn_res_zero_tokens_is_a_no_op(native_lib_path):
    assert attn_res(tokens=0, blocks=None, prefix=None, nblocks=0) == UNSUP  # still no source
    assert attn_res(tokens=0, blocks=None, out=None) == OK


# ---- FC2 data gradient + SiTU-GLU backward: argument checks ---------------------------

DOP, W2P, GUP, DGUP, DRWP, WSP = (0x70000000 + 0x01000000 * k for k in range(6))


def fc2(**kw):
    a = dict(dout=DOP, tokens=256, hidden=128, dout_row_stride=128, w2t=W2P, experts=2, inter=256,
             w2t_row_stride=128, offsets=OFFP, gate_up=GUP, gate_up_row_stride=512, rw=RW, rw_dtype=F32,
             rw_mode=ROW, rw_stride=1, beta=4.0, has_linear_beta=1, linear_beta=25.0, d_gate_up=DGUP,
             d_gate_up_row_stride=512, d_rw=DRWP, d_rw_stride=1, workspace=WSP, workspace_bytes=1 << 20,
             stream=None)
    a.update(kw)
    return abi.situ_glu_fc2_dgrad_bwd(**a)


FC2_CASES = [
    ("inter not a multiple of 256", dict(inter=128, gate_up_row_stride=256, d_gate_up_row_stride=256), UNSUP),
    ("hidden not a multiple of 64", dict(hidden=96, dout_row_stride=96, w2t_row_stride=96), UNSUP),
    ("broadcast weight", dict(rw_mode=SCALAR), UNSUP),
    ("d_rw with no weights", dict(rw_mode=NONE, rw=None), INVALID),
    ("workspace missing", dict(workspace=None, workspace_bytes=0), INVALID),
    ("workspace short", dict(workspace_bytes=16), INVALID),
    ("gate_up stride short", dict(gate_up_row_stride=256), INVALID),
    ("d_gate_up overlaps gate_up", dict(d_gate_up=GUP + 1024), INVALID),
    ("workspace overlaps dout", dict(workspace=DOP + 64), INVALID),
    ("dout misaligned", dict(dout=DOP + 4), MISAL),
    ("gate_up NULL", dict(gate_up=None), INVALID),
]


@pytest.mark.parametrize("name,kw,want", FC2_CASES, ids=[c[0] for c in FC2_CASES])
def test_fc2_argument_errors(name, kw, want, native_lib_path):
    assert fc2(**kw) == want, abi.situ_glu_last_error()


def test_fc2_workspace_query(native_lib_path):
    assert abi.situ_glu_fc2_dgrad_workspace_bytes(1000, 2048, 1) == (1000 * 8 * 4 + 255) // 256 * 256
    assert abi.situ_glu_fc2_dgrad_workspace_bytes(1000, 2048, 0) == 0
    assert abi.situ_glu_fc2_dgrad_workspace_bytes(0, 2048, 1) == 0


def _no_alloc_limit_from_header():
    text = open(os.path.join(ROOT, "include", "situ_glu.h")).read()
    doc = text[:text.index("situ_status_t situ_glu_bwd_no_alloc(")]
    doc = doc[doc.rindex("/*"):]
    flat = " ".join(re.sub(r"^\s*\*", " ", doc, flags=re.M).split())
    limit = int(re.search(r"1 MiB \((\d+)\)", flat).group(1))
    rows_scalar = int(re.search(r"at most (\d+) rows; ceil\(tokens / 16\) \* inter \* 4", flat).group(1))
    col_inter, col_rows = map(int, re.search(r"at inter = (\d+): at most (\d+) rows", flat).groups())
    return limit, rows_scalar, col_inter, col_rows


def test_no_alloc_limit_matches_the_workspace_query(native_lib_path):
    """The allocation-free backward's documented limit is exactly the bytes the
    workspace query reports at the boundary rows of both scratch modes, and one
    row more is rejected on the host (SITU_ERR_UNSUPPORTED, nothing launched)."""
    COL = abi.SITU_RW_COL
    limit, rows_scalar, col_inter, col_rows = _no_alloc_limit_from_header()
    assert limit == 1 << 20
    ws = abi.situ_glu_bwd_workspace_bytes
    assert ws(rows_scalar, 64, SCALAR, 1) == limit < ws(rows_scalar + 1, 64, SCALAR, 1)
    assert ws(col_rows, col_inter, COL, 1) == limit < ws(col_rows + 1, col_inter, COL, 1)
    assert col_rows == 16 * (limit // (col_inter * 4))

    def call(tokens, inter, mode):
        return abi.situ_glu_bwd_no_alloc(GU, BF16, tokens, inter, 2 * inter, RW, F32, mode, 1, 4.0, 1, 25.0,
                                         GO, inter, DGU, 2 * inter, DRW, 1, 0)

    # Only the rejected side is called: a size within the limit would go on to
    # the device.
    assert call(rows_scalar + 1, 64, SCALAR) == UNSUP
    assert "262144" in abi.situ_glu_last_error()
    assert call(col_rows + 1, col_inter, COL) == UNSUP
