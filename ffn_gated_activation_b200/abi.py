"""ctypes declarations of libsitu_glu.so, one Python callable per C entry point.

Every function here has the name, argument order and meaning of its
declaration in include/situ_glu.h (pointers are passed as integers).  Nothing
is computed in Python.  The library is loaded on first use; if it has not been
built the call raises ``NativeLibraryError`` -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import _build

SITU_OK = 0
SITU_ERR_INVALID_ARG = 1
SITU_ERR_UNSUPPORTED = 2
SITU_ERR_MISALIGNED = 3
SITU_ERR_CUDA = 4

SITU_DTYPE_BF16 = 0
SITU_DTYPE_F32 = 1

SITU_RW_ROW = 0
SITU_RW_SCALAR = 1
SITU_RW_NONE = 2
SITU_RW_COL = 3
SITU_RW_FULL = 4

SITU_MX_RULE_OCP = 0
SITU_MX_RULE_CEIL = 1

ABI_VERSION = 8

# Entry points declared in include/situ_glu.h: name -> (restype, argtypes).
_I64, _INT, _DBL, _VP, _SZ = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "situ_glu_fwd": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                            _VP, _I64, _VP]),
    "situ_glu_bwd": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                            _VP, _I64, _VP, _I64, _VP, _I64, _VP, _SZ, _VP]),
    "situ_glu_fwd_mxfp8": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                                  _VP, _I64, _VP, _I64, _INT, _VP]),
    "situ_glu_bwd_mxfp8": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                                  _VP, _I64, _VP, _I64, _VP, _I64, _INT, _VP, _I64, _VP, _SZ, _VP]),
    "situ_glu_fwd_nvfp4": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                                  _VP, _I64, _VP, _I64, _VP, _INT, _VP]),
    "situ_glu_bwd_nvfp4": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                                  _VP, _I64, _VP, _I64, _VP, _I64, _VP, _INT, _VP, _I64, _VP, _SZ, _VP]),
    "situ_glu_fc1_fwd": (_INT, [_VP, _I64, _I64, _I64, _VP, _I64, _I64, _I64, _VP, _VP, _INT, _INT, _I64,
                                _DBL, _INT, _DBL, _VP, _I64, _VP]),
    "situ_glu_fc2_dgrad_bwd": (_INT, [_VP, _I64, _I64, _I64, _VP, _I64, _I64, _I64, _VP, _VP, _I64, _VP, _INT, _INT,
                                      _I64, _DBL, _INT, _DBL, _VP, _I64, _VP, _I64, _VP, _SZ, _VP]),
    "situ_glu_fc2_dgrad_workspace_bytes": (_SZ, [_I64, _I64, _INT]),
    "situ_attn_res_fwd": (_INT, [_VP, _I64, _I64, _I64, _VP, _I64, _INT, _I64, _I64, _VP, _INT, _VP, _INT, _DBL,
                                 _VP, _INT, _I64, _VP]),
    "situ_glu_bwd_workspace_bytes": (_SZ, [_I64, _I64, _INT, _INT]),
    "situ_glu_status_string": (ctypes.c_char_p, [_INT]),
    "situ_glu_last_error": (ctypes.c_char_p, []),
    "situ_glu_abi_version": (_INT, []),
    "situ_glu_set_max_ctas": (_INT, [_INT]),
    "situ_glu_set_load_path": (_INT, [_INT]),
    "situ_glu_device_status": (_INT, [_INT]),
    "situ_glu_wait_probe": (_INT, [_I64, _VP]),
    "situ_glu_bwd_no_alloc": (_INT, [_VP, _INT, _I64, _I64, _I64, _VP, _INT, _INT, _I64, _DBL, _INT, _DBL,
                                     _VP, _I64, _VP, _I64, _VP, _I64, _VP]),
}


class NativeLibraryError(RuntimeError):
    """The native library is missing, stale or does not match this binding."""


class SituError(RuntimeError):
    """A non-OK status returned by the library."""

    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}: {detail}")


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return os.environ.get("SITU_GLU_LIBRARY", _build.LIBRARY)


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once, on first use)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise NativeLibraryError(
                    f"{path} is not built; run `python -m ffn_gated_activation_b200._build` "
                    "(or __graft_entry__.build()) -- there is no fallback implementation")
            handle = ctypes.CDLL(path)
            for name, (restype, argtypes) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = restype
                fn.argtypes = argtypes
            if handle.situ_glu_abi_version() != ABI_VERSION:
                raise NativeLibraryError(f"{path}: ABI {handle.situ_glu_abi_version()} != {ABI_VERSION}")
            _lib = handle
    return _lib


def situ_glu_fwd(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride,
                 beta, has_linear_beta, linear_beta, out, out_row_stride, stream) -> int:
    return lib().situ_glu_fwd(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                              rw_stride, beta, has_linear_beta, linear_beta, out, out_row_stride, stream)


def situ_glu_bwd(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride,
                 beta, has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up,
                 d_gate_up_row_stride, d_rw, d_rw_stride, workspace, workspace_bytes, stream) -> int:
    return lib().situ_glu_bwd(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                              rw_stride, beta, has_linear_beta, linear_beta, grad_out,
                              grad_out_row_stride, d_gate_up, d_gate_up_row_stride, d_rw, d_rw_stride,
                              workspace, workspace_bytes, stream)


def situ_glu_fwd_mxfp8(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride,
                       beta, has_linear_beta, linear_beta, y_data, y_data_row_stride, y_scale,
                       y_scale_row_stride, rule, stream) -> int:
    return lib().situ_glu_fwd_mxfp8(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                    rw_stride, beta, has_linear_beta, linear_beta, y_data, y_data_row_stride,
                                    y_scale, y_scale_row_stride, rule, stream)


def situ_glu_bwd_mxfp8(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride,
                       beta, has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up_data,
                       d_gate_up_data_row_stride, d_gate_up_scale, d_gate_up_scale_row_stride, rule, d_rw,
                       d_rw_stride, workspace, workspace_bytes, stream) -> int:
    return lib().situ_glu_bwd_mxfp8(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                    rw_stride, beta, has_linear_beta, linear_beta, grad_out,
                                    grad_out_row_stride, d_gate_up_data, d_gate_up_data_row_stride,
                                    d_gate_up_scale, d_gate_up_scale_row_stride, rule, d_rw, d_rw_stride,
                                    workspace, workspace_bytes, stream)


def situ_glu_fwd_nvfp4(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                       has_linear_beta, linear_beta, y_data, y_data_row_stride, y_scale, y_scale_row_stride, amax,
                       amax_given, stream) -> int:
    return lib().situ_glu_fwd_nvfp4(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                    rw_stride, beta, has_linear_beta, linear_beta, y_data, y_data_row_stride, y_scale,
                                    y_scale_row_stride, amax, amax_given, stream)


def situ_glu_bwd_nvfp4(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                       has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up_data,
                       d_gate_up_data_row_stride, d_gate_up_scale, d_gate_up_scale_row_stride, amax, amax_given,
                       d_rw, d_rw_stride, workspace, workspace_bytes, stream) -> int:
    return lib().situ_glu_bwd_nvfp4(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                    rw_stride, beta, has_linear_beta, linear_beta, grad_out, grad_out_row_stride,
                                    d_gate_up_data, d_gate_up_data_row_stride, d_gate_up_scale,
                                    d_gate_up_scale_row_stride, amax, amax_given, d_rw, d_rw_stride, workspace,
                                    workspace_bytes, stream)


def situ_glu_fc1_fwd(x, tokens, hidden, x_row_stride, w1, experts, inter, w1_row_stride, offsets, rw, rw_dtype,
                     rw_mode, rw_stride, beta, has_linear_beta, linear_beta, y, y_row_stride, stream) -> int:
    return lib().situ_glu_fc1_fwd(x, tokens, hidden, x_row_stride, w1, experts, inter, w1_row_stride, offsets, rw,
                                  rw_dtype, rw_mode, rw_stride, beta, has_linear_beta, linear_beta, y, y_row_stride,
                                  stream)


def situ_glu_fc2_dgrad_bwd(dout, tokens, hidden, dout_row_stride, w2t, experts, inter, w2t_row_stride, offsets,
                           gate_up, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta, has_linear_beta,
                           linear_beta, d_gate_up, d_gate_up_row_stride, d_rw, d_rw_stride, workspace,
                           workspace_bytes, stream) -> int:
    return lib().situ_glu_fc2_dgrad_bwd(dout, tokens, hidden, dout_row_stride, w2t, experts, inter, w2t_row_stride,
                                        offsets, gate_up, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                                        has_linear_beta, linear_beta, d_gate_up, d_gate_up_row_stride, d_rw,
                                        d_rw_stride, workspace, workspace_bytes, stream)


def situ_glu_fc2_dgrad_workspace_bytes(tokens, inter, want_drw) -> int:
    return lib().situ_glu_fc2_dgrad_workspace_bytes(tokens, inter, want_drw)


def situ_attn_res_fwd(blocks, nblocks, block_row_stride, block_stride, prefix, prefix_row_stride, dtype, tokens,
                      hidden, norm_weight, norm_dtype, proj_weight, proj_dtype, variance_epsilon, out, out_dtype,
                      out_row_stride, stream) -> int:
    return lib().situ_attn_res_fwd(blocks, nblocks, block_row_stride, block_stride, prefix, prefix_row_stride, dtype,
                                   tokens, hidden, norm_weight, norm_dtype, proj_weight, proj_dtype, variance_epsilon,
                                   out, out_dtype, out_row_stride, stream)


def situ_glu_bwd_no_alloc(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride,
                          beta, has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up,
                          d_gate_up_row_stride, d_rw, d_rw_stride, stream) -> int:
    """situ_glu_bwd without caller scratch (the library's fixed scratch; see
    include/situ_glu.h for its row limit and sharing rules)."""
    return lib().situ_glu_bwd_no_alloc(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                       rw_stride, beta, has_linear_beta, linear_beta, grad_out,
                                       grad_out_row_stride, d_gate_up, d_gate_up_row_stride, d_rw, d_rw_stride,
                                       stream)


def situ_glu_bwd_workspace_bytes(tokens, inter, rw_mode, want_drw) -> int:
    return lib().situ_glu_bwd_workspace_bytes(tokens, inter, rw_mode, want_drw)


def situ_glu_status_string(status) -> str:
    return lib().situ_glu_status_string(status).decode()


def situ_glu_last_error() -> str:
    return lib().situ_glu_last_error().decode()


def situ_glu_abi_version() -> int:
    return lib().situ_glu_abi_version()


def situ_glu_set_max_ctas(max_ctas) -> int:
    return lib().situ_glu_set_max_ctas(max_ctas)


def situ_glu_wait_probe(limit_ns, stream=None) -> int:
    return lib().situ_glu_wait_probe(int(limit_ns), stream)


def situ_glu_set_load_path(path) -> int:
    return lib().situ_glu_set_load_path(path)


def situ_glu_device_status(clear) -> int:
    return lib().situ_glu_device_status(clear)


def status_string(status: int) -> str:
    return situ_glu_status_string(status)


def check(status: int, where: str) -> None:
    """Raise SituError for a non-OK status, with the library's own detail."""
    if status != SITU_OK:
        raise SituError(status, where, situ_glu_last_error())
