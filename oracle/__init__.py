"""fp64 CPU oracle for the routing-weighted SiTU-GLU -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path
(``ffn_gated_activation_b200``) never imports it, and it never imports the
product path: the two share no code.

The arithmetic lives in ``situ_oracle.c`` and ``mx_oracle.c`` (plain C, IEEE
double, one element at a time); this module only builds them with gcc and
marshals numpy arrays through ctypes.

Sources followed (see the C file for the per-function citations):
  * Megatron-LM PR #6673 "[Dev] Add SiTU-GLU through Transformer Engine",
    section "Activation": T_g = b1 tanh(G/b1) sigmoid(G), T_u = b2 tanh(U/b2),
    Y = T_g T_u.
  * NeMo AutoModel API, kimi_k3.situ: `_situ_fwd_core` (Y = situ(g) up(u0) w,
    optional linear beta), `_situ_bwd_core` (analytic d_g, d_u and the
    routing-weight reduction), `_WeightedSiTUFunction` (gate/up halves).
  * Megatron-LM PR #6673, "Design": the fused grouped GEMM + SiTU-GLU, taken
    as FC1 (per-expert grouped GEMM) followed by the activation
    (fc1_oracle.c).
  * Megatron-LM PR #6673, "Test results" (the fused path's backward with a
    dSiTU correction): FC2's data gradient followed by the SiTU-GLU backward
    (fc2_oracle.c).
  * NeMo AutoModel API, kimi_k3.situ `_attn_res_core` / `_apply_attn_res`:
    the attention-residual mixing chain (attn_res_oracle.c).
  * OCP Microscaling Formats (MX) v1.0 for the MXFP8 outputs (E4M3 elements,
    E8M0 block scales, blocks of 32), the format of the MXFP8 recipe named in
    Megatron-LM PR #6673 "Test results".

Every function is pinned by tests/test_oracle_pins.py; no function here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "situ_oracle.c")
MX_SOURCE = os.path.join(_HERE, "mx_oracle.c")  # MXFP8 block scaling (OCP MX v1.0)
FC1_SOURCE = os.path.join(_HERE, "fc1_oracle.c")  # FC1 (grouped) followed by SiTU-GLU
ATTN_RES_SOURCE = os.path.join(_HERE, "attn_res_oracle.c")  # attention-residual mixing core
FC2_SOURCE = os.path.join(_HERE, "fc2_oracle.c")  # FC2 data gradient followed by the SiTU-GLU backward
SOURCES = [SOURCE, MX_SOURCE, FC1_SOURCE, ATTN_RES_SOURCE, FC2_SOURCE]
LIBRARY = os.path.join(_HERE, "libsitu_oracle.so")

DTYPE_BF16 = 0
DTYPE_F32 = 1
RW_ROW = 0     # w[T] (or [T, 1]): one weight per row
RW_SCALAR = 1  # one weight for every element
RW_COL = 2     # w[I]: one weight per column, every row
RW_FULL = 3    # w[T, I]: one weight per element
MX_BLOCK = 32         # MXFP8: elements per shared scale
MX_RULE_OCP = 0       # e = floor(log2 amax) - 8, elements clamped to +-448
MX_RULE_CEIL = 1      # smallest e with amax <= 448 * 2^e
MX_SCALE_NAN = 128    # mx_scale_exp's value for a NaN scale (scale byte 255)

# gcc flags: plain IEEE double, no fast-math, no contraction into FMA, so the
# arithmetic is exactly what the C source spells out.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(output: str = LIBRARY, mutant: int = 0, force: bool = False) -> str:
    """Compile situ_oracle.c with gcc into ``output``.  ``mutant`` > 0 builds a
    copy with the planted mistake number ``mutant`` (used only by the pin tests
    to show the pins reject it).  Rebuilds when the source is newer."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= max(os.path.getmtime(p) for p in SOURCES)):
        return output
    tmp = output + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, f"-DSITU_ORACLE_MUTANT={int(mutant)}", *SOURCES, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


_I64 = ctypes.c_int64
_INT = ctypes.c_int
_DBL = ctypes.c_double
_VP = ctypes.c_void_p


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_VP)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return DTYPE_BF16  # raw bf16 bit patterns
    if a.dtype == np.float32:
        return DTYPE_F32
    raise TypeError(f"oracle inputs are bf16 bit patterns (uint16) or float32, got {a.dtype}")


@dataclass
class BackwardResult:
    dg: np.ndarray   # [nrows, inter] float64, dL/dG
    du: np.ndarray   # [nrows, inter] float64, dL/dU
    dw: np.ndarray   # [nrows] float64, per-row routing-weight gradient
    cg: np.ndarray   # [nrows, inter] float64, uncancelled magnitude of dG
    sw: np.ndarray   # [nrows] float64, sum of |go T_g T_u| per row


class Oracle:
    """ctypes handle on one build of situ_oracle.c (the oracle, or a mutant)."""

    def __init__(self, path: str = LIBRARY):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.situ_oracle_gate.argtypes = [_DBL, _DBL, ctypes.POINTER(_DBL), ctypes.POINTER(_DBL), ctypes.POINTER(_DBL)]
        lib.situ_oracle_gate.restype = None
        lib.situ_oracle_up.argtypes = [_DBL, _INT, _DBL, ctypes.POINTER(_DBL), ctypes.POINTER(_DBL)]
        lib.situ_oracle_up.restype = None
        lib.situ_oracle_gate_n.argtypes = [_I64, _VP, _DBL, _VP, _VP, _VP]
        lib.situ_oracle_gate_n.restype = None
        lib.situ_oracle_up_n.argtypes = [_I64, _VP, _INT, _DBL, _VP, _VP]
        lib.situ_oracle_up_n.restype = None
        lib.situ_oracle_fwd.argtypes = [_INT, _VP, _I64, _I64, _VP, _I64, _INT, _VP, _INT, _I64,
                                        _DBL, _INT, _DBL, _VP]
        lib.situ_oracle_fwd.restype = _INT
        lib.situ_oracle_bwd.argtypes = [_INT, _VP, _I64, _I64, _VP, _I64, _INT, _VP, _INT, _I64,
                                        _DBL, _INT, _DBL, _VP, _I64, _VP, _VP, _VP, _VP, _VP]
        lib.situ_oracle_bwd.restype = _INT
        lib.situ_oracle_dw_scalar.argtypes = [_INT, _VP, _I64, _I64, _I64, _DBL, _INT, _DBL, _VP, _I64,
                                              ctypes.POINTER(_DBL), ctypes.POINTER(_DBL)]
        lib.situ_oracle_dw_scalar.restype = _INT
        lib.situ_oracle_dw_columns.argtypes = [_INT, _VP, _I64, _I64, _I64, _DBL, _INT, _DBL, _VP, _I64, _VP, _VP]
        lib.situ_oracle_dw_columns.restype = _INT
        lib.situ_oracle_dw_terms.argtypes = [_INT, _VP, _I64, _I64, _VP, _I64, _DBL, _INT, _DBL, _VP, _I64, _VP]
        lib.situ_oracle_dw_terms.restype = _INT
        lib.situ_oracle_mutant_id.restype = _INT
        lib.situ_oracle_e4m3_encode.argtypes = [_DBL]
        lib.situ_oracle_e4m3_encode.restype = _INT
        lib.situ_oracle_e4m3_encode_n.argtypes = [_VP, _I64, _VP]
        lib.situ_oracle_e4m3_encode_n.restype = None
        lib.situ_oracle_e4m3_decode.argtypes = [_INT]
        lib.situ_oracle_e4m3_decode.restype = _DBL
        lib.situ_oracle_mx_scale_exp.argtypes = [_DBL, _INT]
        lib.situ_oracle_mx_scale_exp.restype = _INT
        lib.situ_oracle_mxfp8_quantize.argtypes = [_VP, _I64, _I64, _I64, _INT, _VP, _VP]
        lib.situ_oracle_mxfp8_quantize.restype = _INT
        lib.situ_oracle_e2m1_encode.argtypes = [_DBL]
        lib.situ_oracle_e2m1_encode.restype = _INT
        lib.situ_oracle_e2m1_encode_n.argtypes = [_VP, _I64, _VP]
        lib.situ_oracle_e2m1_encode_n.restype = None
        lib.situ_oracle_e2m1_decode.argtypes = [_INT]
        lib.situ_oracle_e2m1_decode.restype = _DBL
        lib.situ_oracle_nvfp4_tensor_scale.argtypes = [_DBL]
        lib.situ_oracle_nvfp4_tensor_scale.restype = _DBL
        lib.situ_oracle_nvfp4_quantize.argtypes = [_VP, _I64, _I64, _I64, _DBL, _VP, _VP]
        lib.situ_oracle_nvfp4_quantize.restype = _INT
        lib.situ_oracle_fc1_fwd.argtypes = [_VP, _I64, _I64, _VP, _I64, _I64, _VP, _I64, _VP, _I64, _VP,
                                            _DBL, _INT, _DBL, _VP, _VP, _VP]
        lib.situ_oracle_fc1_fwd.restype = _INT
        lib.situ_oracle_attn_res.argtypes = [_VP, _I64, _I64, _I64, _VP, _I64, _INT, _I64, _VP, _INT, _VP, _INT,
                                             _DBL, _VP, _I64, _VP, _VP, _VP]
        lib.situ_oracle_attn_res.restype = _INT
        lib.situ_oracle_fc2_dgrad.argtypes = [_VP, _I64, _I64, _VP, _I64, _I64, _VP, _I64, _VP, _I64, _VP, _DBL, _INT,
                                              _DBL, _VP, _I64, _VP, _VP, _VP, _VP, _VP]
        lib.situ_oracle_fc2_dgrad.restype = _INT
        self._lib = lib
        self.mutant_id = lib.situ_oracle_mutant_id()

    # -- scalar branches -----------------------------------------------------
    def gate(self, g, beta):
        """T_g, T_g' and the uncancelled magnitude of T_g' at each g (float64)."""
        g = np.ascontiguousarray(np.atleast_1d(np.asarray(g, dtype=np.float64)))
        t, d, m = (np.empty_like(g) for _ in range(3))
        self._lib.situ_oracle_gate_n(g.size, _ptr(g), float(beta), _ptr(t), _ptr(d), _ptr(m))
        return t, d, m

    def up(self, u, linear_beta):
        """T_u and T_u' at each u; linear_beta None means T_u = u."""
        u = np.ascontiguousarray(np.atleast_1d(np.asarray(u, dtype=np.float64)))
        t, d = np.empty_like(u), np.empty_like(u)
        has = linear_beta is not None
        self._lib.situ_oracle_up_n(u.size, _ptr(u), int(has), float(linear_beta if has else 0.0),
                                   _ptr(t), _ptr(d))
        return t, d

    # -- rows ------------------------------------------------------------------
    @staticmethod
    def _rows(rows, n_all):
        if rows is None:
            return None, n_all
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        if r.size and (r.min() < 0 or r.max() >= n_all):
            raise IndexError("row index out of range")
        return r, r.size

    def fwd(self, gate_up, rw, beta, linear_beta=None, rows=None, rw_mode=RW_ROW, inter=None):
        """Y (float64, [nrows, inter]) for the selected rows of gate_up [T, >= 2I].
        rw is float32 or bf16 bits: [T] / [T, 1] (row mode) or one value (scalar)."""
        gate_up = np.ascontiguousarray(gate_up)
        T, width = gate_up.shape
        inter = width // 2 if inter is None else int(inter)
        r, n = self._rows(rows, T)
        rw_c = np.ascontiguousarray(rw).reshape(-1)
        rw_stride = inter if rw_mode == RW_FULL else 1
        y = np.empty((n, inter), dtype=np.float64)
        has = linear_beta is not None
        rc = self._lib.situ_oracle_fwd(_dtype_code(gate_up), _ptr(gate_up), width, inter, _ptr(r), n,
                                       _dtype_code(rw_c), _ptr(rw_c), int(rw_mode), rw_stride,
                                       float(beta), int(has), float(linear_beta if has else 0.0), _ptr(y))
        if rc != 0:
            raise ValueError("oracle fwd rejected its arguments")
        return y

    def bwd(self, gate_up, rw, grad_out, beta, linear_beta=None, rows=None, rw_mode=RW_ROW, inter=None):
        """Analytic backward for the selected rows; grad_out is [T, >= I] in
        gate_up's dtype.  Returns a BackwardResult of float64 arrays."""
        gate_up = np.ascontiguousarray(gate_up)
        grad_out = np.ascontiguousarray(grad_out)
        if grad_out.dtype != gate_up.dtype:
            raise TypeError("grad_out must have gate_up's dtype")
        T, width = gate_up.shape
        inter = width // 2 if inter is None else int(inter)
        r, n = self._rows(rows, T)
        rw_c = np.ascontiguousarray(rw).reshape(-1)
        rw_stride = inter if rw_mode == RW_FULL else 1
        dg = np.empty((n, inter)); du = np.empty((n, inter)); cg = np.empty((n, inter))
        dw = np.empty(n); sw = np.empty(n)
        has = linear_beta is not None
        rc = self._lib.situ_oracle_bwd(_dtype_code(gate_up), _ptr(gate_up), width, inter, _ptr(r), n,
                                       _dtype_code(rw_c), _ptr(rw_c), int(rw_mode), rw_stride,
                                       float(beta), int(has), float(linear_beta if has else 0.0),
                                       _ptr(grad_out), grad_out.shape[1],
                                       _ptr(dg), _ptr(du), _ptr(dw), _ptr(cg), _ptr(sw))
        if rc != 0:
            raise ValueError("oracle bwd rejected its arguments")
        return BackwardResult(dg=dg, du=du, dw=dw, cg=cg, sw=sw)

    def dw_columns(self, gate_up, grad_out, beta, linear_beta=None, inter=None):
        """Gradient of a per-column weight w[I]: (sums over rows [I], sums of |terms| [I])."""
        gate_up = np.ascontiguousarray(gate_up)
        grad_out = np.ascontiguousarray(grad_out)
        T, width = gate_up.shape
        inter = width // 2 if inter is None else int(inter)
        colsum, colmag = np.empty(inter), np.empty(inter)
        has = linear_beta is not None
        rc = self._lib.situ_oracle_dw_columns(_dtype_code(gate_up), _ptr(gate_up), width, inter, T,
                                              float(beta), int(has), float(linear_beta if has else 0.0),
                                              _ptr(grad_out), grad_out.shape[1], _ptr(colsum), _ptr(colmag))
        if rc != 0:
            raise ValueError("oracle dw_columns rejected its arguments")
        return colsum, colmag

    def dw_terms(self, gate_up, grad_out, beta, linear_beta=None, rows=None, inter=None):
        """Gradient of a full [T, I] weight for the selected rows: go T_g T_u, float64."""
        gate_up = np.ascontiguousarray(gate_up)
        grad_out = np.ascontiguousarray(grad_out)
        T, width = gate_up.shape
        inter = width // 2 if inter is None else int(inter)
        r, n = self._rows(rows, T)
        terms = np.empty((n, inter))
        has = linear_beta is not None
        rc = self._lib.situ_oracle_dw_terms(_dtype_code(gate_up), _ptr(gate_up), width, inter, _ptr(r), n,
                                            float(beta), int(has), float(linear_beta if has else 0.0),
                                            _ptr(grad_out), grad_out.shape[1], _ptr(terms))
        if rc != 0:
            raise ValueError("oracle dw_terms rejected its arguments")
        return terms

    def dw_scalar(self, gate_up, grad_out, beta, linear_beta=None, inter=None):
        """Gradient of one routing weight broadcast to all rows: (total, sum of |terms|)."""
        gate_up = np.ascontiguousarray(gate_up)
        grad_out = np.ascontiguousarray(grad_out)
        T, width = gate_up.shape
        inter = width // 2 if inter is None else int(inter)
        total, mag = _DBL(), _DBL()
        has = linear_beta is not None
        rc = self._lib.situ_oracle_dw_scalar(_dtype_code(gate_up), _ptr(gate_up), width, inter, T,
                                             float(beta), int(has), float(linear_beta if has else 0.0),
                                             _ptr(grad_out), grad_out.shape[1],
                                             ctypes.byref(total), ctypes.byref(mag))
        if rc != 0:
            raise ValueError("oracle dw_scalar rejected its arguments")
        return total.value, mag.value


    # -- MXFP8 block scaling (mx_oracle.c) -------------------------------------

    def e4m3_encode(self, x) -> np.ndarray:
        """E4M3 codes (uint8) of reals x: nearest-even, clamped to +-448."""
        x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        out = np.empty(x.shape, dtype=np.uint8)
        self._lib.situ_oracle_e4m3_encode_n(_ptr(x), x.size, _ptr(out))
        return out

    def e4m3_decode(self, codes) -> np.ndarray:
        c = np.asarray(codes, dtype=np.uint8)
        f = self._lib.situ_oracle_e4m3_decode
        return np.array([f(int(v)) for v in c.reshape(-1)], dtype=np.float64).reshape(c.shape)

    def mx_scale_exp(self, amax: float, rule: int = MX_RULE_OCP) -> int:
        """Shared exponent of a block with largest magnitude amax (MX_SCALE_NAN for NaN)."""
        return self._lib.situ_oracle_mx_scale_exp(float(amax), int(rule))

    def mxfp8_quantize(self, v, rule: int = MX_RULE_OCP):
        """(codes [R, C] uint8, scale bytes [R, C / 32] uint8) of the fp64 matrix v."""
        v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
        rows, cols = v.shape
        codes = np.empty((rows, cols), dtype=np.uint8)
        scales = np.empty((rows, cols // MX_BLOCK), dtype=np.uint8)
        rc = self._lib.situ_oracle_mxfp8_quantize(_ptr(v), rows, cols, cols, int(rule), _ptr(codes), _ptr(scales))
        if rc != 0:
            raise ValueError("oracle mxfp8_quantize: columns must be a multiple of 32")
        return codes, scales


    # -- NVFP4 (mx_oracle.c) ----------------------------------------------------

    def e2m1_encode(self, x) -> np.ndarray:
        """E2M1 codes (sign << 3 | magnitude code, uint8) of reals x: nearest-even, clamped to +-6."""
        x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        out = np.empty(x.shape, dtype=np.uint8)
        self._lib.situ_oracle_e2m1_encode_n(_ptr(x), x.size, _ptr(out))
        return out

    def e2m1_decode(self, codes) -> np.ndarray:
        c = np.asarray(codes, dtype=np.uint8)
        f = self._lib.situ_oracle_e2m1_decode
        return np.array([f(int(v)) for v in c.reshape(-1)], dtype=np.float64).reshape(c.shape)

    def nvfp4_tensor_scale(self, amax: float) -> float:
        return self._lib.situ_oracle_nvfp4_tensor_scale(float(amax))

    def nvfp4_quantize(self, v, s_enc=None):
        """(codes [R, C] one 4-bit code per byte, block scale codes [R, C / 16]
        E4M3, s_enc) of the fp64 matrix v; s_enc defaults to the tensor's own."""
        v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
        if s_enc is None:
            fin = v[np.isfinite(v)]
            s_enc = self.nvfp4_tensor_scale(float(np.abs(fin).max()) if fin.size else 0.0)
        rows, cols = v.shape
        codes = np.empty((rows, cols), dtype=np.uint8)
        scales = np.empty((rows, cols // 16), dtype=np.uint8)
        rc = self._lib.situ_oracle_nvfp4_quantize(_ptr(v), rows, cols, cols, float(s_enc), _ptr(codes), _ptr(scales))
        if rc != 0:
            raise ValueError("oracle nvfp4_quantize: columns must be a multiple of 16")
        return codes, scales, s_enc

    # -- FC1 followed by SiTU-GLU (fc1_oracle.c) ------------------------------

    def fc1_fwd(self, x, w1, offsets, inter, rw, beta, linear_beta=None, rows=None):
        """(Y [nrows, I], error scale [nrows, I], unrounded gate_up [nrows, 2I]),
        all float64, for token rows of x (bf16 bits [T, H]) routed by
        ``offsets`` [E + 1] to experts whose FC1 weights are w1 (bf16 bits
        [E * 2I, H]: per expert I gate rows, then I up rows).  rw: float32 [T]
        per-row routing weights, or None for w = 1."""
        x = np.ascontiguousarray(x)
        w1 = np.ascontiguousarray(w1)
        if x.dtype != np.uint16 or w1.dtype != np.uint16:
            raise TypeError("x and w1 are bf16 bit patterns (uint16)")
        off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
        T, hidden = x.shape
        r, n = self._rows(rows, T)
        rw_c = None if rw is None else np.ascontiguousarray(np.asarray(rw, dtype=np.float32).reshape(-1))
        y = np.empty((n, inter))
        err = np.empty((n, inter))
        gu = np.empty((n, 2 * inter))
        has = linear_beta is not None
        rc = self._lib.situ_oracle_fc1_fwd(_ptr(x), x.shape[1], hidden, _ptr(w1), w1.shape[1], int(inter), _ptr(off),
                                           off.size - 1, _ptr(r), n, _ptr(rw_c), float(beta), int(has),
                                           float(linear_beta if has else 0.0), _ptr(y), _ptr(err), _ptr(gu))
        if rc != 0:
            raise ValueError("oracle fc1_fwd rejected its arguments")
        return y, err, gu


    # -- attention-residual mixing core (attn_res_oracle.c) -------------------

    def attn_res(self, blocks, prefix, norm_weight, proj_weight, eps, rows=None):
        """(out [nrows, H], combine magnitude [nrows, H], prob [nrows, S]) in
        float64.  blocks: [T, B, H] stored sums (bf16 bits or float32) or None;
        prefix: [T, H] current sum (same dtype) or None -- appended as the last
        source.  norm_weight, proj_weight: [H] float32 or bf16 bits."""
        if blocks is None and prefix is None:
            raise ValueError("no sources")
        ref = blocks if blocks is not None else prefix
        dtype = _dtype_code(np.asarray(ref))
        blocks_c = None if blocks is None else np.ascontiguousarray(blocks)
        prefix_c = None if prefix is None else np.ascontiguousarray(prefix)
        if blocks_c is not None and prefix_c is not None and blocks_c.dtype != prefix_c.dtype:
            raise TypeError("blocks and prefix must share a dtype")
        T = (blocks_c if blocks_c is not None else prefix_c).shape[0]
        H = (blocks_c if blocks_c is not None else prefix_c).shape[-1]
        nb = 0 if blocks_c is None else blocks_c.shape[1]
        nw = np.ascontiguousarray(norm_weight)
        pw = np.ascontiguousarray(proj_weight)
        r, n = self._rows(rows, T)
        S = nb + (prefix_c is not None)
        out = np.empty((n, H))
        mag = np.empty((n, H))
        prob = np.empty((n, S))
        rc = self._lib.situ_oracle_attn_res(_ptr(blocks_c), nb, nb * H, H, _ptr(prefix_c), H, dtype, H, _ptr(nw),
                                            _dtype_code(nw), _ptr(pw), _dtype_code(pw), float(eps), _ptr(r), n,
                                            _ptr(out), _ptr(mag), _ptr(prob))
        if rc != 0:
            raise ValueError("oracle attn_res rejected its arguments")
        return out, mag, prob


    # -- FC2 data gradient + SiTU-GLU backward (fc2_oracle.c) -----------------

    def fc2_dgrad(self, dout, w2t, offsets, gate_up, rw, beta, linear_beta=None, rows=None):
        """(d_gate_up [n, 2I], d_w [n], dY [n, I], error scales [n, 2I], d_w error
        scales [n]) in float64 for token rows of dout (bf16 bits [T, H]) routed by
        ``offsets`` to experts with transposed FC2 weights w2t (bf16 bits
        [E * I, H]); gate_up: the saved bf16 bits [T, 2I]; rw: float32 [T] or None."""
        dout = np.ascontiguousarray(dout)
        w2t = np.ascontiguousarray(w2t)
        gate_up = np.ascontiguousarray(gate_up)
        for a in (dout, w2t, gate_up):
            if a.dtype != np.uint16:
                raise TypeError("dout, w2t and gate_up are bf16 bit patterns (uint16)")
        off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
        T, hidden = dout.shape
        inter = gate_up.shape[1] // 2
        r, n = self._rows(rows, T)
        rw_c = None if rw is None else np.ascontiguousarray(np.asarray(rw, dtype=np.float32).reshape(-1))
        dgu = np.empty((n, 2 * inter))
        dw = np.empty(n)
        dy = np.empty((n, inter))
        err = np.empty((n, 2 * inter))
        dw_err = np.empty(n)
        has = linear_beta is not None
        rc = self._lib.situ_oracle_fc2_dgrad(_ptr(dout), dout.shape[1], hidden, _ptr(w2t), w2t.shape[1], inter,
                                             _ptr(off), off.size - 1, _ptr(gate_up), gate_up.shape[1], _ptr(rw_c),
                                             float(beta), int(has), float(linear_beta if has else 0.0), _ptr(r), n,
                                             _ptr(dgu), _ptr(dw), _ptr(dy), _ptr(err), _ptr(dw_err))
        if rc != 0:
            raise ValueError("oracle fc2_dgrad rejected its arguments")
        return dgu, dw, dy, err, dw_err


_DEFAULT = None


def load(path: str | None = None) -> Oracle:
    """The oracle (built on first use if the shared object is missing or stale)."""
    global _DEFAULT
    if path is not None:
        return Oracle(path)
    if _DEFAULT is None:
        build()
        _DEFAULT = Oracle(LIBRARY)
    return _DEFAULT
