"""Pins for the fp64 oracle (CPU only).

The oracle is the definition the CUDA path is checked against, so it is
itself checked here against things other than itself:

  * 50-digit mpmath values of the two branch functions, and mpmath's
    numerical derivative of them (independent of the analytic derivative);
  * exact identities that follow from sigmoid(x) + sigmoid(-x) = 1:
        T_g(g) - T_g(-g) = beta tanh(g / beta)
        T_g(g) + T_g(-g) = beta tanh(g / beta) tanh(g / 2);
  * the SwiGLU limit beta, beta_L -> infinity against torch's library SiLU
    and its autograd derivative ("unary F.silu is not equivalent" -- the
    Megatron-LM PR #6673 "Design" list -- holds only at finite beta);
  * central finite differences of the oracle's own forward;
  * torch float64 autograd of the formula for whole rows (independent
    derivatives, strided rows, both dtypes, both routing-weight modes);
  * special rows (G = 0, U = 0) whose gradients have closed forms;
  * brute-force compensated sums for the routing-weight gradient;
  * MXFP8 (mx_oracle.c): torch's float8_e4m3fn encoding and decoding, the
    OCP MX format's clamp at 448, and the scale rules' defining inequalities;
  * FC1 + SiTU-GLU (fc1_oracle.c): fsum dot products and 50-digit element
    values, exact agreement with the activation oracle on bf16-exact FC1
    outputs, and the grouped call against per-expert calls;
  * FC2 data gradient + SiTU-GLU backward (fc2_oracle.c): fsum dot products
    with 50-digit derivatives, exact agreement with the activation backward
    on bf16-exact dY, per-expert calls;
  * attention-residual core (attn_res_oracle.c): torch's float64 rms_norm and
    softmax, invariants (identical sources, zero projection, one source,
    scaling), large logits, and the two-array source layout.

Each pin is a plain function of an oracle handle.  ``test_mutant_rejected``
rebuilds situ_oracle.c with each planted mistake (-DSITU_ORACLE_MUTANT=n: a
dropped term, a wrong sign, a transposed operand, swapped halves, an ignored
stride, ...) and checks that at least one pin rejects it.
"""
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
import workloads

mpmath.mp.dps = 50
RNG_SEED = 12345


# ---- high-precision restatements (mpmath, 50 digits) --------------------------

def _mp_gate(g, beta):
    g = mpmath.mpf(g)
    return beta * mpmath.tanh(g / beta) / (1 + mpmath.exp(-g))


def _mp_up(u, lb):
    return lb * mpmath.tanh(mpmath.mpf(u) / lb)


def _mp_diff(f, x):
    """mpmath's numerical derivative at 400 working digits: enough that a slope
    as small as 1e-174 next to function values near 1 keeps its double digits."""
    with mpmath.workdps(400):
        return float(mpmath.diff(f, mpmath.mpf(x)))


def _close(a, b, rtol, atol=0.0):
    return abs(a - b) <= rtol * abs(b) + atol


# ---- pins ------------------------------------------------------------------------

def pin_gate_values_mpmath(o):
    """T_g and T_g' against 50-digit values, including saturation at |g| = 20, 60
    (the fixed-value coverage asked for in the Megatron-LM PR #6673 review)."""
    pts = [0.0, 0.5, -0.5, 1.0, -1.0, 4.0, -4.0, 20.0, -20.0, 60.0, -60.0, 7.3, -7.3,
           1e-6, -1e-6, -1.2187557268720125, 2.5e-3, -33.0]
    for beta in (1.0, 4.0, 16.0):
        t, d, m = o.gate(pts, beta)
        for k, g in enumerate(pts):
            ref = float(_mp_gate(g, beta))
            assert _close(t[k], ref, 4e-15, 1e-300), (beta, g, t[k], ref)
            dref = _mp_diff(lambda x: _mp_gate(x, beta), g)
            assert abs(d[k] - dref) <= 1e-14 * m[k] + 1e-300, (beta, g, d[k], dref)


def pin_up_values_mpmath(o):
    """T_u and T_u' against 50-digit values, including the beta_L soft cap."""
    pts = [0.0, 1.0, -1.0, 25.0, -25.0, 60.0, -60.0, 1e-3, 200.0, -3.75]
    for lb in (25.0, 1.0, 1000.0):
        t, d = o.up(pts, lb)
        for k, u in enumerate(pts):
            ref = float(_mp_up(u, lb))
            assert _close(t[k], ref, 4e-15, 1e-300), (lb, u, t[k], ref)
            dref = _mp_diff(lambda x: _mp_up(x, lb), u)
            assert _close(d[k], dref, 1e-14, 1e-300), (lb, u, d[k], dref)


def pin_gate_parity_identities(o):
    """sigmoid(x) + sigmoid(-x) = 1 and sigmoid(x) - sigmoid(-x) = tanh(x/2)
    give the odd and even parts of T_g in closed form."""
    rng = np.random.default_rng(RNG_SEED)
    g = np.concatenate([rng.normal(0.0, 3.0, 400), rng.uniform(-70, 70, 100)])
    for beta in (0.5, 1.0, 4.0, 16.0):
        tp, _, _ = o.gate(g, beta)
        tn, _, _ = o.gate(-g, beta)
        scale = np.abs(tp) + np.abs(tn)
        odd = np.array([beta * math.tanh(x / beta) for x in g])
        even = np.array([beta * math.tanh(x / beta) * math.tanh(x / 2.0) for x in g])
        assert np.all(np.abs((tp - tn) - odd) <= 1e-14 * scale + 1e-300)
        assert np.all(np.abs((tp + tn) - even) <= 1e-14 * scale + 1e-300)


def pin_gate_special_points(o):
    """T_g(0) = 0 and T_g'(0) = 1/2 exactly; for beta = 4, T_g' vanishes at the
    single negative minimum G* (found by mpmath) and T_g is smallest there."""
    for beta in (1.0, 4.0, 16.0):
        t, d, _ = o.gate([0.0], beta)
        assert t[0] == 0.0 and d[0] == 0.5
    g_star = float(mpmath.findroot(lambda x: mpmath.diff(lambda y: _mp_gate(y, 4.0), x), -1.2))
    assert abs(g_star - (-1.2187557268720125)) < 1e-12
    t, d, m = o.gate([g_star, g_star - 1e-3, g_star + 1e-3], 4.0)
    assert abs(d[0]) <= 1e-15 * m[0]
    assert t[1] > t[0] and t[2] > t[0]


def pin_bounds_and_sign(o):
    """|T_g| <= beta with the sign of g; |T_u| <= min(|u|, beta_L) with the sign of u."""
    rng = np.random.default_rng(RNG_SEED + 1)
    x = np.concatenate([rng.normal(0, 4, 500), rng.uniform(-100, 100, 200)])
    for beta in (1.0, 4.0, 16.0):
        t, _, _ = o.gate(x, beta)
        assert np.all(np.abs(t) <= beta)
        assert np.all(np.sign(t) == np.sign(x))
    for lb in (1.0, 25.0):
        t, _ = o.up(x, lb)
        assert np.all(np.abs(t) <= np.minimum(np.abs(x), lb))
        assert np.all(np.sign(t) == np.sign(x))
    t, _ = o.up([60.0, -60.0], 25.0)
    assert t[0] < 25.0 and t[1] > -25.0


def pin_swiglu_limit(o):
    """As beta, beta_L -> infinity, T_g -> SiLU(g) = g sigmoid(g) and T_u -> u:
    compare with torch's SiLU and its autograd derivative in float64."""
    rng = np.random.default_rng(RNG_SEED + 2)
    g = rng.normal(0, 3, 300)
    gt = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    silu = torch.nn.functional.silu(gt)
    (dsilu,) = torch.autograd.grad(silu.sum(), gt)
    t, d, _ = o.gate(g, 1e12)
    np.testing.assert_allclose(t, silu.detach().numpy(), rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(d, dsilu.numpy(), rtol=1e-11, atol=1e-14)
    tu, du = o.up(g, 1e12)
    np.testing.assert_allclose(tu, g, rtol=1e-12)
    np.testing.assert_allclose(du, 1.0, rtol=1e-12)


def pin_linear_beta_none(o):
    """Without a linear beta the up branch is the identity, exactly."""
    rng = np.random.default_rng(RNG_SEED + 3)
    u = rng.normal(0, 10, 200)
    t, d = o.up(u, None)
    assert np.array_equal(t, u) and np.all(d == 1.0)


def pin_finite_differences(o):
    """Central differences of the oracle's forward against its analytic derivatives."""
    rng = np.random.default_rng(RNG_SEED + 4)
    x = np.concatenate([rng.normal(0, 3, 200), rng.uniform(-40, 40, 50)])
    h = 1e-5 * np.maximum(1.0, np.abs(x))
    for beta in (1.0, 4.0, 16.0):
        tp, _, _ = o.gate(x + h, beta)
        tm, _, _ = o.gate(x - h, beta)
        _, d, m = o.gate(x, beta)
        fd = (tp - tm) / (2 * h)
        assert np.all(np.abs(fd - d) <= 1e-7 * (m + np.abs(fd)) + 1e-12), beta
    for lb in (1.0, 25.0):
        tp, _ = o.up(x + h, lb)
        tm, _ = o.up(x - h, lb)
        _, d = o.up(x, lb)
        fd = (tp - tm) / (2 * h)
        assert np.all(np.abs(fd - d) <= 1e-7 * np.abs(fd) + 1e-12), lb


def _torch_rows(gu, rw, go, inter, beta, lb, scalar):
    """float64 torch statement of the chain, differentiated by autograd."""
    G = torch.tensor(gu[:, :inter], dtype=torch.float64, requires_grad=True)
    U = torch.tensor(gu[:, inter:2 * inter], dtype=torch.float64, requires_grad=True)
    W = torch.tensor(rw, dtype=torch.float64, requires_grad=True)
    GO = torch.tensor(go[:, :inter], dtype=torch.float64)
    tg = beta * torch.tanh(G / beta) * torch.sigmoid(G)
    tu = U if lb is None else lb * torch.tanh(U / lb)
    Y = tg * tu * (W if scalar else W[:, None])
    (Y * GO).sum().backward()
    return Y.detach().numpy(), G.grad.numpy(), U.grad.numpy(), W.grad.numpy()


def _as_f64(a):
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def pin_torch_autograd_rows(o):
    """Whole rows (padded row stride, bf16 and fp32 storage, row-aligned and
    scalar routing weights, with and without a linear beta) against float64
    autograd of the formula."""
    rng = np.random.default_rng(RNG_SEED + 5)
    T, I, pad = 5, 16, 3
    for dtype in ("bf16", "f32"):
        for lb in (25.0, 1.5, None):
            for scalar in (False, True):
                raw = rng.normal(0, 3, (T, 2 * I + pad)).astype(np.float32)
                raw[0, 2] = 45.0
                raw[1, I + 4] = -60.0
                raw_go = rng.normal(0, 1, (T, I + pad)).astype(np.float32)
                if dtype == "bf16":
                    gu, go = workloads.f32_to_bf16_bits(raw), workloads.f32_to_bf16_bits(raw_go)
                else:
                    gu, go = raw, raw_go
                rw = (rng.uniform(0.1, 1.0, 1 if scalar else T)).astype(np.float32)
                mode = oracle.RW_SCALAR if scalar else oracle.RW_ROW
                beta = 4.0
                Y, dG, dU, dW = _torch_rows(_as_f64(gu), rw.astype(np.float64), _as_f64(go),
                                             I, beta, lb, scalar)
                y = o.fwd(gu, rw, beta, lb, rw_mode=mode, inter=I)
                b = o.bwd(gu, rw, go, beta, lb, rw_mode=mode, inter=I)
                np.testing.assert_allclose(y, Y, rtol=1e-13, atol=1e-300)
                np.testing.assert_allclose(b.dg, dG, rtol=1e-12, atol=1e-13 * np.abs(dG).max())
                np.testing.assert_allclose(b.du, dU, rtol=1e-12, atol=1e-13 * np.abs(dU).max())
                if scalar:
                    total, _ = o.dw_scalar(gu, go, beta, lb, inter=I)
                    assert _close(total, dW[0], 1e-12, 1e-13 * b.sw.sum())
                else:
                    np.testing.assert_allclose(b.dw, dW, rtol=1e-12, atol=1e-13 * b.sw.max())


def pin_elementwise_weights(o):
    """Per-column [I] and per-element [T, I] routing weights against float64
    autograd of the formula: Y, dG, dU and the weight gradients (column sums
    over rows for [I]; the elementwise terms for [T, I])."""
    rng = np.random.default_rng(RNG_SEED + 8)
    T, I = 6, 24
    for dtype in ("bf16", "f32"):
        raw = rng.normal(0, 3, (T, 2 * I)).astype(np.float32)
        raw_go = rng.normal(0, 1, (T, I)).astype(np.float32)
        if dtype == "bf16":
            gu, go = workloads.f32_to_bf16_bits(raw), workloads.f32_to_bf16_bits(raw_go)
        else:
            gu, go = raw, raw_go
        for mode, shape in ((oracle.RW_COL, (I,)), (oracle.RW_FULL, (T, I))):
            w = rng.uniform(-1.0, 1.0, shape).astype(np.float32)
            G = torch.tensor(_as_f64(gu)[:, :I], requires_grad=True)
            U = torch.tensor(_as_f64(gu)[:, I:], requires_grad=True)
            W = torch.tensor(w.astype(np.float64), requires_grad=True)
            Y = 4.0 * torch.tanh(G / 4.0) * torch.sigmoid(G) * 25.0 * torch.tanh(U / 25.0) * W
            (Y * torch.tensor(_as_f64(go))).sum().backward()
            y = o.fwd(gu, w, 4.0, 25.0, rw_mode=mode)
            b = o.bwd(gu, w, go, 4.0, 25.0, rw_mode=mode)
            np.testing.assert_allclose(y, Y.detach().numpy(), rtol=1e-13, atol=1e-300)
            np.testing.assert_allclose(b.dg, G.grad.numpy(), rtol=1e-12, atol=1e-13 * np.abs(G.grad.numpy()).max())
            np.testing.assert_allclose(b.du, U.grad.numpy(), rtol=1e-12, atol=1e-13 * np.abs(U.grad.numpy()).max())
            if mode == oracle.RW_COL:
                cs, cm = o.dw_columns(gu, go, 4.0, 25.0)
                np.testing.assert_allclose(cs, W.grad.numpy(), rtol=1e-12, atol=1e-13 * cm.max())
            else:
                terms = o.dw_terms(gu, go, 4.0, 25.0)
                np.testing.assert_allclose(terms, W.grad.numpy(), rtol=1e-13, atol=1e-300)
                # the per-row sums of the full gradient are the row-aligned gradient
                np.testing.assert_allclose(terms.sum(axis=1), b.dw, rtol=1e-12, atol=1e-13 * b.sw.max())


def pin_special_rows(o):
    """A zero gate column gives Y = 0, dU = 0, dG = go w T_u / 2; a zero up
    column gives Y = 0, dG = 0, dU = go w T_g (sech^2(0) = 1)."""
    I = 8
    g_vals = np.array([1.5, -2.0, 3.0, -0.75, 5.0, -6.0, 0.0, 0.0], dtype=np.float32)
    u_vals = np.array([0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 2.5, -1.25], dtype=np.float32)
    gu = np.concatenate([g_vals, u_vals])[None, :]
    go = np.array([[0.5, -1.0, 2.0, 1.5, -0.25, 3.0, -2.0, 0.75]], dtype=np.float32)
    rw = np.array([0.625], dtype=np.float32)
    w = 0.625
    for lb in (25.0, None):
        y = o.fwd(gu, rw, 4.0, lb, inter=I)
        b = o.bwd(gu, rw, go, 4.0, lb, inter=I)
        tg, _, _ = o.gate(g_vals.astype(np.float64), 4.0)
        tu, _ = o.up(u_vals.astype(np.float64), lb)
        assert np.all(y == 0.0)
        # up column zero (first six): dG = 0, dU = go w T_g
        assert np.all(b.dg[0, :6] == 0.0)
        np.testing.assert_allclose(b.du[0, :6], go[0, :6] * w * tg[:6], rtol=1e-15)
        # gate column zero (last two): dU = 0, dG = go w T_u / 2
        assert np.all(b.du[0, 6:] == 0.0)
        np.testing.assert_allclose(b.dg[0, 6:], go[0, 6:] * w * tu[6:] / 2.0, rtol=1e-15)


def pin_dw_bruteforce(o):
    """The row-aligned routing-weight gradient is sum_i go * Y / w (Y is linear
    in w), summed here with math.fsum; the broadcast-scalar gradient is the
    sum of those over every row."""
    rng = np.random.default_rng(RNG_SEED + 6)
    T, I = 6, 40
    gu = workloads.f32_to_bf16_bits(rng.normal(0, 2, (T, 2 * I)).astype(np.float32))
    go = workloads.f32_to_bf16_bits(rng.normal(0, 1, (T, I)).astype(np.float32))
    rw = rng.uniform(0.2, 1.0, T).astype(np.float32)
    y = o.fwd(gu, rw, 4.0, 25.0)
    b = o.bwd(gu, rw, go, 4.0, 25.0)
    gof = _as_f64(go)
    for r in range(T):
        ref = math.fsum((gof[r] * y[r] / float(rw[r])).tolist())
        assert _close(b.dw[r], ref, 1e-13, 1e-15 * b.sw[r]), (r, b.dw[r], ref)
        assert _close(b.sw[r], math.fsum(np.abs(gof[r] * y[r] / float(rw[r])).tolist()), 1e-13)
    total, mag = o.dw_scalar(gu, go, 4.0, 25.0)
    assert _close(total, math.fsum(b.dw.tolist()), 1e-13, 1e-15 * mag)


def pin_bf16_loading(o):
    """bf16 bit patterns decode exactly: the same values given as float32
    produce identical results."""
    rng = np.random.default_rng(RNG_SEED + 7)
    f = rng.normal(0, 4, (3, 24)).astype(np.float32)
    bits = workloads.f32_to_bf16_bits(f)
    exact = workloads.bf16_bits_to_f32(bits)
    go_bits = workloads.f32_to_bf16_bits(rng.normal(0, 1, (3, 12)).astype(np.float32))
    rw = np.array([0.5, 1.0, 0.25], dtype=np.float32)
    assert np.array_equal(o.fwd(bits, rw, 4.0, 25.0), o.fwd(exact, rw, 4.0, 25.0))
    b1 = o.bwd(bits, rw, go_bits, 4.0, 25.0)
    b2 = o.bwd(exact, rw, workloads.bf16_bits_to_f32(go_bits), 4.0, 25.0)
    assert np.array_equal(b1.dg, b2.dg) and np.array_equal(b1.dw, b2.dw)
    one = np.array([[0x3F80, 0x3F80]], dtype=np.uint16)  # G = U = 1.0
    y = o.fwd(one, np.array([1.0], dtype=np.float32), 4.0, 25.0)
    assert _close(y[0, 0], float(_mp_gate(1.0, 4.0) * _mp_up(1.0, 25.0)), 4e-15)


# ---- MXFP8 block scaling (mx_oracle.c, OCP MX v1.0) -----------------------------

def pin_e4m3_decode_torch(o):
    """All 256 E4M3 codes decode to the values torch's float8_e4m3fn gives them."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = o.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def pin_e4m3_encode_torch(o):
    """Nearest-even encoding against torch's float32 -> float8_e4m3fn conversion:
    every finite bf16 value with |x| <= 464 (above that torch overflows to NaN
    where the MX conversion clamps) and random fp32 values from the subnormals
    (below 2^-6) to the top binade."""
    x = workloads.bf16_bits_to_f32(np.arange(1 << 16, dtype=np.uint32).astype(np.uint16))
    x = x[np.isfinite(x) & (np.abs(x) <= 464.0)]
    rng = np.random.default_rng(RNG_SEED)
    y = (rng.standard_normal(20000) * np.exp2(rng.integers(-14, 9, 20000))).astype(np.float32)
    v = np.concatenate([x, y[np.abs(y) <= 464.0]])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = o.e4m3_encode(v.astype(np.float64))
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, (v[bad[:5]], got[bad[:5]], ref[bad[:5]])


def pin_e4m3_saturation(o):
    """E4M3 has no infinities: the MX conversion clamps magnitudes at or above
    its largest normal 448 (code 0x7E) to +-448; NaN stays NaN."""
    got = o.e4m3_encode([448.0, 449.0, 470.0, 1e9, float("inf"), -500.0, -float("inf")])
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE], list(got)
    assert (int(o.e4m3_encode([float("nan")])[0]) & 0x7F) == 0x7F


def pin_mx_scale_rules(o):
    """Shared exponents.  The spec's rule makes the block maximum land in
    [2^8, 2^9) after scaling (floor(log2 amax) - 8); the no-clamp rule takes
    the smallest power of two with amax / X <= 448, so amax / X > 224.  Closed
    forms at the boundaries; zero, tiny, NaN and infinite blocks."""
    OCP, CEIL = oracle.MX_RULE_OCP, oracle.MX_RULE_CEIL
    cases = {1.0: (-8, -8), 448.0: (0, 0), 500.0: (0, 1), 511.0: (0, 1), 512.0: (1, 1), 224.0: (-1, -1),
             224.5: (-1, 0), 0.0: (-127, -127), 2.0 ** -140: (-127, -127), 1.99 * 2.0 ** 127: (119, 120)}
    for amax, (e_ocp, e_ceil) in cases.items():
        assert o.mx_scale_exp(amax, OCP) == e_ocp, (amax, o.mx_scale_exp(amax, OCP))
        assert o.mx_scale_exp(amax, CEIL) == e_ceil, (amax, o.mx_scale_exp(amax, CEIL))
    for bad in (float("nan"), float("inf")):
        assert o.mx_scale_exp(bad, OCP) == oracle.MX_SCALE_NAN
    rng = np.random.default_rng(RNG_SEED + 1)
    for amax in np.exp2(rng.uniform(-118.0, 120.0, 4000)):
        r = amax / 2.0 ** o.mx_scale_exp(amax, OCP)
        assert 256.0 <= r < 512.0, (amax, r)
        r = amax / 2.0 ** o.mx_scale_exp(amax, CEIL)
        assert 224.0 < r <= 448.0, (amax, r)


def pin_mxfp8_blocks(o):
    """Blocks of 32 along each row: scale byte = e + 127 from the block's own
    largest magnitude (checked by the rules' inequalities), codes = torch's E4M3
    conversion of v / 2^e, clamped to 448 under the spec's rule.  Rows hold an
    all-zero block, a NaN, tiny values and an outlier."""
    rng = np.random.default_rng(RNG_SEED + 2)
    v = (rng.standard_normal((7, 96)) * np.exp2(rng.integers(-20, 20, (7, 1)))).astype(np.float32)
    v[1, 32:64] = 0.0
    v[2, 5] = np.nan
    v[3, 64:96] *= np.float32(2.0 ** -100)
    v[4, 7] = 1e4
    v = v.astype(np.float64)
    for rule in (oracle.MX_RULE_OCP, oracle.MX_RULE_CEIL):
        codes, scales = o.mxfp8_quantize(v, rule)
        assert codes.shape == v.shape and scales.shape == (7, 3)
        for r in range(7):
            for b in range(3):
                blk = v[r, 32 * b:32 * b + 32]
                s = int(scales[r, b])
                if np.isnan(blk).any():
                    assert s == 255
                    continue
                amax = np.abs(blk).max()
                if amax == 0.0:
                    assert s == 0 and not np.any(codes[r, 32 * b:32 * b + 32] & 0x7F)
                    continue
                ratio = amax / 2.0 ** (s - 127)
                if rule == oracle.MX_RULE_OCP:
                    assert 256.0 <= ratio < 512.0, (r, b, ratio)
                else:
                    assert 224.0 < ratio <= 448.0, (r, b, ratio)
                scaled = (blk / 2.0 ** (s - 127)).astype(np.float32)
                ref = torch.from_numpy(np.clip(scaled, -448.0, 448.0)).to(torch.float8_e4m3fn)
                assert np.array_equal(codes[r, 32 * b:32 * b + 32], ref.view(torch.uint8).numpy()), (r, b)


# ---- NVFP4 (mx_oracle.c) ----------------------------------------------------------------

_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def pin_e2m1_nearest_even(o):
    """Every E2M1 code decodes to the format's 8 magnitudes with its sign; the
    encoding of random values is the nearest of them by brute-force search,
    ties to the even code (the midpoints 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5),
    and magnitudes from 6 up clamp to 6."""
    codes = np.arange(16, dtype=np.uint8)
    dec = o.e2m1_decode(codes)
    assert list(np.abs(dec[:8])) == _E2M1 and list(-dec[8:]) == _E2M1 and np.all(np.signbit(dec[8:]))
    mids = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 6.0: 6.0, 7.0: 6.0, 1e9: 6.0}
    for x, want in mids.items():
        assert o.e2m1_decode(o.e2m1_encode([x]))[0] == want, x
        assert o.e2m1_decode(o.e2m1_encode([-x]))[0] == -want, -x
    rng = np.random.default_rng(RNG_SEED + 13)
    x = rng.uniform(-7.0, 7.0, 4000)
    got = o.e2m1_decode(o.e2m1_encode(x))
    grid = np.array(_E2M1)
    for xv, g in zip(x, got):
        d = np.abs(np.abs(xv) - grid)
        assert abs(abs(g) - grid[np.argmin(d)]) == 0.0 or abs(xv) >= 6.0, (xv, g)
        assert np.sign(g) in (0.0, np.sign(xv))


def pin_nvfp4_blocks(o):
    """The two scaling levels of NVFP4 as consequences of their definition:
    the tensor scale maps the tensor's largest magnitude onto the top of both
    formats at once, so the block holding it gets the largest E4M3 scale (448)
    and that element the largest E2M1 code (6), and no block scale saturates;
    each 16-element block's scale is torch's E4M3 conversion of
    amax_b * S_enc / 6; decoded codes times s_b / S_enc lie within half an
    E2M1 step (scaled) of v."""
    rng = np.random.default_rng(RNG_SEED + 14)
    v = rng.standard_normal((5, 64)) * np.exp2(rng.integers(-6, 6, (5, 1)))
    v[2, 16:32] = 0.0
    codes, scales, s_enc = o.nvfp4_quantize(v)
    top = np.unravel_index(np.argmax(np.abs(v)), v.shape)
    assert o.e4m3_decode(scales[top[0], top[1] // 16:top[1] // 16 + 1])[0] == 448.0
    assert o.e2m1_decode(codes[top[0], top[1]:top[1] + 1])[0] == np.sign(v[top]) * 6.0
    assert o.e4m3_decode(scales).max() == 448.0
    # so the largest element decodes back to itself: code x block scale / S_enc
    top_dec = (o.e2m1_decode(codes[top[0], top[1]:top[1] + 1])[0]
               * o.e4m3_decode(scales[top[0], top[1] // 16:top[1] // 16 + 1])[0] / s_enc)
    assert abs(top_dec - v[top]) <= 1e-15 * abs(v[top])
    for r in range(5):
        for b in range(4):
            blk = v[r, 16 * b:16 * b + 16]
            want = torch.tensor([np.abs(blk).max() * s_enc / 6.0], dtype=torch.float32).to(torch.float8_e4m3fn)
            assert scales[r, b] == want.view(torch.uint8).item(), (r, b)
            sb = o.e4m3_decode(scales[r, b:b + 1])[0]
            dec = o.e2m1_decode(codes[r, 16 * b:16 * b + 16]) * sb / s_enc
            if sb == 0:
                assert not np.any(codes[r, 16 * b:16 * b + 16] & 7)
                continue
            y = blk * s_enc / sb
            step = np.where(np.abs(y) < 2, 0.5, np.where(np.abs(y) < 4, 1.0, 2.0))
            assert np.all(np.abs(dec - blk) <= 0.5 * step * sb / s_enc * (1 + 1e-12) + (np.abs(y) > 6) * np.abs(blk)), (r, b)


# ---- FC1 followed by SiTU-GLU (fc1_oracle.c) ---------------------------------------

def _bf16(a):
    return workloads.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _widen(bits):
    return workloads.bf16_bits_to_f32(bits).astype(np.float64)


def pin_fc1_bruteforce(o):
    """A tiny grouped case (3 experts, one of them empty): every FC1 output is a
    math.fsum dot product over the hidden axis with the owning expert's gate or
    up row, and Y is the 50-digit value of T_g(G) T_u(U) w."""
    rng = np.random.default_rng(RNG_SEED + 3)
    E, I, H, T = 3, 8, 24, 11
    x = _bf16(rng.standard_normal((T, H)))
    w1 = _bf16(0.3 * rng.standard_normal((E * 2 * I, H)))
    offsets = [0, 4, 4, 11]
    rw = rng.random(T).astype(np.float32)
    y, err, gu = o.fc1_fwd(x, w1, offsets, I, rw, 4.0, 25.0)
    xf, wf = _widen(x), _widen(w1)
    for r in range(T):
        e = 0 if r < 4 else 2
        for i in range(I):
            g = math.fsum(xf[r] * wf[e * 2 * I + i])
            u = math.fsum(xf[r] * wf[e * 2 * I + I + i])
            assert _close(gu[r, i], g, 1e-14, 1e-14) and _close(gu[r, I + i], u, 1e-14, 1e-14), (r, i)
            ref = float(_mp_gate(g, 4.0) * _mp_up(u, 25.0)) * float(rw[r])
            assert _close(y[r, i], ref, 1e-12, 1e-15), (r, i, y[r, i], ref)
            assert err[r, i] >= 0.0


def pin_fc1_matches_activation_oracle(o):
    """With inputs in {-1/4, 0, 1/4} every FC1 output is k/16, |k| <= 16, a bf16
    number: the fused oracle then equals the pinned activation oracle applied
    to that gate_up, exactly, for every beta form."""
    rng = np.random.default_rng(RNG_SEED + 4)
    T, H, I = 6, 16, 8
    x = _bf16(rng.integers(-1, 2, (T, H)) / 4.0)
    w1 = _bf16(rng.integers(-1, 2, (2 * I, H)) / 4.0)
    rw = rng.random(T).astype(np.float32)
    for beta, lb in ((4.0, 25.0), (1.0, None), (16.0, 2.0)):
        y, _, gu = o.fc1_fwd(x, w1, [0, T], I, rw, beta, lb)
        gu_bits = _bf16(gu)
        assert np.array_equal(_widen(gu_bits), gu)
        assert np.array_equal(y, o.fwd(gu_bits, rw, beta, lb))


def pin_fc1_grouped_equals_per_expert(o):
    """The grouped call equals one call per expert on that expert's rows and weights."""
    rng = np.random.default_rng(RNG_SEED + 5)
    E, I, H = 4, 8, 32
    sizes = [5, 0, 9, 3]
    offsets = np.concatenate([[0], np.cumsum(sizes)])
    T = int(offsets[-1])
    x = _bf16(rng.standard_normal((T, H)))
    w1 = _bf16(0.2 * rng.standard_normal((E * 2 * I, H)))
    rw = rng.random(T).astype(np.float32)
    y, _, _ = o.fc1_fwd(x, w1, offsets, I, rw, 4.0, 25.0)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        ye, _, _ = o.fc1_fwd(x[a:b], w1[e * 2 * I:(e + 1) * 2 * I], [0, b - a], I, rw[a:b], 4.0, 25.0)
        assert np.array_equal(y[a:b], ye), e


# ---- attention-residual mixing core (attn_res_oracle.c) -----------------------------

def _torch_attn_res(x, nw, pw, eps):
    """float64 torch library routines: rms_norm, a matmul projection, softmax,
    and the weighted sum of the raw values."""
    xt = torch.from_numpy(x)
    k = torch.nn.functional.rms_norm(xt, (x.shape[-1],), weight=torch.from_numpy(nw), eps=eps)
    logits = k @ torch.from_numpy(pw)
    prob = torch.softmax(logits, dim=-1)
    return torch.einsum("tb,tbh->th", prob, xt).numpy(), prob.numpy()


def pin_attn_res_torch(o):
    """Against torch's float64 rms_norm / softmax: stored sums and a current sum
    (appended last), bf16 values, one source of tiny values (where epsilon
    matters), fp32 weights."""
    rng = np.random.default_rng(RNG_SEED + 6)
    T, B, H = 5, 3, 64
    blocks = _bf16(rng.standard_normal((T, B, H)) * 2.0)
    blocks[:, 1] = _bf16(_widen(blocks[:, 1]) * 1e-3)
    prefix = _bf16(rng.standard_normal((T, H)))
    nw = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    pw = (0.2 * rng.standard_normal(H)).astype(np.float32)
    eps = 1e-6
    out, mag, prob = o.attn_res(blocks, prefix, nw, pw, eps)
    x = np.concatenate([_widen(blocks), _widen(prefix)[:, None, :]], axis=1)
    ref, pref = _torch_attn_res(x, nw.astype(np.float64), pw.astype(np.float64), eps)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14), np.abs(out - ref).max()
    assert np.allclose(prob, pref, rtol=1e-12, atol=1e-15)
    assert np.all(mag >= np.abs(out) * (1 - 1e-12))


def pin_attn_res_invariants(o):
    """Identical sources give that source back; a zero projection gives the plain
    average; a single source is returned as is; doubling every value (exact in
    bf16) with epsilon 0 doubles the output and leaves the weights."""
    rng = np.random.default_rng(RNG_SEED + 7)
    T, H = 4, 48
    v = _bf16(rng.standard_normal((T, H)))
    nw = rng.random(H).astype(np.float32) + 0.5
    pw = rng.standard_normal(H).astype(np.float32)
    same = np.repeat(v[:, None, :], 4, axis=1)
    out, _, _ = o.attn_res(same, None, nw, pw, 1e-6)
    assert np.allclose(out, _widen(v), rtol=1e-15, atol=0)
    blocks = _bf16(rng.standard_normal((T, 3, H)))
    out, _, prob = o.attn_res(blocks, None, nw, np.zeros(H, np.float32), 1e-6)
    assert np.allclose(prob, 1.0 / 3.0, rtol=1e-15) and np.allclose(out, _widen(blocks).mean(axis=1), rtol=1e-14)
    out, _, _ = o.attn_res(None, v, nw, pw, 1e-6)
    assert np.array_equal(out, _widen(v))
    o1, _, p1 = o.attn_res(blocks, v, nw, pw, 0.0)
    o2, _, p2 = o.attn_res(_bf16(_widen(blocks) * 2), _bf16(_widen(v) * 2), nw, pw, 0.0)
    assert np.allclose(p1, p2, rtol=1e-13) and np.allclose(o2, 2 * o1, rtol=1e-13, atol=1e-300)


def pin_attn_res_large_logits(o):
    """Logits of thousands: the softmax must stay finite and match torch's."""
    rng = np.random.default_rng(RNG_SEED + 8)
    T, B, H = 3, 5, 32
    blocks = _bf16(rng.standard_normal((T, B, H)))
    nw = np.ones(H, np.float32)
    pw = (1e3 * rng.standard_normal(H)).astype(np.float32)
    out, _, prob = o.attn_res(blocks, None, nw, pw, 1e-6)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(prob))
    ref, pref = _torch_attn_res(_widen(blocks), nw.astype(np.float64), pw.astype(np.float64), 1e-6)
    assert np.allclose(prob, pref, rtol=1e-9, atol=1e-300) and np.allclose(out, ref, rtol=1e-9, atol=1e-12)


def pin_attn_res_two_arrays(o):
    """Stored sums plus the current sum equal the same sources stacked in one array."""
    rng = np.random.default_rng(RNG_SEED + 9)
    T, B, H = 4, 2, 40
    blocks = _bf16(rng.standard_normal((T, B, H)))
    prefix = _bf16(rng.standard_normal((T, H)))
    nw = rng.random(H).astype(np.float32) + 0.5
    pw = rng.standard_normal(H).astype(np.float32)
    a, _, _ = o.attn_res(blocks, prefix, nw, pw, 1e-6)
    b, _, _ = o.attn_res(np.concatenate([blocks, prefix[:, None, :]], axis=1), None, nw, pw, 1e-6)
    assert np.array_equal(a, b)


# ---- FC2 data gradient + SiTU-GLU backward (fc2_oracle.c) ---------------------------

def pin_fc2_dgrad_bruteforce(o):
    """A tiny grouped case: dY as fsum dot products with the owning expert's
    transposed FC2 rows, dG, dU from 50-digit derivatives of the branch
    functions, d_w an fsum over the row."""
    rng = np.random.default_rng(RNG_SEED + 10)
    E, I, H, T = 2, 8, 24, 9
    dout = _bf16(rng.standard_normal((T, H)))
    w2t = _bf16(0.3 * rng.standard_normal((E * I, H)))
    gu = _bf16(2.0 * rng.standard_normal((T, 2 * I)))
    offsets = [0, 5, 9]
    rw = rng.random(T).astype(np.float32)
    dgu, dw, dy, err, dw_err = o.fc2_dgrad(dout, w2t, offsets, gu, rw, 4.0, 25.0)
    df, wf, gf = _widen(dout), _widen(w2t), _widen(gu)
    for r in range(T):
        e = 0 if r < 5 else 1
        terms = []
        for i in range(I):
            d = math.fsum(df[r] * wf[e * I + i])
            assert _close(dy[r, i], d, 1e-14, 1e-14), (r, i)
            g, u = gf[r, i], gf[r, I + i]
            tg, tu = float(_mp_gate(g, 4.0)), float(_mp_up(u, 25.0))
            dtg = _mp_diff(lambda v: _mp_gate(v, 4.0), g)
            dtu = _mp_diff(lambda v: _mp_up(v, 25.0), u)
            assert _close(dgu[r, i], d * float(rw[r]) * tu * dtg, 1e-12, 1e-14), (r, i)
            assert _close(dgu[r, I + i], d * float(rw[r]) * tg * dtu, 1e-12, 1e-14), (r, i)
            terms.append(d * tg * tu)
        assert _close(dw[r], math.fsum(terms), 1e-12, 1e-14), r
    assert np.all(err >= 0) and np.all(dw_err >= 0)


def pin_fc2_dgrad_matches_activation_backward(o):
    """With inputs in {-1/4, 0, 1/4} every dY is k/16, a bf16 number: the fused
    oracle then equals the pinned activation backward with grad_out = dY."""
    rng = np.random.default_rng(RNG_SEED + 11)
    T, H, I = 5, 16, 8
    dout = _bf16(rng.integers(-1, 2, (T, H)) / 4.0)
    w2t = _bf16(rng.integers(-1, 2, (I, H)) / 4.0)
    gu = _bf16(rng.standard_normal((T, 2 * I)) * 3.0)
    rw = rng.random(T).astype(np.float32)
    for beta, lb in ((4.0, 25.0), (1.0, None)):
        dgu, dw, dy, _, _ = o.fc2_dgrad(dout, w2t, [0, T], gu, rw, beta, lb)
        dy_bits = _bf16(dy)
        assert np.array_equal(_widen(dy_bits), dy)
        ref = o.bwd(gu, rw, dy_bits, beta, lb)
        assert np.array_equal(dgu[:, :I], ref.dg) and np.array_equal(dgu[:, I:], ref.du)
        assert np.allclose(dw, ref.dw, rtol=1e-14, atol=1e-15)


def pin_fc2_dgrad_grouped_equals_per_expert(o):
    rng = np.random.default_rng(RNG_SEED + 12)
    E, I, H = 3, 8, 32
    offsets = np.array([0, 4, 4, 11], dtype=np.int64)
    T = 11
    dout = _bf16(rng.standard_normal((T, H)))
    w2t = _bf16(0.2 * rng.standard_normal((E * I, H)))
    gu = _bf16(rng.standard_normal((T, 2 * I)))
    rw = rng.random(T).astype(np.float32)
    dgu, dw, _, _, _ = o.fc2_dgrad(dout, w2t, offsets, gu, rw, 4.0, 25.0)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if a == b:
            continue
        de, we, _, _, _ = o.fc2_dgrad(dout[a:b], w2t[e * I:(e + 1) * I], [0, b - a], gu[a:b], rw[a:b], 4.0, 25.0)
        assert np.array_equal(dgu[a:b], de) and np.array_equal(dw[a:b], we)


PINS = [
    pin_gate_values_mpmath,
    pin_up_values_mpmath,
    pin_gate_parity_identities,
    pin_gate_special_points,
    pin_bounds_and_sign,
    pin_swiglu_limit,
    pin_linear_beta_none,
    pin_finite_differences,
    pin_torch_autograd_rows,
    pin_elementwise_weights,
    pin_special_rows,
    pin_dw_bruteforce,
    pin_bf16_loading,
    pin_e4m3_decode_torch,
    pin_e4m3_encode_torch,
    pin_e4m3_saturation,
    pin_mx_scale_rules,
    pin_mxfp8_blocks,
    pin_e2m1_nearest_even,
    pin_nvfp4_blocks,
    pin_fc1_bruteforce,
    pin_fc1_matches_activation_oracle,
    pin_fc1_grouped_equals_per_expert,
    pin_attn_res_torch,
    pin_attn_res_invariants,
    pin_attn_res_large_logits,
    pin_attn_res_two_arrays,
    pin_fc2_dgrad_bruteforce,
    pin_fc2_dgrad_matches_activation_backward,
    pin_fc2_dgrad_grouped_equals_per_expert,
]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin, oracle_lib):
    assert oracle_lib.mutant_id == 0
    pin(oracle_lib)


# Planted mistakes compiled into situ_oracle.c under -DSITU_ORACLE_MUTANT=n.
MUTANTS = {
    1: "dropped product-rule term in T_g'",
    2: "wrong sign of the second T_g' term",
    3: "u * beta_L instead of u / beta_L",
    4: "sigmoid(-g) instead of sigmoid(g)",
    5: "routing weight dropped from Y",
    6: "dG uses T_g where T_u belongs",
    7: "dU uses T_u where T_g belongs",
    8: "gate and up halves swapped",
    9: "upstream gradient dropped from d_w",
    10: "linear beta ignored",
    11: "sech^2 with exp(-|a|) instead of exp(-2|a|)",
    12: "row stride ignored",
    13: "per-column weight indexed by the row",
    14: "MX shared exponent from ceil(log2 amax)",
    15: "MX shared exponent with E4M3 emax 7",
    16: "E4M3 overflow to NaN instead of clamping",
    17: "E4M3 ties rounded away from zero",
    18: "E4M3 subnormal spacing 2^-10",
    19: "no-clamp scale rule bumps the exponent at equality",
    20: "FC1 uses the next expert's weights",
    21: "FC1 up rows taken from the gate rows",
    22: "FC1 dot product drops the last product",
    23: "FC1 boundary row assigned to the earlier expert",
    24: "RMSNorm with the sum instead of the mean of squares",
    25: "RMSNorm epsilon dropped",
    26: "RMSNorm weight not applied",
    27: "softmax without the max shift",
    28: "a transformed value combined instead of the raw one",
    29: "FC2 weight read untransposed in the data gradient",
    30: "routing weight dropped from the fused dG",
    31: "upstream gradient dropped from the fused d_w",
    32: "E2M1 ties to the larger magnitude",
    33: "NVFP4 block scale from amax / 4",
    34: "NVFP4 tensor scale not applied",
    35: "NVFP4 tensor scale 448 / amax (the E2M1 range left out)",
    36: "NVFP4 tensor scale inverted (amax / 2688)",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=[f"m{k}" for k in sorted(MUTANTS)])
def test_mutant_rejected(mutant, tmp_path):
    path = oracle.build(output=os.path.join(tmp_path, f"libsitu_oracle_m{mutant}.so"),
                        mutant=mutant, force=True)
    o = oracle.Oracle(path)
    assert o.mutant_id == mutant
    caught = []
    for pin in PINS:
        try:
            pin(o)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin rejects mutant {mutant} ({MUTANTS[mutant]})"
