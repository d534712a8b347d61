"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs, element by element (tolerance rule in parity.py).

Small cases cover every element; they span several CTAs and ragged tails
(T in {1, 3, 257, ...}, I in {8, 24, 520, ...}), both storage dtypes, every
gate-exponent specialisation (beta = 4, 2, 1 and generic), with and without a
linear beta, every routing-weight mode, strided rows, special values, and
guard bytes around every output.  Full-size workloads are in
test_gpu_fullsize.py.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

import parity
from parity import Guarded, as_f64, call_bwd, call_fwd, check_dw, check_output, to_device, to_host

pytestmark = pytest.mark.gpu


def case_inputs(dtype: str, T: int, I: int, seed: int):
    """gate_up [T, 2I], rw [T] (fp32), grad_out [T, I]: G, U ~ N(0, 3) with 1 %
    outliers +-U(20, 60) (tanh saturation), w ~ U(0, 1), go ~ N(0, 1)."""
    wl = dataclasses.replace(workloads.workload(2), dtype=dtype, tokens=T, inter=I, seed=1000 + seed,
                             rw_kind="uniform")
    x = workloads.inputs(wl)
    return x["gate_up"], x["routing_weights"], x["grad_out"]


def rw_for(kind: str, rw32: np.ndarray):
    """Host routing weights and the mode for a case kind."""
    if kind == "row_f32":
        return rw32, abi.SITU_RW_ROW
    if kind == "row_bf16":
        return workloads.f32_to_bf16_bits(rw32), abi.SITU_RW_ROW
    if kind == "scalar":
        return rw32[:1].copy(), abi.SITU_RW_SCALAR
    if kind == "none":
        return None, abi.SITU_RW_NONE
    raise ValueError(kind)


def oracle_rw(rw_host, T):
    """The oracle's view of the weights (it has no 'none' mode: w = 1)."""
    if rw_host is None:
        return np.ones(T, dtype=np.float32), oracle.RW_ROW
    return rw_host, (oracle.RW_SCALAR if rw_host.size == 1 and T != 1 else oracle.RW_ROW)


def run_case(dev, dtype, T, I, beta, lb, kind, seed, want_drw=True):
    gu_h, rw32, go_h = case_inputs(dtype, T, I, seed)
    rw_h, mode = rw_for(kind, rw32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gu, go = to_device(gu_h, dev), to_device(go_h, dev)
    rw = to_device(rw_h, dev) if rw_h is not None else None
    out = Guarded(T, I, I, tdt, dev)
    dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
    want = want_drw and rw is not None
    d_rw = None
    if want:
        d_rw = torch.full((rw.numel(),), float("nan"), dtype=rw.dtype, device=dev)
    abi.check(call_fwd(gu, I, rw, mode, beta, lb, out), "fwd")
    abi.check(call_bwd(gu, I, rw, mode, beta, lb, go, dgu, d_rw=d_rw), "bwd")
    torch.cuda.synchronize()
    out.check()
    dgu.check()

    o = oracle.load()
    orw, omode = oracle_rw(rw_h, T)
    ref_y = o.fwd(gu_h, orw, beta, lb, rw_mode=omode)
    ref = o.bwd(gu_h, orw, go_h, beta, lb, rw_mode=omode)
    rep = {"y": check_output("Y", to_host(out.view), ref_y)}
    d = to_host(dgu.view)
    rep["dg"] = check_output("dG", d[:, :I], ref.dg, cancel_scale=ref.cg)
    rep["du"] = check_output("dU", d[:, I:], ref.du)
    if want:
        got = to_host(d_rw)
        if mode == abi.SITU_RW_SCALAR:
            total, mag = o.dw_scalar(gu_h, go_h, beta, lb)
            rep["dw"] = check_dw("d_w (scalar)", got, np.array([total]), np.array([mag]))
        else:
            rep["dw"] = check_dw("d_w", got, ref.dw, ref.sw)
    return rep


SHAPES = [("bf16", 1, 8), ("bf16", 3, 24), ("bf16", 257, 520), ("bf16", 64, 2048), ("bf16", 40, 3072),
          ("f32", 1, 4), ("f32", 3, 12), ("f32", 257, 260), ("f32", 33, 4096)]
COMBOS = [
    (4.0, 25.0, "row_f32"),   # Kimi-K3 defaults, exponent squared
    (4.0, None, "row_bf16"),  # no linear clamp, bf16 weights
    (1.0, 25.0, "scalar"),    # beta = 1: E_t = E_s^2; broadcast weight
    (2.0, 1.5, "row_f32"),    # beta = 2: one shared exponential; tight linear clamp
    (16.0, None, "none"),     # generic exponentials; unweighted
    (0.5, 25.0, "row_f32"),   # generic, beta below 1
    (1e6, 1e6, "row_f32"),    # close to the SwiGLU limit (series branch everywhere)
]


@pytest.mark.parametrize("dtype,T,I", SHAPES, ids=[f"{d}-{t}x{i}" for d, t, i in SHAPES])
@pytest.mark.parametrize("beta,lb,kind", COMBOS, ids=[f"b{b}-lb{l}-{k}" for b, l, k in COMBOS])
def test_parity_small(dtype, T, I, beta, lb, kind, cuda_device):
    run_case(cuda_device, dtype, T, I, beta, lb, kind, seed=T * 7 + I)


def test_strided_rows_and_weights(cuda_device):
    """Row pitches wider than the data, a strided routing-weight column and a
    strided weight-gradient column; the padding must stay untouched."""
    dev = cuda_device
    T, I = 131, 264
    gu_h, rw32, go_h = case_inputs("bf16", T, I, seed=5)
    gpitch, opitch, gopitch, dpitch, rws, drws = 2 * I + 24, I + 8, I + 16, 2 * I + 40, 3, 2
    gu_pad = np.zeros((T, gpitch), dtype=np.uint16); gu_pad[:, :2 * I] = gu_h
    go_pad = np.zeros((T, gopitch), dtype=np.uint16); go_pad[:, :I] = go_h
    rw_pad = np.zeros((T, rws), dtype=np.float32); rw_pad[:, 0] = rw32
    gu, go, rw = to_device(gu_pad, dev), to_device(go_pad, dev), to_device(rw_pad, dev)
    out = Guarded(T, I, opitch, torch.bfloat16, dev)
    dgu = Guarded(T, 2 * I, dpitch, torch.bfloat16, dev)
    d_rw_buf = torch.full((T, drws), float("nan"), dtype=torch.float32, device=dev)
    abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, out, rw_stride=rws), "fwd")
    abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, dgu, d_rw=d_rw_buf, rw_stride=rws,
                       d_rw_stride=drws), "bwd")
    torch.cuda.synchronize()
    out.check(); dgu.check()
    assert torch.all(torch.isnan(d_rw_buf[:, 1])), "weight-gradient stride not respected"
    o = oracle.load()
    ref_y = o.fwd(gu_h, rw32, 4.0, 25.0)
    ref = o.bwd(gu_h, rw32, go_h, 4.0, 25.0)
    check_output("Y", to_host(out.view), ref_y)
    d = to_host(dgu.view)
    check_output("dG", d[:, :I], ref.dg, ref.cg)
    check_output("dU", d[:, I:], ref.du)
    check_dw("d_w", to_host(d_rw_buf[:, 0]), ref.dw, ref.sw)


def test_special_values(cuda_device):
    """Zeros of both signs, +-inf, huge, tiny and subnormal inputs, and the
    gate-derivative zero G* = -1.21875 (the bf16 value nearest -1.2187557)."""
    dev = cuda_device
    specials = [0.0, -0.0, np.inf, -np.inf, 3e38, -3e38, 1e-30, -1e-30, 1e-39, -1e-39,
                -1.21875, 1.21875, 60.0, -60.0, 88.0, -88.0, 100.0, -100.0, 1e-3, -1e-3]
    for dtype in ("bf16", "f32"):
        T, I = 24, 40 if dtype == "bf16" else 44
        gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=77)
        vals = np.array(specials, dtype=np.float32)
        vals_st = workloads.f32_to_bf16_bits(vals) if dtype == "bf16" else vals
        base = gu_h
        for beta, lb in ((4.0, 25.0), (16.0, None), (1.0, 2.0)):
            gu_h = base.copy()
            for r in range(T):
                gu_h[r, :len(specials)] = np.roll(vals_st, r)           # gate column specials
                if lb is not None:  # without a clamp, U = 3e38 overflows fp32 but not the oracle
                    gu_h[r, I:I + len(specials)] = np.roll(vals_st, 3 * r)
            tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
            gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
            out = Guarded(T, I, I, tdt, dev)
            dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
            d_rw = torch.empty(T, dtype=torch.float32, device=dev)
            abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, beta, lb, out), "fwd")
            abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, beta, lb, go, dgu, d_rw=d_rw), "bwd")
            torch.cuda.synchronize()
            o = oracle.load()
            ref_y = o.fwd(gu_h, rw32, beta, lb)
            ref = o.bwd(gu_h, rw32, go_h, beta, lb)
            check_output(f"Y {dtype} beta={beta}", to_host(out.view), ref_y)
            d = to_host(dgu.view)
            check_output(f"dG {dtype} beta={beta}", d[:, :I], ref.dg, ref.cg)
            check_output(f"dU {dtype} beta={beta}", d[:, I:], ref.du)
            check_dw(f"d_w {dtype} beta={beta}", to_host(d_rw), ref.dw, ref.sw)


@pytest.mark.parametrize("lb", [25.0, None])
def test_small_gate_values_around_the_series_threshold(lb, cuda_device):
    """Gate values of magnitude 2^-13 to 2^-4, log-uniform with random signs,
    where 1 - exp(-2g/beta) is small and its relative accuracy decides the
    outputs' relative accuracy.  Even rows hold only |g| >= 2^-9 (whole
    vectors that need no series); odd rows span the full range, with
    2^-9 and the bf16 value just below it planted at vector boundaries.
    Every element of Y, dG, dU and d_w against the oracle (bf16, beta = 4)."""
    dev = cuda_device
    T, I = 96, 2048
    gu_h, rw32, go_h = case_inputs("bf16", T, I, seed=91)
    rng = np.random.default_rng(91)
    mag = np.where((np.arange(T) % 2 == 0)[:, None], rng.uniform(-9.0, -4.0, (T, I)), rng.uniform(-13.0, -4.0, (T, I)))
    g = (np.exp2(mag) * rng.choice([-1.0, 1.0], (T, I))).astype(np.float32)
    g[1::2, 0::8] = np.float32(2.0 ** -9)
    g[1::2, 7::16] = -np.float32(2.0 ** -9)
    below = workloads.f32_to_bf16_bits(np.array([2.0 ** -9], dtype=np.float32)) - 1  # 0x3AFF
    gu_h = gu_h.copy()
    gu_h[:, :I] = workloads.f32_to_bf16_bits(g)
    gu_h[1::4, 8::32] = below
    gu_h[3::4, 15::32] = below | 0x8000
    gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
    out = Guarded(T, I, I, torch.bfloat16, dev)
    dgu = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    d_rw = torch.empty(T, dtype=torch.float32, device=dev)
    abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, lb, out), "fwd")
    abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, lb, go, dgu, d_rw=d_rw), "bwd")
    torch.cuda.synchronize()
    out.check()
    dgu.check()
    o = oracle.load()
    check_output("Y", to_host(out.view), o.fwd(gu_h, rw32, 4.0, lb))
    ref = o.bwd(gu_h, rw32, go_h, 4.0, lb)
    d = to_host(dgu.view)
    check_output("dG", d[:, :I], ref.dg, ref.cg)
    rep = check_output("dU", d[:, I:], ref.du)
    assert rep["faithful_only"] <= 1e-2 * rep["n"], rep
    check_dw("d_w", to_host(d_rw), ref.dw, ref.sw)


def test_drw_not_wanted_leaves_gradients_identical(cuda_device):
    dev = cuda_device
    T, I = 97, 1024
    gu_h, rw32, go_h = case_inputs("bf16", T, I, seed=9)
    gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
    a = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    b = Guarded(T, 2 * I, 2 * I, torch.bfloat16, dev)
    d_rw = torch.empty(T, dtype=torch.float32, device=dev)
    abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, a, d_rw=d_rw), "bwd")
    abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, b, d_rw=None), "bwd")
    torch.cuda.synchronize()
    assert torch.equal(a.view.view(torch.int16), b.view.view(torch.int16))
    a.check(); b.check()


@pytest.mark.parametrize("dtype,I", [("bf16", 2048), ("bf16", 3072), ("f32", 4096)])
def test_grid_size_invariance(dtype, I, cuda_device):
    """Every output is bitwise identical whatever the number of CTAs (the
    chunked-equals-eager guarantee of NeMo `_WeightedSiTUFunction`, restated
    for a persistent grid)."""
    dev = cuda_device
    T = 300
    gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=11)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
    results = []
    prev = abi.situ_glu_set_max_ctas(0)
    try:
        for cap in (0, 1, 3, 148, 1000):
            abi.situ_glu_set_max_ctas(cap)
            out = Guarded(T, I, I, tdt, dev)
            dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
            dgu_s = Guarded(T, 2 * I, 2 * I, tdt, dev)
            d_rw = torch.empty(T, dtype=torch.float32, device=dev)
            d_rw_s = torch.empty(1, dtype=torch.float32, device=dev)
            abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, out), "fwd")
            abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, dgu, d_rw=d_rw), "bwd")
            abi.check(call_bwd(gu, I, rw[:1], abi.SITU_RW_SCALAR, 4.0, 25.0, go, dgu_s, d_rw=d_rw_s), "bwd")
            torch.cuda.synchronize()
            results.append([to_host(out.view), to_host(dgu.view), to_host(d_rw), to_host(d_rw_s)])
    finally:
        abi.situ_glu_set_max_ctas(prev)
    for other in results[1:]:
        for a, b in zip(results[0], other):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_zero_tokens(cuda_device):
    dev = cuda_device
    gu = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    rw = torch.empty(0, 1, dtype=torch.float32, device=dev)
    y = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
    assert y.shape == (0, 32)
    d_gu, d_rw = pkg.situ_glu_bwd(gu, rw, torch.empty(0, 32, dtype=torch.bfloat16, device=dev))
    assert d_gu.shape == (0, 64) and d_rw.shape == (0, 1)
    # a broadcast weight over no rows has a zero gradient
    d_scalar = torch.full((1,), 7.0, device=dev)
    pkg.situ_glu_bwd(gu, torch.ones(1, device=dev), torch.empty(0, 32, dtype=torch.bfloat16, device=dev),
                     d_rw=d_scalar)
    torch.cuda.synchronize()
    assert d_scalar.item() == 0.0


def test_side_stream(cuda_device):
    """Work is enqueued on the caller's stream."""
    dev = cuda_device
    T, I = 64, 512
    gu_h, rw32, go_h = case_inputs("bf16", T, I, seed=13)
    gu, rw = to_device(gu_h, dev), to_device(rw32, dev).reshape(T, 1)
    s = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
    s.synchronize()
    ref = oracle.load().fwd(gu_h, rw32, 4.0, 25.0)
    check_output("Y (side stream)", to_host(y), ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_autograd_function(dtype, cuda_device):
    """weighted_situ through torch.autograd: leading batch dims, the saved-input
    contract, d_routing_weights only when needed, and the unweighted situlu."""
    dev = cuda_device
    B, S, I = 3, 37, 264 if dtype == "bf16" else 132
    T = B * S
    gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=21)
    gu = to_device(gu_h, dev).reshape(B, S, 2 * I).requires_grad_(True)
    rw = to_device(rw32, dev).reshape(B, S, 1).requires_grad_(True)
    go = to_device(go_h, dev).reshape(B, S, I)
    y = pkg.weighted_situ(gu, rw, 4.0, 25.0)
    assert y.dtype == gu.dtype and y.shape == (B, S, I)
    y.backward(go)
    o = oracle.load()
    ref_y = o.fwd(gu_h, rw32, 4.0, 25.0)
    ref = o.bwd(gu_h, rw32, go_h, 4.0, 25.0)
    check_output("Y", to_host(y.reshape(T, I)), ref_y)
    g = to_host(gu.grad.reshape(T, 2 * I))
    check_output("dG", g[:, :I], ref.dg, ref.cg)
    check_output("dU", g[:, I:], ref.du)
    check_dw("d_w", to_host(rw.grad.reshape(T)), ref.dw, ref.sw)

    # routing weights that need no gradient: no reduction, gate_up grad unchanged
    gu2 = gu.detach().clone().requires_grad_(True)
    y2 = pkg.weighted_situ(gu2, rw.detach(), 4.0, 25.0)
    y2.backward(go)
    assert torch.equal(gu2.grad.view(torch.int16 if dtype == "bf16" else torch.int32),
                       gu.grad.view(torch.int16 if dtype == "bf16" else torch.int32))

    # unweighted form: w = 1
    gu3 = gu.detach().clone().requires_grad_(True)
    y3 = pkg.situlu(gu3, 4.0, None)
    y3.backward(go)
    ones = np.ones(T, dtype=np.float32)
    check_output("Y (unweighted)", to_host(y3.reshape(T, I)), o.fwd(gu_h, ones, 4.0, None))
    r3 = o.bwd(gu_h, ones, go_h, 4.0, None)
    g3 = to_host(gu3.grad.reshape(T, 2 * I))
    check_output("dG (unweighted)", g3[:, :I], r3.dg, r3.cg)
    check_output("dU (unweighted)", g3[:, I:], r3.du)


def test_errors_surface_from_the_library(cuda_device):
    dev = cuda_device
    gu = torch.zeros(4, 24, dtype=torch.bfloat16, device=dev)  # I = 12: not a 16-byte multiple
    with pytest.raises(pkg.SituError, match="MISALIGNED"):
        pkg.situ_glu_fwd(gu, torch.ones(4, 1, device=dev))
    with pytest.raises(ValueError):
        pkg.situ_glu_fwd(torch.zeros(4, 32, dtype=torch.bfloat16, device=dev), None, beta=0.0)


def assert_same_results(first, second):
    """[Y, d_gate_up, d_w] of two launch layouts.  Y and d_gate_up are computed
    element by element with the same arithmetic: bitwise equal.  d_w sums each
    row in an order fixed by how the layout assigns vectors to threads, so two
    layouts agree within its tolerance (the order is fixed per layout, which the
    grid-invariance test checks bitwise)."""
    for a, b in zip(first[:2], second[:2]):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
    da, db = first[2].astype(np.float64), second[2].astype(np.float64)
    assert np.all(np.abs(da - db) <= parity.DW_REL * np.abs(db) + 1e-6 * np.abs(db).max())


@pytest.mark.parametrize("dtype,T,I,lb", [("bf16", 257, 520, 25.0), ("bf16", 64, 3072, None),
                                          ("f32", 33, 4096, 25.0), ("bf16", 5, 8, 25.0)])
def test_load_paths_agree(dtype, T, I, lb, cuda_device):
    """The shared-memory ring (TMA bulk copies) and the direct-load path run the
    same arithmetic (see assert_same_results)."""
    dev = cuda_device
    gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=31)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    gu, go, rw = to_device(gu_h, dev), to_device(go_h, dev), to_device(rw32, dev)
    results = []
    prev = abi.situ_glu_set_load_path(0)
    try:
        for path in (0, 1):
            abi.situ_glu_set_load_path(path)
            out = Guarded(T, I, I, tdt, dev)
            dgu = Guarded(T, 2 * I, 2 * I, tdt, dev)
            d_rw = torch.empty(T, dtype=torch.float32, device=dev)
            abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, lb, out), "fwd")
            abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, lb, go, dgu, d_rw=d_rw), "bwd")
            torch.cuda.synchronize()
            out.check(); dgu.check()
            results.append([to_host(out.view), to_host(dgu.view), to_host(d_rw)])
    finally:
        abi.situ_glu_set_load_path(prev)
    assert_same_results(*results)


@pytest.mark.parametrize("dtype,T,I", [("bf16", 150, 2048), ("bf16", 33, 512), ("f32", 70, 1024)])
def test_wide_and_two_vector_layouts_agree(dtype, T, I, cuda_device):
    """Row pitches that are multiples of 32 bytes take the 256-bit-per-thread
    kernels; pitches that are only 16-byte multiples take the two-vector ones.
    Same data, same arithmetic (see assert_same_results)."""
    dev = cuda_device
    gu_h, rw32, go_h = case_inputs(dtype, T, I, seed=41)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    es = 2 if dtype == "bf16" else 4
    pad16 = 16 // es  # one extra 16-byte vector per row: pitch no longer a 32-byte multiple
    results = []
    for pad in (0, pad16):
        gpitch, opitch = 2 * I + pad, I + pad
        gu_p = np.zeros((T, gpitch), dtype=gu_h.dtype); gu_p[:, :2 * I] = gu_h
        go_p = np.zeros((T, opitch), dtype=go_h.dtype); go_p[:, :I] = go_h
        gu, go, rw = to_device(gu_p, dev), to_device(go_p, dev), to_device(rw32, dev)
        out = Guarded(T, I, opitch, tdt, dev)
        dgu = Guarded(T, 2 * I, gpitch, tdt, dev)
        d_rw = torch.empty(T, dtype=torch.float32, device=dev)
        abi.check(call_fwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, out), "fwd")
        abi.check(call_bwd(gu, I, rw, abi.SITU_RW_ROW, 4.0, 25.0, go, dgu, d_rw=d_rw), "bwd")
        torch.cuda.synchronize()
        out.check(); dgu.check()
        results.append([to_host(out.view), to_host(dgu.view), to_host(d_rw)])
    assert_same_results(*results)
    o = oracle.load()
    check_output("Y", results[0][0], o.fwd(gu_h, rw32, 4.0, 25.0))


def test_no_bounded_wait_expired(cuda_device):
    """No kernel launched by the tests above gave up on a shared-memory stage."""
    assert abi.situ_glu_device_status(0) == 0


def test_expired_wait_sets_the_status_and_the_context_survives(cuda_device):
    """A bounded wait that runs out: the probe waits 5 ms on an mbarrier that
    nothing completes, gives up, sets the status word and returns.  The host
    reads 1, clears it, and the next launches on the same context still match
    the oracle."""
    assert abi.situ_glu_device_status(1) == 0
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    abi.check(abi.situ_glu_wait_probe(5_000_000, stream), "wait probe")
    assert abi.situ_glu_device_status(1) == 1
    assert abi.situ_glu_device_status(0) == 0
    wl = workloads.workload(0)
    x = workloads.inputs(wl, tokens=64)
    gu = to_device(x["gate_up"], cuda_device)
    rw = to_device(x["routing_weights"], cuda_device).reshape(64, 1)
    y = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
    torch.cuda.synchronize()
    check_output("Y after an expired wait", to_host(y), oracle.load().fwd(x["gate_up"], x["routing_weights"], 4.0, 25.0))
    assert abi.situ_glu_device_status(0) == 0
