"""GPU parity of the fused FC2 data gradient + SiTU-GLU backward
(situ_glu_fc2_dgrad_bwd) against the fp64 oracle (oracle/fc2_oracle.c).

Tolerance: dG and dU follow the bf16 rule of parity.py (2^-8 relative +
1e-6, or a faithful rounding) plus 2^-18 times the oracle's error scale (the
fp32 accumulation of H products into dY, and for dG the uncancelled
magnitude of T_g'); d_w within 1e-4 |ref| + 2^-18 times its scale.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import CANCEL, DW_REL, as_f64, bf16_faithful, by_row_chunks, to_device, to_host

pytestmark = pytest.mark.gpu

SENTINEL_BF16 = 0x7FC1


def run_fc2(dev, T, H, I, offsets, beta=4.0, lb=25.0, weights=True, rw_bf16=False, seed=0, check_rows=None):
    E = len(offsets) - 1
    d = workloads.fc2_inputs(T, H, I, E, seed)
    offsets = np.asarray(offsets, dtype=np.int64)
    dout, w2t, gu = to_device(d["dout"], dev), to_device(d["w2t"], dev), to_device(d["gate_up"], dev)
    off = torch.from_numpy(offsets).to(dev)
    rw32 = d["routing_weights"]
    rw_o = None
    rw = None
    if weights:
        if rw_bf16:
            bits = workloads.f32_to_bf16_bits(rw32)
            rw, rw_o = to_device(bits, dev).reshape(T, 1), workloads.bf16_bits_to_f32(bits)
        else:
            rw, rw_o = to_device(rw32, dev).reshape(T, 1), rw32
    dgu = torch.full((T, 2 * I), SENTINEL_BF16, dtype=torch.int16, device=dev).view(torch.bfloat16)
    d_rw = torch.full((T, 1), float("nan"), dtype=rw.dtype, device=dev) if weights else None
    pkg.situ_glu_fc2_dgrad_bwd(dout, w2t, off, gu, rw, beta, lb, d_gate_up=dgu, d_rw=d_rw)
    torch.cuda.synchronize()
    assert pkg.abi.situ_glu_device_status(0) == 0
    got = to_host(dgu)
    lo, hi = int(max(0, offsets[0])), int(min(T, offsets[-1]))
    assert np.all(got[:lo] == SENTINEL_BF16) and np.all(got[hi:] == SENTINEL_BF16), "wrote outside the experts"
    rows = np.arange(lo, hi) if check_rows is None else np.asarray(check_rows, dtype=np.int64)
    o = oracle.load()
    ref, dw, _, err, dw_err = by_row_chunks(
        lambda r: o.fc2_dgrad(d["dout"], d["w2t"], offsets, d["gate_up"], rw_o, beta, lb, rows=r), rows)
    g = got[rows]
    y = as_f64(g)
    ok = (np.abs(y - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 + CANCEL * err) | bf16_faithful(g, ref)
    bad = np.flatnonzero(~ok)
    assert bad.size == 0, (f"{bad.size} of {ok.size} out of tolerance; first: got {y.flat[bad[0]]!r}, oracle "
                           f"{ref.flat[bad[0]]!r}, scale {err.flat[bad[0]]!r}")
    if weights:
        gd = as_f64(to_host(d_rw).reshape(-1)[rows])
        tol = DW_REL * np.abs(dw) + CANCEL * dw_err + (2.0 ** -8 * np.abs(dw) if rw_bf16 else 0.0)
        assert np.all(np.abs(gd - dw) <= tol), np.max(np.abs(gd - dw) / np.maximum(tol, 1e-300))
    return got


@pytest.mark.parametrize("T,H,I,offsets", [
    (128, 64, 256, [0, 128]),
    (300, 192, 512, [0, 100, 100, 300]),
    (517, 128, 256, [3, 4, 5, 129, 300, 510]),
    (1000, 256, 256, list(range(0, 1001, 40))),
])
def test_fc2_small(T, H, I, offsets, cuda_device):
    run_fc2(cuda_device, T, H, I, offsets, seed=T + H)


@pytest.mark.parametrize("beta,lb,weights,rw_bf16", [(4.0, 25.0, True, True), (1.0, None, True, False),
                                                     (2.0, 1.5, False, False), (16.0, None, True, False)])
def test_fc2_forms(beta, lb, weights, rw_bf16, cuda_device):
    run_fc2(cuda_device, 260, 128, 256, [0, 7, 260], beta=beta, lb=lb, weights=weights, rw_bf16=rw_bf16, seed=13)


def test_fc2_grid_invariant(cuda_device):
    outs = []
    for ctas in (0, 1, 5):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_fc2(cuda_device, 600, 128, 512, [0, 250, 600], seed=3))
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        assert np.array_equal(other, outs[0])


def test_fc2_routed_moe_size_every_row(cuda_device):
    """The routed-MoE FC2 data gradient: 32768 token rows over 8 local experts
    (an uneven split), hidden 7168, I = 2048: every row against the oracle (on
    the host's threads)."""
    T, H, I, E = 32768, 7168, 2048, 8
    off = workloads.expert_offsets(T, E, seed=22, skew=2.0)
    run_fc2(cuda_device, T, H, I, off, seed=22)
