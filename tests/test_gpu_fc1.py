"""GPU parity of the fused FC1 grouped GEMM + SiTU-GLU forward
(situ_glu_fc1_fwd) against the fp64 oracle (oracle/fc1_oracle.c).

Tolerance: the bf16 rule of parity.py (2^-8 relative + 1e-6, or a faithful
rounding) plus 2^-18 times the oracle's accumulation-error scale
|dY/dG| sum_k |x w_g| + |dY/dU| sum_k |x w_u|.  A tensor-core fp32
accumulation of H products stays far inside 2^-18 of that sum (its typical
error is about 2^-24 of it), while a missing K slice, a wrong expert or a
swapped half moves Y by percents.

Small cases cover every element: several experts (empty ones, one-row ones,
ragged row tails), rows outside every expert (which must stay untouched),
every routing-weight form and gate-exponent form.  The routed-MoE
FC1 (32768 rows, hidden 7168, 8 experts) is compared in full.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import CANCEL, as_f64, bf16_faithful, by_row_chunks, to_device, to_host

pytestmark = pytest.mark.gpu

SENTINEL_BF16 = 0x7FC1  # a NaN pattern the kernel never writes


def check_fc1(name, got_bits, ref, err):
    y = as_f64(got_bits)
    diff = np.abs(y - ref)
    ok = (diff <= 2.0 ** -8 * np.abs(ref) + 1e-6 + CANCEL * err) | bf16_faithful(got_bits, ref)
    bad = np.flatnonzero(~ok)
    if bad.size:
        i = bad[0]
        raise AssertionError(f"{name}: {bad.size} of {ok.size} out of tolerance; first at flat {i}: got "
                             f"{y.flat[i]!r}, oracle {ref.flat[i]!r}, error scale {err.flat[i]!r}")


def run_fc1(dev, T, H, I, offsets, beta=4.0, lb=25.0, kind="row_f32", seed=0, check_rows=None):
    E = len(offsets) - 1
    d = workloads.fc1_inputs(T, H, I, E, seed)
    x_h, w1_h, rw32 = d["x"], d["w1"], d["routing_weights"]
    offsets = np.asarray(offsets, dtype=np.int64)
    x, w1 = to_device(x_h, dev), to_device(w1_h, dev)
    off = torch.from_numpy(offsets).to(dev)
    if kind == "row_f32":
        rw, rw_o = to_device(rw32, dev).reshape(T, 1), rw32
    elif kind == "row_bf16":
        bits = workloads.f32_to_bf16_bits(rw32)
        rw, rw_o = to_device(bits, dev).reshape(T, 1), workloads.bf16_bits_to_f32(bits)
    elif kind == "scalar":
        rw, rw_o = to_device(rw32[:1].copy(), dev), np.full(T, rw32[0], dtype=np.float32)
    else:
        rw, rw_o = None, None
    y = torch.full((T, I), SENTINEL_BF16, dtype=torch.int16, device=dev).view(torch.bfloat16)
    pkg.situ_glu_fc1_fwd(x, w1, off, rw, beta, lb, out=y)
    torch.cuda.synchronize()
    assert pkg.abi.situ_glu_device_status(0) == 0
    got = to_host(y)
    lo, hi = int(max(0, offsets[0])), int(min(T, offsets[-1]))
    assert np.all(got[:lo] == SENTINEL_BF16) and np.all(got[hi:] == SENTINEL_BF16), "wrote outside the experts"
    rows = np.arange(lo, hi) if check_rows is None else np.asarray(check_rows, dtype=np.int64)
    o = oracle.load()
    ref, err, _ = by_row_chunks(lambda r: o.fc1_fwd(x_h, w1_h, offsets, I, rw_o, beta, lb, rows=r), rows)
    check_fc1("Y", got[rows], ref, err)
    return got


@pytest.mark.parametrize("T,H,I,offsets", [
    (128, 64, 128, [0, 128]),                      # one tile, one K slice
    (300, 256, 256, [0, 100, 100, 300]),           # empty expert, ragged tails
    (517, 192, 384, [3, 4, 5, 129, 300, 510]),     # one-row experts; rows outside every expert
    (1000, 512, 128, list(range(0, 1001, 40))),    # 25 experts of 40 rows
])
def test_fc1_small(T, H, I, offsets, cuda_device):
    run_fc1(cuda_device, T, H, I, offsets, seed=T + H)


@pytest.mark.parametrize("beta,lb,kind", [(4.0, 25.0, "row_bf16"), (1.0, None, "scalar"), (2.0, 1.5, "none"),
                                          (16.0, None, "row_f32")])
def test_fc1_forms(beta, lb, kind, cuda_device):
    run_fc1(cuda_device, 260, 128, 256, [0, 7, 260], beta=beta, lb=lb, kind=kind, seed=11)


def test_fc1_random_split_many_experts(cuda_device):
    T, E = 2000, 64
    off = workloads.expert_offsets(T, E, seed=5, skew=0.3)
    run_fc1(cuda_device, T, 256, 128, off, seed=5)


def test_fc1_grid_invariant(cuda_device):
    outs = []
    for ctas in (0, 1, 5):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_fc1(cuda_device, 600, 128, 256, [0, 250, 600], seed=3))
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        assert np.array_equal(other, outs[0])


def test_fc1_routed_moe_size_every_row(cuda_device):
    """The routed-MoE FC1: 32768 token rows over 8 local experts (an uneven
    split), hidden 7168, I = 2048: every row against the oracle (on the
    host's threads)."""
    T, H, I, E = 32768, 7168, 2048, 8
    off = workloads.expert_offsets(T, E, seed=21, skew=2.0)
    run_fc1(cuda_device, T, H, I, off, seed=21)


def test_fc1_zero_tokens(cuda_device):
    dev = cuda_device
    x = torch.empty(0, 64, dtype=torch.bfloat16, device=dev)
    w1 = torch.zeros(2 * 128, 64, dtype=torch.bfloat16, device=dev)
    off = torch.zeros(2, dtype=torch.int64, device=dev)
    y = pkg.situ_glu_fc1_fwd(x, w1, off, None)
    assert y.shape == (0, 128)
