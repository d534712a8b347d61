"""GPU parity of the attention-residual mixing core (situ_attn_res_fwd)
against the fp64 oracle (oracle/attn_res_oracle.c).

Tolerance: a bf16 output must be within 2^-8 |ref| + 1e-6 + 2^-18 M of the
oracle (M = sum_b prob_b |x_b|, the scale of the combine's rounding: the
fp32 sums over hidden, the approximate rsqrt and exp of the softmax move the
probabilities by a few 1e-7 relative, ten times below 2^-18), or be a
faithful bf16 rounding of it; an fp32 output within 1e-5 |ref| + 2^-18 M.  The probabilities enter every element of a
row, so a wrong norm, epsilon, weight or source order fails whole rows.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import workloads
from ffn_gated_activation_b200 import abi
import ffn_gated_activation_b200 as pkg

from parity import check_ar, to_device, to_host

pytestmark = pytest.mark.gpu


def run_ar(dev, T, B, H, with_prefix=True, dtype="bf16", out_dtype=torch.bfloat16, weights_bf16=False, seed=0,
           eps=1e-6, rows=None):
    d = workloads.attn_res_inputs(T, B, H, seed, dtype)
    blocks_h, prefix_h = d["blocks"], (d["prefix"] if with_prefix else None)
    nw_h, pw_h = d["norm_weight"], d["proj_weight"]
    if weights_bf16:
        nw_h, pw_h = workloads.f32_to_bf16_bits(nw_h), workloads.f32_to_bf16_bits(pw_h)
    blocks = to_device(blocks_h, dev) if B > 0 else None
    prefix = to_device(prefix_h, dev) if prefix_h is not None else None
    nw, pw = to_device(nw_h, dev), to_device(pw_h, dev)
    if prefix is not None and blocks is not None:
        out = pkg.apply_attn_res(prefix, blocks, pw, nw, eps, out_dtype)
    elif blocks is not None:
        out = pkg.attn_res_core(blocks, nw, pw, eps, out_dtype)
    else:
        out = pkg.apply_attn_res(prefix, torch.empty(T, 0, H, dtype=prefix.dtype, device=dev), pw, nw, eps, out_dtype)
    torch.cuda.synchronize()
    got = to_host(out)
    o = oracle.load()
    ref, mag, _ = o.attn_res(blocks_h if B > 0 else None, prefix_h, nw_h, pw_h, eps, rows=rows)
    check_ar("out", got if rows is None else got[rows], ref, mag)
    return got


@pytest.mark.parametrize("T,B,H", [(1, 1, 8), (3, 2, 64), (257, 8, 512), (130, 3, 7168), (64, 15, 1024),
                                   (37, 5, 1032),  # 129 vectors a row: two per thread, the last thread one
                                   (50, 8, 8192), (33, 8, 7176)])  # 1024 and 897 vectors: 512 and 480 threads
def test_attn_res_bf16(T, B, H, cuda_device):
    run_ar(cuda_device, T, B, H, seed=T + B)


@pytest.mark.parametrize("T,B,H", [(33, 4, 256), (70, 8, 4096), (40, 8, 2048), (21, 4, 1028)])
def test_attn_res_fp32_values_and_output(T, B, H, cuda_device):
    run_ar(cuda_device, T, B, H, dtype="f32", out_dtype=torch.float32, seed=7)


def test_attn_res_forms(cuda_device):
    dev = cuda_device
    run_ar(dev, 50, 6, 256, with_prefix=False, seed=1)                       # _attn_res_core: one stacked array
    run_ar(dev, 50, 0, 256, with_prefix=True, seed=2)                        # only the current sum
    run_ar(dev, 50, 5, 256, weights_bf16=True, out_dtype=torch.float32, seed=3)
    run_ar(dev, 50, 5, 256, eps=0.0, seed=4)


def test_attn_res_strided_sources(cuda_device):
    """Block sums taken from a wider stacked tensor (a view), the prefix sum a column slice."""
    dev = cuda_device
    T, B, H = 40, 4, 512
    d = workloads.attn_res_inputs(T, B + 2, H, 9)
    big = to_device(d["blocks"], dev)              # [T, B + 2, H]
    blocks = big[:, 1:B + 1]                      # strided view of B sources
    wide = torch.zeros(T, 2 * H, dtype=torch.bfloat16, device=dev)
    wide[:, H:] = to_device(d["prefix"], dev)
    prefix = wide[:, H:]
    nw, pw = to_device(d["norm_weight"], dev), to_device(d["proj_weight"], dev)
    out = pkg.apply_attn_res(prefix, blocks, pw, nw, 1e-6)
    torch.cuda.synchronize()
    ref, mag, _ = oracle.load().attn_res(np.ascontiguousarray(d["blocks"][:, 1:B + 1]), d["prefix"],
                                         d["norm_weight"], d["proj_weight"], 1e-6)
    check_ar("strided", to_host(out), ref, mag)


def test_attn_res_grid_invariant(cuda_device):
    outs = []
    for ctas in (0, 1, 3):
        prev = abi.situ_glu_set_max_ctas(ctas)
        try:
            outs.append(run_ar(cuda_device, 90, 8, 1024, seed=5))
        finally:
            abi.situ_glu_set_max_ctas(prev)
    for other in outs[1:]:
        assert np.array_equal(other, outs[0])


def test_attn_res_full_size_sampled_rows(cuda_device):
    """16384 tokens, 8 stored sums + the current sum, hidden 7168: 64 sampled rows."""
    rows = np.random.default_rng(3).choice(16384, 64, replace=False)
    run_ar(cuda_device, 16384, 8, 7168, seed=11, rows=np.sort(rows))


def test_attn_res_full_size_every_element(cuda_device):
    """The bench's workload (16384 tokens, 8 stored sums + the current sum,
    hidden 7168, bf16) in the bench's launch configuration: every output
    element against the oracle, in row chunks over the host's threads."""
    dev = cuda_device
    T, B, H = 16384, 8, 7168
    d = workloads.attn_res_inputs(T, B, H, 2)
    blocks, prefix = to_device(d["blocks"], dev), to_device(d["prefix"], dev)
    nw, pw = to_device(d["norm_weight"], dev), to_device(d["proj_weight"], dev)
    out = pkg.apply_attn_res(prefix, blocks, pw, nw, 1e-6)
    torch.cuda.synchronize()
    got = to_host(out)
    del out, blocks, prefix
    o = oracle.load()

    def chunk(r0):
        rows = np.arange(r0, min(T, r0 + 256), dtype=np.int64)
        ref, mag, _ = o.attn_res(d["blocks"], d["prefix"], d["norm_weight"], d["proj_weight"], 1e-6, rows=rows)
        check_ar(f"out rows {r0}..{rows[-1]}", got[rows], ref, mag)

    with ThreadPoolExecutor(max_workers=max(1, min(96, os.cpu_count() or 1))) as pool:
        list(pool.map(chunk, range(0, T, 256)))
