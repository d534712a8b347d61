"""The seeded input generators (CPU): determinism, rounding, distributions."""
import numpy as np
import torch

import workloads


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 3, 100000), rng.uniform(-70, 70, 1000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1e-40]]).astype(np.float32)
    ours = workloads.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(workloads.bf16_bits_to_f32(ours),
                          torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generation_is_deterministic_and_thread_independent(monkeypatch):
    wl = workloads.workload(2)
    a = workloads.inputs(wl, tokens=300)
    monkeypatch.setattr(workloads, "_threads", lambda: 1)
    b = workloads.inputs(wl, tokens=300)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    # a prefix of a larger draw is the smaller draw (block-keyed streams)
    c = workloads.gate_up(wl, tokens=200)
    assert np.array_equal(c, a["gate_up"][:200])


def test_distributions():
    wl = workloads.workload(1)
    x = workloads.inputs(wl, tokens=512)
    g = workloads.bf16_bits_to_f32(x["gate_up"])
    assert abs(g[:, :wl.inter].std() - 2.0) < 0.02
    assert abs(g[:, wl.inter:].std() - 1.0) < 0.01
    assert np.all(x["routing_weights"] == 1.0)
    go = workloads.bf16_bits_to_f32(x["grad_out"])
    assert abs(go.std() - 0.1) < 0.002


def test_routed_moe_outliers_and_topk_weights():
    wl = workloads.workload(2)
    x = workloads.inputs(wl, tokens=1024)
    g = workloads.bf16_bits_to_f32(x["gate_up"]).astype(np.float64)
    big = np.abs(g) >= 20.0
    frac = big.mean()
    assert 0.008 < frac < 0.012                  # ~1 % outliers
    assert np.abs(g).max() <= 60.0
    assert abs(np.sign(g[big]).mean()) < 0.1     # fair sign
    rw = x["routing_weights"].reshape(-1, wl.topk)
    assert np.all(rw > 0) and np.all(rw < 1)
    assert np.all(np.diff(rw, axis=1) <= 0)      # top-k in descending order
    assert np.all(rw.sum(axis=1) < 1.0)          # not renormalised over the top 8


def test_fp32_workload_storage():
    wl = workloads.workload(3)
    x = workloads.inputs(wl, tokens=64)
    assert x["gate_up"].dtype == np.float32 and x["grad_out"].dtype == np.float32
    assert x["gate_up"].shape == (64, 2 * wl.inter)
    assert wl.linear_beta is None and wl.betas == (1.0, 4.0, 16.0)


def test_algorithmic_bytes():
    # fwd = T (2 I s + 4 + I s); bwd = T (2 I s + I s + 4 + 2 I s + 4)
    assert workloads.workload(0).fwd_bytes() == 787_456
    assert workloads.workload(0).bwd_bytes() == 1_312_768
    assert workloads.workload(2).fwd_bytes() == 402_784_256
    assert workloads.workload(3).bwd_bytes() == 1_342_308_352
    assert workloads.workload(4).fwd_bytes() == 3_221_749_760


def test_elementwise_weight_generators_are_prefix_stable():
    wl = workloads.workload(0)
    a = workloads.element_weights(wl, tokens=130, inter=24)
    b = workloads.element_weights(wl, tokens=70, inter=24)
    assert a.dtype == np.float32 and a.shape == (130, 24)
    assert np.array_equal(a[:70], b)
    assert np.all((a >= 0) & (a < 1))
    c = workloads.column_weights(wl, inter=24)
    assert c.shape == (24,) and np.array_equal(c, workloads.column_weights(wl, inter=24))
