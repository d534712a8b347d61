"""GPU tests of HostPipeline: forward + backward over host tensors streamed
through the GPU in row chunks (uploads, kernels and downloads of successive
chunks on three streams).  The outputs must equal, bit for bit, the same
kernels run on the whole device-resident problem (rows are independent and
the kernels' results do not depend on the launch size), including a ragged
last chunk, no routing weights, fp32 storage and a reused pipeline."""
import dataclasses

import numpy as np
import pytest
import torch

import workloads
import ffn_gated_activation_b200 as pkg

from parity import to_host

pytestmark = pytest.mark.gpu


def host(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
    return t.pin_memory()


@pytest.mark.parametrize("dtype,T,I,chunk,weighted", [("bf16", 5000, 512, 1024, True), ("bf16", 700, 256, 4096, True),
                                                     ("bf16", 3000, 1024, 512, False), ("f32", 1500, 256, 640, True)])
def test_host_pipeline_matches_device_run(dtype, T, I, chunk, weighted, cuda_device):
    wl = dataclasses.replace(workloads.workload(2), dtype=dtype, tokens=T, inter=I, seed=5000 + T, rw_kind="uniform")
    x = workloads.inputs(wl)
    gu_h, go_h = host(x["gate_up"]), host(x["grad_out"])
    rw_h = host(x["routing_weights"].reshape(T, 1)) if weighted else None
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    pipe = pkg.HostPipeline(I, dt, chunk_rows=chunk, device=cuda_device)
    for _ in range(2):  # the second run reuses the ring
        y, dgu, drw = pipe.run(gu_h, rw_h, go_h, 4.0, 25.0)
        torch.cuda.synchronize()
    gu, go = gu_h.to(cuda_device), go_h.to(cuda_device)
    rw = rw_h.to(cuda_device) if weighted else None
    y_ref = pkg.situ_glu_fwd(gu, rw, 4.0, 25.0)
    dgu_ref, drw_ref = pkg.situ_glu_bwd(gu, rw, go, 4.0, 25.0)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(y), to_host(y_ref))
    assert np.array_equal(to_host(dgu), to_host(dgu_ref))
    if weighted:
        assert np.array_equal(to_host(drw), to_host(drw_ref))
    else:
        assert drw is None


def test_host_pipeline_rejects_bad_inputs(cuda_device):
    pipe = pkg.HostPipeline(64, torch.bfloat16, chunk_rows=16, device=cuda_device)
    gu = torch.zeros(10, 128, dtype=torch.bfloat16)
    go = torch.zeros(10, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pipe.run(gu, torch.ones(10), go)                     # not [T, 1]
    with pytest.raises(TypeError):
        pipe.run(gu.float(), None, go.float())               # wrong dtype
    with pytest.raises(ValueError):
        pipe.run(gu.to(cuda_device), None, go)               # device input
