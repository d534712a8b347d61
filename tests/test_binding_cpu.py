"""CPU checks of the Python binding's host logic: the validation of caller
output buffers (the library sees a pointer and a row pitch only, so the
binding must refuse a buffer the kernels would write past) and the
routing-weight classification's fast path for [T, 1] weights."""
import pytest
import torch

from ffn_gated_activation_b200 import abi
from ffn_gated_activation_b200 import functional as F

CPU = torch.device("cpu")


def test_given_accepts_a_matching_buffer():
    t = torch.empty(6, 8, dtype=torch.bfloat16)
    v = F._given(t, (6, 8), CPU, "out", torch.bfloat16)
    assert v.data_ptr() == t.data_ptr() and tuple(v.shape) == (6, 8)
    t3 = torch.empty(2, 3, 8, dtype=torch.float32)
    v3 = F._given(t3, (2, 3, 8), CPU, "out", torch.float32)
    assert tuple(v3.shape) == (6, 8) and v3.stride(0) == 8
    wide = torch.empty(6, 24, dtype=torch.uint8)  # rows with a pitch: a column slice
    v = F._given(wide[:, 8:16], (6, 8), CPU, "MXFP8 data")
    assert v.stride(0) == 24 and v.stride(1) == 1
    assert F._given(torch.empty(0, 8), (0, 8), CPU, "out", torch.float32).numel() == 0


@pytest.mark.parametrize("case", ["short", "long", "wide", "dtype", "one_byte", "device", "strided", "overlap",
                                  "not_a_view"])
def test_given_refuses(case):
    shape, dtype, device = (6, 8), torch.bfloat16, CPU
    t = torch.empty(6, 8, dtype=torch.bfloat16)
    if case == "short":
        t = torch.empty(5, 8, dtype=torch.bfloat16)
    elif case == "long":
        t = torch.empty(7, 8, dtype=torch.bfloat16)
    elif case == "wide":
        t = torch.empty(6, 9, dtype=torch.bfloat16)
    elif case == "dtype":
        t = torch.empty(6, 8, dtype=torch.float32)
    elif case == "one_byte":
        t, dtype = torch.empty(6, 8, dtype=torch.int16), None
    elif case == "device":
        device = torch.device("cuda", 0)
    elif case == "strided":
        t = torch.empty(6, 16, dtype=torch.bfloat16)[:, ::2]
    elif case == "overlap":
        t = torch.empty(64, dtype=torch.bfloat16).as_strided((6, 8), (4, 1))
    elif case == "not_a_view":
        t = torch.empty(3, 8, 2, dtype=torch.bfloat16).transpose(1, 2)  # [3, 2, 8], rows not evenly spaced
        shape = (3, 2, 8)
    with pytest.raises((ValueError, TypeError)):
        F._given(t, shape, device, "out", dtype)


def test_given_drw():
    rw = torch.empty(6, 1)
    assert F._given_drw(torch.empty(6, 1), rw, CPU).shape == (6, 1)
    for bad in (torch.empty(6), torch.empty(6, 1, dtype=torch.bfloat16), torch.empty(5, 1)):
        with pytest.raises(ValueError):
            F._given_drw(bad, rw, CPU)
    with pytest.raises(ValueError):
        F._given_drw(torch.empty(6, 1), rw, torch.device("cuda", 0))


@pytest.mark.parametrize("make", [lambda: torch.rand(9, 1), lambda: torch.rand(9, 4)[:, 2:3],
                                  lambda: torch.rand(1, 1).expand(9, 1)])
def test_row_weights_fast_path_matches_the_flat_view(make):
    """[T, 1] weights go to the library as they are, with their row stride:
    the same address and stride as the flat view the general path takes."""
    rw = make()
    mode, view, stride = F.routing_mode((9,), 16, rw)
    assert mode == abi.SITU_RW_ROW
    flat = rw.reshape(-1)
    assert view.data_ptr() == flat.data_ptr() and stride == flat.stride(0)
    # a leading shape of more than one axis takes the general path
    mode3, view3, stride3 = F.routing_mode((3, 3), 16, rw.reshape(3, 3, 1))
    assert mode3 == abi.SITU_RW_ROW and view3.dim() == 1
