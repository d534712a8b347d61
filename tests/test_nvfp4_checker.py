"""The NVFP4 parity checker (parity.check_nvfp4) on the CPU: it accepts the
oracle's own NVFP4 quantisation of a matrix and rejects plausible kernel
mistakes (a block scale one step off, a code one step off, a flipped sign,
swapped nibbles, a missing NaN scale, a wrong tensor maximum, the per-tensor
scale left out)."""
import numpy as np
import pytest

import oracle
from parity import check_nvfp4, unpack_e2m1


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def _matrix(seed=6):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((7, 96)) * np.exp2(rng.integers(-6, 6, (7, 1)))
    v[2, 3] = np.nan
    v[4, 32:48] = 0.0
    v[5, 16:32] *= 1e-9   # block scale underflows to zero
    return v


def _quantised(v):
    o = oracle.load()
    codes, scales, s = o.nvfp4_quantize(v)
    amax = float(np.abs(v[np.isfinite(v)]).max())
    return pack_e2m1(codes), scales.copy(), amax


def test_unpack_round_trip():
    c = np.arange(32, dtype=np.uint8).reshape(2, 16) & 0xF
    assert np.array_equal(unpack_e2m1(pack_e2m1(c)), c)
    assert unpack_e2m1(np.array([[0x21]], dtype=np.uint8)).tolist() == [[1, 2]]


def test_checker_accepts_the_oracle():
    v = _matrix()
    packed, scales, amax = _quantised(v)
    rep = check_nvfp4("oracle", packed, scales, amax, v, 1e-9 * np.abs(np.nan_to_num(v)))
    assert rep["exact"] == rep["codes"] and rep["scales_equal"] == 1.0


@pytest.mark.parametrize("mistake", ["scale+1", "code+1", "sign", "nibbles", "nan_scale", "amax*2", "no_tensor_scale"])
def test_checker_rejects_mistakes(mistake):
    o = oracle.load()
    v = _matrix()
    packed, scales, amax = _quantised(v)
    tol = 1e-9 * np.abs(np.nan_to_num(v))
    codes = unpack_e2m1(packed)
    if mistake == "scale+1":
        scales[1, 2] += 1
    elif mistake == "code+1":
        i = int(np.flatnonzero((codes[6] & 7) < 6)[0])
        codes[6, i] += 1
    elif mistake == "sign":
        i = int(np.flatnonzero(codes[3] & 7)[0])
        codes[3, i] ^= 8
    elif mistake == "nibbles":
        k = int(np.flatnonzero(codes[0, 0::2] != codes[0, 1::2])[0])
        codes[0, 2 * k], codes[0, 2 * k + 1] = codes[0, 2 * k + 1], codes[0, 2 * k]
    elif mistake == "nan_scale":
        scales[2, 0] = 0x00
    elif mistake == "amax*2":
        amax *= 2
    elif mistake == "no_tensor_scale":
        c, sc, _ = o.nvfp4_quantize(v, s_enc=1.0)
        codes, scales = c, sc
    with pytest.raises(AssertionError):
        check_nvfp4("mistake", pack_e2m1(codes), scales, amax, v, tol)
